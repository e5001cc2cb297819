"""Throughput of the SVDQuant W4A4 NVFP4 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = the whole per-forward path on one batch of synthetic input:
svdq_quantize_act (smooth + NVFP4 quantize + low-rank down) then
svdq_w4a4_linear (block-scaled FP4 GEMM + fused epilogue).  The one-time
svdq_repack_weights is timed separately (config.repack_us).

Metric: TFLOP/s = (2 M N K + 2 M R (K + N)) / step time.  Default workload:
the qkv projection of a 30-block DiT, M = 4352 tokens, K = 3840,
N = 11520, R = 128.  Inputs rotate over several sets whose total exceeds
the 126 MB L2, so every step reads weights and activations from HBM.

Under torchrun each rank runs its own batch of the same shape (the layer
is independent per token: weak scaling, no collective on the data path);
the time is the max over ranks.

Prints one JSON line (rank 0).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "SVDQ W4A4 linear TFLOP/s & % of dense NVFP4 roofline at DiT shapes"
SMALL_M = 64          # svdq_w4a4_linear runs its few-token GEMM at M <= 64
PAIR_M = 129          # ... and its CTA-pair GEMM at M >= 129
UNIT = "TFLOP/s"
R = 128
L2_BYTES = 126 * 1024 * 1024
FP4_OVER_BF16 = 4.0   # nominal dense FP4 : BF16 tensor ratio (9 : 2.25 PFLOP/s)


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qkv_m4352_k3840_n11520")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end (host buffer) measurement")
    ap.add_argument("--no-graph", action="store_true",
                    help="stack workloads: skip the CUDA-graph replay measurement")
    ap.add_argument("--unfused-w2", action="store_true",
                    help="stack workloads: form w2's input with svdq_silu_mul in HBM, then "
                         "quantize it (for comparison with the fused activation kernel)")
    return ap.parse_args(argv)


def flops_per_step(M, K, N, r=R):
    return 2 * M * N * K + 2 * M * r * (K + N)


def is_plain(workload):
    """Workloads of the plain NVFP4 layer (no low-rank branch, no smoothing)."""
    return workload.startswith("nvfp4_")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, \
            "fallback"


KERNEL_SOURCES = {
    "w4a4_linear_kernel": "kg_w4a4_linear.cuh",
    "w4a4_linear_pair_kernel": "kg2_w4a4_linear_pair.cuh",
    "quantize_act_kernel": "kq_quantize_act.cuh",
}


def kernel_source_hash(kernel_key):
    import hashlib
    path = os.path.join(ROOT, "nvfp4_w4a4_quantized_smooth_b200", "csrc",
                        KERNEL_SOURCES[kernel_key])
    with open(path, "rb") as f:
        return hashlib.sha1(f.read()).hexdigest()[:12]


def load_traffic(kernel_key):
    """Per-launch DRAM bytes (read + write) of a kernel from the committed ncu
    summary, or None if there is none or the kernel source changed since the
    counters were taken (each line carries the source hash it was taken at)."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        for line in open(path):
            parts = line.split()
            if len(parts) >= 3 and parts[0] == kernel_key:
                if parts[2] != kernel_source_hash(kernel_key):
                    return None
                return float(parts[1])
    except OSError:
        pass
    return None


# ------------------------------------------------------------ clocks ----

class ClockSampler:
    """nvidia-smi samples (SM clock, throttle reasons) while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 8:
                self.samples.append(parts)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(s[0]) for s in self.samples if s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for s in self.samples:
            for n, v in zip(names, s[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(self.samples)}


# -------------------------------------------------------- distributed ----

def dist_setup(backend="nccl"):
    """Join the job torchrun started (RANK / WORLD_SIZE / MASTER_* from the
    environment).  Ranks are independent replicas: the only collectives are
    the barriers around the timed region and the max of the elapsed times.
    `gloo` (CPU) serves the host-side tests of this logic."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=120)
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout,
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=timeout)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value, world):
    """Max of a per-rank float over all ranks (every rank gets it)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(workload, rank):
    """Each rank draws its own token batch (weak scaling: independent
    problems of the same shape on every GPU)."""
    from nvfp4_w4a4_quantized_smooth_b200 import synth
    return synth.workload_seed(workload) + 7919 * rank


def job_value(flops_one_step, steps, world, elapsed_ms):
    """Whole-job TFLOP/s: the work of every rank over the slowest rank's time."""
    return flops_one_step * steps * world / (elapsed_ms * 1e-3) / 1e12


# ------------------------------------------------------ our CUDA path ----

def make_sets(M, K, N, nsets, seed, dev, plain=False):
    import torch
    from nvfp4_w4a4_quantized_smooth_b200 import svdq, synth
    sets = []
    for i in range(nsets):
        L = synth.make_layer(M, K, N, seed=seed + i)
        d = {k: (None if v is None else v.to(dev)) for k, v in vars(L).items()}
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        e0.record()
        d["wscales_tiled"] = svdq.repack_weights(d["wscales"])
        e1.record()
        d["repack_s"] = time.perf_counter() - t0
        e1.synchronize()
        d["repack_gpu_ms"] = e0.elapsed_time(e1)
        d["proj_up_folded"] = None
        d["fold_gpu_ms"] = 0.0
        if not plain:
            # the up-projection folded into the accumulator's units, once
            # per weight (kept unfolded if some element does not fold)
            e0.record()
            folded, bad = svdq.fold_proj_up(d["proj_up"], d["wcscales"], d["wtscale"])
            e1.record()
            e1.synchronize()
            d["fold_gpu_ms"] = e0.elapsed_time(e1)
            d["proj_up_folded"] = folded if bad == 0 else None
        d["qact"] = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
        d["asc"] = torch.empty(svdq.ascales_tiled_bytes(M, K), dtype=torch.uint8, device=dev)
        d["lr"] = torch.empty(M, R, dtype=torch.bfloat16, device=dev)
        if plain:       # R = 0, no smoothing
            d["smooth"] = d["proj_down"] = d["proj_up"] = d["lr"] = None
            d["proj_up_folded"] = None
        d["y"] = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        sets.append(d)
    return sets


def set_bytes(d):
    import torch
    return sum(v.numel() * v.element_size() for v in d.values() if isinstance(v, torch.Tensor))


def gemm_kernel_name(M):
    """The GEMM kernel svdq_w4a4_linear runs for M tokens."""
    if M <= SMALL_M:
        return "w4a4_linear_small_kernel"
    return "w4a4_linear_pair_kernel" if M >= PAIR_M else "w4a4_linear_kernel"


def gemm_roofline(M, bytes_kg, flops_kg, kg_avg_ms, hbm_gbs, fp4_tflops, peak_src, traffic):
    """Roofline object of the GEMM launch: bound by HBM when its algorithmic
    bytes take longer than its flops at the measured peaks (the few-token
    GEMM streaming the weights), else by the FP4 tensor pipe."""
    kg_s = kg_avg_ms * 1e-3
    if bytes_kg / (hbm_gbs * 1e9) > flops_kg / (fp4_tflops * 1e12):
        achieved = bytes_kg / kg_s / 1e9
        out = {"bound": "hbm", "kernel": gemm_kernel_name(M), "achieved": round(achieved, 1),
               "peak": round(hbm_gbs, 1), "unit": "GB/s", "frac": round(achieved / hbm_gbs, 4),
               "traffic": traffic, "peak_source": f"{peak_src} copy bandwidth",
               "algorithmic_bytes_per_launch": bytes_kg}
    else:
        achieved = flops_kg / kg_s / 1e12
        out = {"bound": "tensor", "kernel": gemm_kernel_name(M), "achieved": round(achieved, 1),
               "peak": round(fp4_tflops, 1), "unit": "TFLOP/s",
               "frac": round(achieved / fp4_tflops, 4), "traffic": traffic,
               "peak_source": f"{peak_src} bf16 burst x {FP4_OVER_BF16:g} (nominal "
                              "FP4:BF16 dense ratio)",
               "algorithmic_flops_per_launch": flops_kg}
    out.update({"avg_launch_ms": round(kg_avg_ms, 5),
                "timing": "CUDA events on its stream around a run of the kernel alone, launched "
                          "back to back over the timed steps' inputs; average per launch"})
    return out


def run_kq(svdq, d, stream):
    svdq.quantize_act(d["x"], d["smooth"], d["proj_down"], qact=d["qact"], ascales_tiled=d["asc"],
                      lowrank=d["lr"], stream=stream)


def run_kg(svdq, d, stream):
    svdq.w4a4_linear(d["qact"], d["asc"], d["lr"], d["qweight"], d["wscales_tiled"],
                     d["wcscales"], d["wtscale"], d["proj_up"], d["bias"], y=d["y"],
                     stream=stream, proj_up_folded=d["proj_up_folded"])


def run_step(svdq, d, stream):
    run_kq(svdq, d, stream)
    run_kg(svdq, d, stream)


def bench_ours(args, world, rank, local):
    import torch
    from nvfp4_w4a4_quantized_smooth_b200 import build as b
    if rank == 0:
        b.build()
    barrier(world)
    from nvfp4_w4a4_quantized_smooth_b200 import svdq, synth

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    M, K, N = synth.WORKLOADS[args.workload]
    plain = is_plain(args.workload)
    r = 0 if plain else R
    seed = rank_seed(args.workload, rank)
    one = flops_per_step(M, K, N, r)

    # rotating sets: enough that a set is evicted from L2 before it returns
    probe = make_sets(M, K, N, 1, seed, dev, plain)
    per_set = set_bytes(probe[0])
    nsets = max(3, -(-3 * L2_BYTES // per_set))
    sets = probe + make_sets(M, K, N, nsets - 1, seed + 1, dev, plain)
    repack_us = 1e6 * statistics.median(d["repack_s"] for d in sets)
    repack_gpu_us = 1e3 * statistics.median(d["repack_gpu_ms"] for d in sets)
    fold_gpu_us = 1e3 * statistics.median(d["fold_gpu_ms"] for d in sets)
    folded = all(d["proj_up_folded"] is not None for d in sets)

    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            run_step(svdq, sets[i % nsets], stream)
        svdq.check_device_error(stream)

        K_steps = args.steps
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        clocks = ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ else
                              int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local]))
        clocks.start()
        time.sleep(0.2)
        barrier(world)
        torch.cuda.synchronize(dev)
        start.record(stream)
        for i in range(K_steps):
            run_step(svdq, sets[i % nsets], stream)
        end.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        # Per-kernel durations: each kernel alone, launched back to back over
        # the same K steps' inputs (rotating sets), between two events; the
        # average is its launch duration in a stream of its own launches.
        # (Events between the kernels of every step would add the launch
        # gap after each event to the kernel's time.)
        kq_e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        kg_e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        kq_e[0].record(stream)
        for i in range(K_steps):
            run_kq(svdq, sets[i % nsets], stream)
        kq_e[1].record(stream)
        kg_e[0].record(stream)
        for i in range(K_steps):
            run_kg(svdq, sets[i % nsets], stream)
        kg_e[1].record(stream)
        torch.cuda.synchronize(dev)
        # The same steps from a CUDA graph (one step per rotating set,
        # captured once, replayed): what the kernels take without the
        # per-call host cost, which dominates at few tokens.  Reported
        # beside the stream number.
        graph = None
        if not args.no_graph:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for j in range(nsets):
                    run_step(svdq, sets[j], stream)
            for _ in range(2):
                g.replay()
            torch.cuda.synchronize(dev)
            reps = max(1, -(-K_steps // nsets))
            gs = torch.cuda.Event(enable_timing=True)
            ge = torch.cuda.Event(enable_timing=True)
            barrier(world)
            gs.record(stream)
            for _ in range(reps):
                g.replay()
            ge.record(stream)
            torch.cuda.synchronize(dev)
            barrier(world)
            gms = max_over_ranks(gs.elapsed_time(ge), world)
            graph = {"value": round(job_value(one, reps * nsets, world, gms), 2), "unit": UNIT,
                     "ms_per_step": round(gms / (reps * nsets), 5), "steps": reps * nsets,
                     "what": f"one step per rotating set captured once in a CUDA graph, "
                             f"replayed {reps} times"}
            del g
        clocks.stop()
        svdq.check_device_error(stream)

    elapsed_ms = max_over_ranks(start.elapsed_time(end), world)
    kq_avg = kq_e[0].elapsed_time(kq_e[1]) / K_steps
    kg_avg = kg_e[0].elapsed_time(kg_e[1]) / K_steps

    value = job_value(one, K_steps, world, elapsed_ms)
    peaks, peak_src = load_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    hbm = peaks["hbm_gbs"]

    # roofline of the whole step and of each kernel
    sm_bytes = 0 if plain else 2 * K
    bytes_kq = 2 * M * K + sm_bytes + 2 * K * r + M * K // 2 + M * K // 16 + 2 * M * r
    bytes_kg = (M * K // 2 + M * K // 16 + N * K // 2 + N * K // 16 + 4 * N + 2 + 2 * M * r
                + 2 * N * r + 2 * M * N)
    flops_kg = 2 * M * N * K + 2 * M * r * N
    t_roof_step = max(one / (fp4_peak * 1e12), (bytes_kq + bytes_kg) / (hbm * 1e9))
    step_s = elapsed_ms * 1e-3 / K_steps
    kg_tflops = flops_kg / (kg_avg * 1e-3) / 1e12
    kg_gbs = bytes_kg / (kg_avg * 1e-3) / 1e9
    kq_gbs = bytes_kq / (kq_avg * 1e-3) / 1e9
    kg_name = gemm_kernel_name(M)
    traffic = load_traffic(kg_name) if kg_name in KERNEL_SOURCES else None
    roofline = gemm_roofline(M, bytes_kg, flops_kg, kg_avg, hbm, fp4_peak, peak_src, traffic)

    # end to end through the public API with host buffers
    e2e = None if args.no_e2e else bench_e2e(args, svdq, sets[0], dev, M, K, N, world, r)

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": K_steps, "warmup": max(args.warmup, 3),
        "ms_per_step": round(elapsed_ms / K_steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e4m3 block16, fp32 accumulate) + bf16 low-rank",
        "data": "synthetic (seeded; random weights of the layer's shapes)",
        "config": {"workload": args.workload, "M": M, "K": K, "N": N, "R": r,
                   "smooth": not plain,
                   "parallelism": f"dp{world} (independent token batches per GPU)",
                   "l2": f"inputs larger than L2: {nsets} rotating sets x "
                         f"{per_set / 2**20:.0f} MiB",
                   "repack_us": round(repack_us, 1),
                   "repack_gpu_us": round(repack_gpu_us, 1),
                   "lowrank_form": ("folded: proj_up / (wtscale * wcscales) prepared once per "
                                    "weight by svdq_fold_proj_up, the low-rank product "
                                    "accumulated with the block-scaled one" if folded else
                                    "separate accumulator" if not plain else "none (R = 0)"),
                   "fold_gpu_us": round(fold_gpu_us, 1),
                   "repack_timing": ("repack_us: host wall time of svdq_repack_weights, which "
                                     "synchronizes to read back the bad-scale count; "
                                     "repack_gpu_us: CUDA events around the call on its "
                                     "stream (counter reset, repack kernel, readback)"),
                   "roofline_frac_of_step": round(t_roof_step / step_s, 4),
                   "cuda_graph": graph},
        "roofline": roofline,
        "kernels": {
            "quantize_act_kernel": {"avg_ms": round(kq_avg, 5), "bytes": bytes_kq,
                                    "GB/s": round(kq_gbs, 1), "peak_GB/s": hbm,
                                    "frac": round(kq_gbs / hbm, 4), "bound": "hbm"},
            kg_name: {"avg_ms": round(kg_avg, 5), "flops": flops_kg,
                      "TFLOP/s": round(kg_tflops, 1), "bytes": bytes_kg,
                      "GB/s": round(kg_gbs, 1)},
        },
        "e2e": e2e,
        "gpu_launches": 2 * K_steps,
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.workload, sample_rows=256 if not plain else 512)
    if rank == 0:
        print(json.dumps(out), flush=True)


def bench_e2e(args, svdq, d, dev, M, K, N, world, r=R):
    """Same metric through the public API with the input in pinned host
    memory and the output read back to pinned host memory every step.

    Steps are pipelined the way a server would run them: the host->device
    copy of step i+1 and the device->host copy of step i-1 run on their own
    streams while step i computes (PCIe is full duplex), with two device
    buffers for x and y so that no copy touches a buffer in use."""
    import torch
    s_h2d = torch.cuda.Stream(device=dev)
    s_cmp = torch.cuda.Stream(device=dev)
    s_d2h = torch.cuda.Stream(device=dev)
    x_host = d["x"].cpu().pin_memory()
    y_host = torch.empty(M, N, dtype=torch.bfloat16).pin_memory()
    x_dev = [torch.empty_like(d["x"]) for _ in range(2)]
    y_dev = [d["y"], torch.empty_like(d["y"])]
    ev = lambda: torch.cuda.Event()
    h2d_done = [ev(), ev()]
    cmp_done = [ev(), ev()]
    d2h_done = [ev(), ev()]
    for e in h2d_done + cmp_done + d2h_done:
        e.record(s_h2d)   # recorded once so that the first waits pass
    steps = max(args.e2e_steps, 1)

    def one_step(i):
        b = i % 2
        s_h2d.wait_event(cmp_done[b])          # x_dev[b] no longer read
        with torch.cuda.stream(s_h2d):
            x_dev[b].copy_(x_host, non_blocking=True)
        h2d_done[b].record(s_h2d)
        s_cmp.wait_event(h2d_done[b])
        s_cmp.wait_event(d2h_done[b])          # y_dev[b] already read back
        with torch.cuda.stream(s_cmp):
            svdq.quantize_act(x_dev[b], d["smooth"], d["proj_down"], qact=d["qact"],
                              ascales_tiled=d["asc"], lowrank=d["lr"], stream=s_cmp)
            svdq.w4a4_linear(d["qact"], d["asc"], d["lr"], d["qweight"], d["wscales_tiled"],
                             d["wcscales"], d["wtscale"], d["proj_up"], d["bias"], y=y_dev[b],
                             stream=s_cmp, proj_up_folded=d["proj_up_folded"])
        cmp_done[b].record(s_cmp)
        s_d2h.wait_event(cmp_done[b])
        with torch.cuda.stream(s_d2h):
            y_host.copy_(y_dev[b], non_blocking=True)
        d2h_done[b].record(s_d2h)

    for i in range(3):
        one_step(i)
    torch.cuda.synchronize(dev)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier(world)
    start.record(s_h2d)
    s_cmp.wait_event(start)
    s_d2h.wait_event(start)
    for i in range(steps):
        one_step(i)
    s_d2h.wait_event(cmp_done[(steps - 1) % 2])
    end.record(s_d2h)
    torch.cuda.synchronize(dev)
    barrier(world)
    svdq.check_device_error(s_cmp)
    ms = max_over_ranks(start.elapsed_time(end), world)
    val = job_value(flops_per_step(M, K, N, r), steps, world, ms)
    return {"value": round(val, 2), "unit": UNIT,
            "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
            "d2h_bytes_per_step": y_host.numel() * y_host.element_size(),
            "steps": steps, "ms_per_step": round(ms / steps, 4),
            "pipelining": "copies of neighbouring steps overlap compute (3 streams, "
                          "2 device buffers)"}


# -------------------------------------------------- the 30-block stack ---

def stack_flops(M=None):
    from nvfp4_w4a4_quantized_smooth_b200 import synth
    M = synth.TOKENS if M is None else M
    return synth.DIT_BLOCKS * sum(flops_per_step(M, K, N) for _, K, N in synth.DIT_BLOCK_LINEARS)


def bench_stack(args, world, rank, local):
    """One step = all 150 linears of the 30-block stack (qkv, out, w1, w3,
    w2 per block; quantize + GEMM each) back to back in one stream.  Block
    inputs are resident; w2's input silu(y_w1) * y_w3 is formed inside the
    step by the fused activation kernel from that block's w1 / w3 outputs;
    weights (3.2 GB) stream from HBM, so no L2 flush is needed."""
    import torch
    from nvfp4_w4a4_quantized_smooth_b200 import build as b
    if rank == 0:
        b.build()
    barrier(world)
    from nvfp4_w4a4_quantized_smooth_b200 import svdq, synth
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    M = synth.DIT_STACKS[args.workload]
    host = synth.make_stack(M=M, x_seed_offset=7919 * rank)
    stream = torch.cuda.Stream(device=dev)
    order = [name for name, _, _ in synth.DIT_BLOCK_LINEARS]
    with torch.cuda.stream(stream):
        blocks = []
        for layers in host:
            w = {n: svdq.PreparedWeights(L.qweight.to(dev), L.wscales.to(dev),
                                         L.wcscales.to(dev), L.wtscale.to(dev),
                                         L.smooth.to(dev), L.proj_down.to(dev),
                                         L.proj_up.to(dev), L.bias.to(dev), stream=stream)
                 for n, L in layers.items()}
            blocks.append({"w": w, "x": layers["qkv"].x.to(dev)})
        del host
        # work buffers, one per K (activation side) and per linear (outputs)
        act = {}
        for K in {k for _, k, _ in synth.DIT_BLOCK_LINEARS}:
            act[K] = (torch.empty(M, K // 2, dtype=torch.uint8, device=dev),
                      torch.empty(svdq.ascales_tiled_bytes(M, K), dtype=torch.uint8, device=dev),
                      torch.empty(M, R, dtype=torch.bfloat16, device=dev))
        ybuf = {n: torch.empty(M, N, dtype=torch.bfloat16, device=dev)
                for n, _, N in synth.DIT_BLOCK_LINEARS}

        def linear(x, w, y):
            qa, asc, lr = act[w.K]
            svdq.quantize_act(x, w.smooth, w.proj_down, qact=qa, ascales_tiled=asc, lowrank=lr,
                              stream=stream)
            svdq.w4a4_linear(qa, asc, lr, w.qweight, w.wscales_tiled, w.wcscales, w.wtscale,
                             w.proj_up, w.bias, y=y, stream=stream,
                             proj_up_folded=w.proj_up_folded)

        hbuf = torch.empty_like(ybuf["w1"]) if args.unfused_w2 else None

        def w2_linear(w, y):
            # w2's input silu(y_w1) * y_w3 is formed on chip by the
            # activation kernel (never written to HBM), or, for comparison,
            # in HBM by svdq_silu_mul and then quantized
            qa, asc, lr = act[w.K]
            if hbuf is not None:
                svdq.silu_mul(ybuf["w1"], ybuf["w3"], out=hbuf, stream=stream)
                svdq.quantize_act(hbuf, w.smooth, w.proj_down, qact=qa, ascales_tiled=asc,
                                  lowrank=lr, stream=stream)
            else:
                svdq.silu_mul_quantize_act(ybuf["w1"], ybuf["w3"], w.smooth, w.proj_down,
                                           qact=qa, ascales_tiled=asc, lowrank=lr, stream=stream)
            svdq.w4a4_linear(qa, asc, lr, w.qweight, w.wscales_tiled, w.wcscales, w.wtscale,
                             w.proj_up, w.bias, y=y, stream=stream,
                             proj_up_folded=w.proj_up_folded)

        def step(evs=None):
            j = 0
            for blk in blocks:
                for n in order:
                    if evs is not None:
                        evs[j].record(stream)
                    if n == "w2":
                        w2_linear(blk["w"][n], ybuf[n])
                    else:
                        linear(blk["x"], blk["w"][n], ybuf[n])
                    j += 1
            if evs is not None:
                evs[j].record(stream)

        for _ in range(max(args.warmup, 3)):
            step()
        svdq.check_device_error(stream)
        steps = args.steps
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        clocks = ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ else
                              int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local]))
        clocks.start()
        time.sleep(0.2)
        barrier(world)
        torch.cuda.synchronize(dev)
        start.record(stream)
        for _ in range(steps):
            step()
        end.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        # per-linear durations, one more pass with an event between linears
        n_lin = len(blocks) * len(order)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_lin + 1)]
        step(evs)
        torch.cuda.synchronize(dev)
        svdq.check_device_error(stream)
        # The same step captured once as a CUDA graph and replayed: the 300
        # launches cost one graph launch (reported beside the stream number).
        graph = None
        if not args.no_graph:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                step()
            for _ in range(2):
                g.replay()
            torch.cuda.synchronize(dev)
            gs = torch.cuda.Event(enable_timing=True)
            ge = torch.cuda.Event(enable_timing=True)
            barrier(world)
            gs.record(stream)
            for _ in range(steps):
                g.replay()
            ge.record(stream)
            torch.cuda.synchronize(dev)
            barrier(world)
            svdq.check_device_error(stream)
            gms = max_over_ranks(gs.elapsed_time(ge), world)
            graph = {"value": round(job_value(stack_flops(M), steps, world, gms), 2),
                     "unit": UNIT, "ms_per_step": round(gms / steps, 4),
                     "what": "the step captured once in a CUDA graph, replayed `steps` times"}
            del g
        clocks.stop()

    elapsed_ms = max_over_ranks(start.elapsed_time(end), world)
    flops = stack_flops(M)
    value = job_value(flops, steps, world, elapsed_ms)
    per_name = {n: 0.0 for n in order}
    for j in range(n_lin):
        per_name[order[j % len(order)]] += evs[j].elapsed_time(evs[j + 1])
    peaks, peak_src = load_peaks()
    fp4_peak = peaks["bf16_tflops_sustained"] * FP4_OVER_BF16
    per_linear = {}
    for n, K, N in synth.DIT_BLOCK_LINEARS:
        ms = per_name[n] / len(blocks)
        per_linear[n] = {"K": K, "N": N, "avg_ms": round(ms, 5),
                         "TFLOP/s": round(flops_per_step(M, K, N) / (ms * 1e-3) / 1e12, 1)}
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": steps, "warmup": max(args.warmup, 3),
        "ms_per_step": round(elapsed_ms / steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e4m3 block16, fp32 accumulate) + bf16 low-rank",
        "data": "synthetic (seeded; random weights of the stack's shapes)",
        "config": {"workload": args.workload, "M": M, "blocks": len(blocks),
                   "linears_per_step": n_lin, "R": R, "cuda_graph": graph,
                   "w2_input": "svdq_silu_mul then svdq_quantize_act" if args.unfused_w2
                               else "formed on chip (svdq_silu_mul_quantize_act)",
                   "parallelism": f"dp{world} (independent token batches per GPU)",
                   "l2": "weights of 150 linears (3.2 GB) stream from HBM every step",
                   "per_linear": per_linear},
        "roofline": {"bound": "tensor", "kernel": "whole step (150 x quantize + GEMM)",
                     "achieved": round(value / world, 1), "peak": round(fp4_peak, 1),
                     "unit": "TFLOP/s", "frac": round(value / world / fp4_peak, 4),
                     "traffic": None,
                     "peak_source": f"{peak_src} bf16 sustained x {FP4_OVER_BF16:g} (nominal "
                                    "FP4:BF16 dense ratio; a step of ~16 ms is a sustained load)"},
        "e2e": None,
        "gpu_launches": (2 * n_lin + (len(blocks) if args.unfused_w2 else 0)) * steps,
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_stack(sample_rows=16)
    if rank == 0:
        print(json.dumps(out), flush=True)


def _stack_oracle_args(rows):
    """Oracle arguments for `rows` tokens through each linear of block 0 (the
    w2 input is a seeded plain N(0, 1) stand-in for silu(y_w1) * y_w3)."""
    import torch
    from nvfp4_w4a4_quantized_smooth_b200 import synth
    b = synth.bits
    layers = synth.make_stack(blocks=1, M=rows)[0]
    h = synth.make_x(rows, synth.FFN, torch.Generator().manual_seed(4005), outliers=0)
    args = []
    for n, L in layers.items():
        x = h if n == "w2" else L.x
        args.append((b(x), b(L.smooth), b(L.proj_down), b(L.qweight), b(L.wscales),
                     b(L.wcscales), b(L.wtscale), b(L.proj_up), b(L.bias)))
    return args, sum(flops_per_step(rows, K, N) for _, K, N in synth.DIT_BLOCK_LINEARS)


def cpu_baseline_stack(sample_rows=16, min_seconds=10.0):
    """The oracle on a bounded sample of the stack: `sample_rows` tokens
    through each of the five linear shapes of block 0, repeated until
    `min_seconds` of CPU work."""
    from oracle import svdq_ref as ref
    args, fl = _stack_oracle_args(sample_rows)
    reps = 0
    t0 = time.perf_counter()
    while True:
        for a in args:
            ref.svdq_linear_from_x(*a)
        reps += 1
        if time.perf_counter() - t0 >= min_seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": round(fl * reps / dt / 1e12, 6), "unit": UNIT, "cores": _blas_threads(),
            "kind": "oracle",
            "sample": f"{sample_rows} tokens through the 5 linears of one block, {reps} passes, "
                      f"{dt:.1f} s"}


# ------------------------------------------------------- the oracle ------

def cpu_baseline(workload, sample_rows=256, min_seconds=10.0):
    """The fp64 CPU oracle, as it stands, on a bounded sample of the workload:
    `sample_rows` tokens of the same layer (all K, all N), repeated until
    `min_seconds` of CPU work.  Returns the metric in TFLOP/s."""
    from nvfp4_w4a4_quantized_smooth_b200 import synth
    from oracle import svdq_ref as ref
    M, K, N = synth.WORKLOADS[workload]
    rows = min(sample_rows, M)
    plain = is_plain(workload)
    fn, args = _oracle_call(synth.make_layer(rows, K, N, seed=synth.workload_seed(workload)),
                            plain)
    reps = 0
    t0 = time.perf_counter()
    while True:
        fn(*args)
        reps += 1
        if time.perf_counter() - t0 >= min_seconds:
            break
    dt = time.perf_counter() - t0
    value = flops_per_step(rows, K, N, 0 if plain else R) * reps / dt / 1e12
    return {"value": round(value, 6), "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{rows} of {M} tokens of {workload} (all K, all N), {reps} passes, "
                      f"{dt:.1f} s"}


def _oracle_call(L, plain):
    """(oracle function, its arguments) for one layer's operands: the full
    layer, or the plain NVFP4 layer (no low-rank branch, no smoothing)."""
    from nvfp4_w4a4_quantized_smooth_b200 import synth
    from oracle import svdq_ref as ref
    b = synth.bits
    if plain:
        return ref.plain_linear_from_x, (b(L.x), b(L.qweight), b(L.wscales), b(L.wcscales),
                                         b(L.wtscale), b(L.bias))
    return ref.svdq_linear_from_x, (b(L.x), b(L.smooth), b(L.proj_down), b(L.qweight),
                                    b(L.wscales), b(L.wcscales), b(L.wtscale), b(L.proj_up),
                                    b(L.bias))


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def bench_reference(args, world, rank):
    """The oracle (CPU, fp64) as the reference arm, rank 0 only."""
    if rank != 0:
        return
    from nvfp4_w4a4_quantized_smooth_b200 import synth
    from oracle import svdq_ref as ref
    if args.workload in synth.DIT_STACKS:
        bench_reference_stack(args, world)
        return
    M, K, N = synth.WORKLOADS[args.workload]
    rows = min(32, M)
    plain = is_plain(args.workload)
    fn, a = _oracle_call(synth.make_layer(rows, K, N, seed=synth.workload_seed(args.workload)),
                         plain)
    for _ in range(min(args.warmup, 1)):
        fn(*a)
    steps = max(1, min(args.steps, 20))
    t0 = time.perf_counter()
    for _ in range(steps):
        fn(*a)
    dt = time.perf_counter() - t0
    value = flops_per_step(rows, K, N, 0 if plain else R) * steps / dt / 1e12
    sample = f"each step: {rows} of {M} tokens of {args.workload} (all K, all N)"
    out = {
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
        "steps": steps, "warmup": min(args.warmup, 1), "ms_per_step": round(1e3 * dt / steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "impl": "reference",
        "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": args.workload, "M": M, "K": K, "N": N, "R": 0 if plain else R},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": _blas_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def bench_reference_stack(args, world):
    """Reference arm on the stack: each step pushes 16 tokens through the
    five linears of block 0 with the oracle."""
    from oracle import svdq_ref as ref
    from nvfp4_w4a4_quantized_smooth_b200 import synth
    oargs, fl = _stack_oracle_args(16)
    for a in oargs:
        ref.svdq_linear_from_x(*a)
    steps = max(1, min(args.steps, 10))
    t0 = time.perf_counter()
    for _ in range(steps):
        for a in oargs:
            ref.svdq_linear_from_x(*a)
    dt = time.perf_counter() - t0
    value = fl * steps / dt / 1e12
    out = {
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
        "steps": steps, "warmup": 1, "ms_per_step": round(1e3 * dt / steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "impl": "reference",
        "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": args.workload, "M": synth.DIT_STACKS[args.workload], "blocks": synth.DIT_BLOCKS,
                   "R": R},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": _blas_threads(),
                         "kind": "oracle",
                         "sample": "each step: 16 tokens through the 5 linears of one block"},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main(argv=None):
    args = parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        bench_reference(args, world, rank)
        return
    world, rank, local = dist_setup()
    try:
        from nvfp4_w4a4_quantized_smooth_b200 import synth
        if args.workload in synth.DIT_STACKS:
            bench_stack(args, world, rank, local)
        else:
            bench_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
