"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Bit-exact: packed E2M1 codes, e4m3 activation scales, the repacked weight
scales (round trip).  Within the stated tolerance: y and L.  All inputs are
seeded synthetic operands of the shapes the layer runs at.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import nvfp4 as nv
from oracle import svdq_ref as ref
from nvfp4_w4a4_quantized_smooth_b200 import synth

import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from nvfp4_w4a4_quantized_smooth_b200 import build
    build.build()
    torch.cuda.init()
    yield


# ------------------------------------------------------------- repack ---

@pytest.mark.parametrize("N,K", [(512, 512), (96, 64), (100, 128), (3840, 3840), (11520, 3840),
                                 (3840, 10240)])
def test_repack_round_trip(N, K):
    s = H.svdq()
    g = torch.Generator().manual_seed(N + K)
    ws = torch.randint(0, 0x7F, (K // 16, N), generator=g, dtype=torch.uint8)
    t = s.repack_weights(ws.cuda())
    assert t.numel() == s.wscales_tiled_bytes(N, K)
    back = s.unpack_scales(t, N, K, kind="weight").cpu()
    assert torch.equal(back, ws.t().contiguous())
    # padding rows (beyond N) of the tiled buffer are zero scales
    rows_pad = (N + 255) // 256 * 256
    if rows_pad > N:
        full = s.unpack_scales(t, rows_pad, K, kind="weight").cpu()
        assert torch.all(full[N:] == 0)


@pytest.mark.parametrize("bad", [0x80, 0xB8, 0x7F, 0xFF])
def test_repack_rejects_sign_and_nan_scales(bad):
    s = H.svdq()
    ws = torch.full((8, 64), 0x38, dtype=torch.uint8)
    ws[3, 17] = bad
    with pytest.raises(s.SvdqError) as e:
        s.repack_weights(ws.cuda())
    assert e.value.status == s.SVDQ_ERR_INVALID_ARG


# ----------------------------------------------------------- quantize ---

@pytest.mark.parametrize("M,K", [(1, 64), (17, 128), (128, 512), (129, 512), (300, 192),
                                 (64, 3840), (513, 1024), (16, 10240), (100, 640), (1000, 448),
                                 (2000, 256), (4352, 256)])
def test_quantize_act_bit_exact_and_lowrank(M, K):
    s = H.svdq()
    L = synth.make_layer(M, K, 32, seed=M * 7 + K)
    qact, asc, lr = s.quantize_act(L.x.cuda(), L.smooth.cuda(), L.proj_down.cuda())
    s.check_device_error()
    q_ref, a_ref = H.oracle_quant(L.x, L.smooth)
    H.assert_quant_exact(qact.cpu(), s.unpack_scales(asc, M, K).cpu(), q_ref, a_ref,
                         f"M={M} K={K}")
    L_ref = ref.lowrank_down(H.bits(L.x), H.bits(L.proj_down))
    H.assert_lowrank_close(lr.cpu(), L_ref, f"M={M} K={K}")


def test_quantize_plans_fit_one_wave():
    # 64- or 128-row tiles; a K split forms a cluster of 2, 4 or 8 CTAs with
    # at least 256 k each, or of 16 with at least 128 k each; the grid runs
    # in one wave when it can.
    s = H.svdq()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for M in (1, 16, 64, 100, 256, 1024, 4352, 17408, 40000):
        for K in (64, 512, 3840, 10240):
            bm, split = s.quantize_plan(M, K)
            tiles = -(-M // bm)
            assert bm in (64, 128), (M, K, bm)
            assert split in (1, 2, 4, 8, 16), (M, K, split)
            assert split == 1 or bm == 64, (M, K, bm, split)   # a split takes 64-row tiles
            assert split == 1 or (256 if split <= 8 else 128) * split <= K, (M, K, split)
            if tiles * split > sms:
                assert split == 1 and bm == 128, (M, K, bm, split)
            if M <= 64:
                assert bm == 64, (M, K, bm)       # the tile that pads M least


@pytest.mark.parametrize("M,K", [(300, 3840), (4352, 3840), (16, 10240)])
def test_quantize_results_repeat_bit_for_bit(M, K):
    # The split-K partial sums are added in a fixed order on chip, so two
    # calls give identical bits.
    s = H.svdq()
    L = synth.make_layer(M, K, 256, seed=31)
    d = H.to_dev(L)
    out1 = s.quantize_act(d["x"], d["smooth"], d["proj_down"])
    out2 = s.quantize_act(d["x"], d["smooth"], d["proj_down"])
    s.check_device_error()
    for a, b in zip(out1, out2):
        assert torch.equal(a, b)
    L_ref = ref.lowrank_down(H.bits(L.x), H.bits(L.proj_down))
    H.assert_lowrank_close(out1[2].cpu(), L_ref, f"M={M} K={K}")


def _golden_rows():
    """x rows built from the hand-worked groups of tests/golden/ (smooth = 1)."""
    import test_oracle_pins as P
    rows, scales, codes = [], [], []
    for name in ("nvfp4_block_a.txt", "nvfp4_block_b.txt"):
        g = P.read_golden(name)
        rows.append([float(v) for v in g["v"]])
        scales.append(int(g["scale"][0], 16))
        codes.append([int(c, 16) for c in g["codes"]])
    g = P.read_golden("nvfp4_block_c.txt")
    for c in ("c1", "c2", "c3", "c4", "c5", "c6"):
        rows.append([float(v) for v in g[c + "_v"]])
        scales.append(int(g[c + "_scale"][0], 16))
        codes.append([int(v, 16) for v in g[c + "_codes"]])
    return rows, scales, codes


def test_quantize_golden_groups_bit_exact():
    # Each golden group is placed in every one of the 4 group slots of a
    # 64-wide row (the other slots hold a plain group), so every position of
    # the shared-memory swizzle and of the scale tile is exercised.
    s = H.svdq()
    rows, scales, codes = _golden_rows()
    filler = [1.0] * 16
    X, want_sc, want_codes = [], [], []
    for gv, gs, gc in zip(rows, scales, codes):
        for slot in range(4):
            line = [filler] * 4
            line[slot] = gv
            X.append(sum(line, []))
            want_sc.append((slot, gs))
            want_codes.append((slot, gc))
    M = len(X)
    K = 64
    x = torch.tensor(X, dtype=torch.float64).to(torch.bfloat16)
    assert torch.equal(x.to(torch.float64), torch.tensor(X, dtype=torch.float64))
    smooth = torch.ones(K, dtype=torch.bfloat16)
    pd = torch.zeros(K, 128, dtype=torch.bfloat16)
    qact, asc, lr = s.quantize_act(x.cuda(), smooth.cuda(), pd.cuda())
    s.check_device_error()
    asc_l = s.unpack_scales(asc, M, K).cpu().numpy()
    cod = nv.unpack_nibbles(qact.cpu().numpy())
    for m in range(M):
        slot, gs = want_sc[m]
        assert asc_l[m, slot] == gs, (m, hex(asc_l[m, slot]), hex(gs))
        assert list(cod[m, 16 * slot:16 * slot + 16]) == want_codes[m][1], m
    # and the oracle agrees everywhere (filler groups included)
    q_ref, a_ref = H.oracle_quant(x, smooth)
    H.assert_quant_exact(qact.cpu(), torch.from_numpy(asc_l), q_ref, a_ref, "golden rows")
    assert torch.all(lr.cpu() == 0)


def test_quantize_ties_signed_zeros_and_saturation():
    # Elements planted on every E2M1 midpoint for many scales, signed zeros,
    # tiny negatives, scale saturation and subnormal scales.
    rng = np.random.default_rng(11)
    rows = []
    for scale_code in list(range(0x01, 0x7E, 3)):
        d = float(nv.decode_e4m3(scale_code))
        mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
        v = [6 * d] + [m * d for m in mids] + [-m * d for m in mids] + [-0.0]
        rows.append(v)
    rows.append([3e4, -2e4] + [0.0] * 14)
    rows.append([-1e-3, 2e-3, -0.0, 0.0] * 4)
    x = torch.tensor(rows, dtype=torch.float64).to(torch.bfloat16)
    M = x.shape[0]
    x = torch.cat([x, x.flip(1), x * 0.5, -x], dim=1)   # K = 64
    smooth = torch.ones(64, dtype=torch.bfloat16)
    s = H.svdq()
    qact, asc, _ = s.quantize_act(x.cuda(), smooth.cuda(), torch.zeros(64, 128, dtype=torch.bfloat16).cuda())
    s.check_device_error()
    q_ref, a_ref = H.oracle_quant(x, smooth)
    H.assert_quant_exact(qact.cpu(), s.unpack_scales(asc, M, 64).cpu(), q_ref, a_ref, "ties")


def test_quantize_respects_row_stride():
    s = H.svdq()
    L = synth.make_layer(40, 256, 32, seed=5)
    big = torch.zeros(40, 320, dtype=torch.bfloat16)
    big[:, :256] = L.x
    xd = big.cuda()[:, :256]
    qact, asc, lr = s.quantize_act(xd, L.smooth.cuda(), L.proj_down.cuda())
    s.check_device_error()
    q_ref, a_ref = H.oracle_quant(L.x, L.smooth)
    H.assert_quant_exact(qact.cpu(), s.unpack_scales(asc, 40, 256).cpu(), q_ref, a_ref, "stride")


# ------------------------------------------------------------- linear ---

@pytest.mark.parametrize("M,K,N", [(128, 512, 512), (1, 256, 256), (17, 256, 96), (200, 768, 288),
                                   (129, 512, 544), (256, 1024, 768)])
def test_linear_parity(M, K, N):
    L = synth.make_layer(M, K, N, seed=M + 3 * K + 7 * N)
    r = H.gpu_layer(L)
    y_ref, q_ref, a_ref, _ = H.oracle_y(L)
    H.assert_quant_exact(r["qact"], r["ascales"], q_ref, a_ref, "quant")
    H.assert_y_close(r["y"], y_ref, f"M={M} K={K} N={N}")
    H.assert_y_close(r["y_fold"], y_ref, f"folded M={M} K={K} N={N}")
    if M <= 128:   # only the CTA-pair GEMM takes the folded factor
        assert torch.equal(r["y_fold"].view(torch.int16), r["y"].view(torch.int16))


@pytest.mark.parametrize("M,K,N,with_smooth", [(300, 512, 384, False), (128, 1024, 512, True),
                                               (16, 3840, 3840, False), (1000, 768, 1280, True)])
def test_plain_nvfp4_layer(M, K, N, with_smooth):
    # R = 0: no low-rank branch; without smooth, x is quantized as it is.
    L = synth.make_layer(M, K, N, seed=3 * M + K + 7 * N + with_smooth)
    r = H.gpu_plain_layer(L, with_smooth)
    y_ref, q_ref, a_ref = H.oracle_plain_y(L, with_smooth)
    H.assert_quant_exact(r["qact"], r["ascales"], q_ref, a_ref, "plain quant")
    H.assert_y_close(r["y"], y_ref, f"plain M={M} K={K} N={N}")


def test_plain_nvfp4_layer_full_size_qkv():
    name = "qkv_m4352_k3840_n11520"
    M, K, N = synth.WORKLOADS[name]
    L = synth.make_layer(M, K, N, seed=synth.workload_seed(name))
    r = H.gpu_plain_layer(L, False)
    y_ref, q_ref, a_ref = H.oracle_plain_y(L, False)
    H.assert_quant_exact(r["qact"], r["ascales"], q_ref, a_ref, "plain qkv quant")
    H.assert_y_close(r["y"], y_ref, "plain qkv")


def test_linear_without_bias():
    L = synth.make_layer(64, 512, 256, seed=21, with_bias=False)
    r = H.gpu_layer(L)
    y_ref, *_ = H.oracle_y(L)
    H.assert_y_close(r["y"], y_ref, "no bias")


def test_integer_grid_invariant_bit_exact():
    # Unit scales, no low-rank term, x groups on the E2M1 grid with amax 6:
    # y must equal the bf16 rounding of the exact integer-grid product.
    rng = np.random.default_rng(12)
    M, K, N = 160, 512, 256
    cx = rng.integers(0, 16, (M, K), dtype=np.uint8)
    cx[:, ::16] = 7
    x = torch.from_numpy(nv.decode_e2m1(cx)).to(torch.bfloat16)
    L = synth.make_layer(M, K, N, seed=13)
    L.x = x
    L.smooth = torch.ones(K, dtype=torch.bfloat16)
    L.wscales = torch.full((K // 16, N), 0x38, dtype=torch.uint8)
    L.wcscales = torch.ones(N, dtype=torch.bfloat16)
    L.wtscale = torch.ones(1, dtype=torch.bfloat16)
    L.proj_down = torch.zeros(K, 128, dtype=torch.bfloat16)
    L.proj_up = torch.zeros(N, 128, dtype=torch.bfloat16)
    L.bias = torch.zeros(N, dtype=torch.bfloat16)
    r = H.gpu_layer(L)
    y_ref, *_ = H.oracle_y(L)
    want = nv.f64_to_bf16_bits_rne(y_ref)
    for key in ("y", "y_fold"):
        got = H.bits(r[key])
        assert np.array_equal(got, want), f"{key}: {(got != want).sum()} outputs differ"


def test_unit_scales_random_codes_exact():
    # Same as above but with random per-block weight scales and wcscales that
    # are powers of two: every product and partial sum stays exact in fp32.
    rng = np.random.default_rng(14)
    M, K, N = 128, 256, 256
    cx = rng.integers(0, 16, (M, K), dtype=np.uint8)
    cx[:, ::16] = 7
    x = torch.from_numpy(nv.decode_e2m1(cx)).to(torch.bfloat16)
    L = synth.make_layer(M, K, N, seed=15)
    L.x = x
    L.smooth = torch.ones(K, dtype=torch.bfloat16)
    L.wscales = torch.from_numpy(rng.choice([0x30, 0x38, 0x40, 0x48], (K // 16, N)).astype(np.uint8))
    L.wcscales = torch.from_numpy(rng.choice([0.5, 1.0, 2.0], N)).to(torch.bfloat16)
    L.wtscale = torch.ones(1, dtype=torch.bfloat16)
    L.proj_down = torch.zeros(K, 128, dtype=torch.bfloat16)
    L.proj_up = torch.zeros(N, 128, dtype=torch.bfloat16)
    L.bias = torch.zeros(N, dtype=torch.bfloat16)
    r = H.gpu_layer(L)
    y_ref, *_ = H.oracle_y(L)
    want = nv.f64_to_bf16_bits_rne(y_ref)
    for key in ("y", "y_fold"):
        got = H.bits(r[key])
        assert np.array_equal(got, want), f"{key}: {(got != want).sum()} outputs differ"


def test_zero_weights_give_lowrank_branch_only():
    L = synth.make_layer(192, 512, 512, seed=16)
    L.qweight = torch.zeros_like(L.qweight)
    r = H.gpu_layer(L)
    lr = (oracle.bf16_bits_to_f64(H.bits(L.x)) @ oracle.bf16_bits_to_f64(H.bits(L.proj_down))
          @ oracle.bf16_bits_to_f64(H.bits(L.proj_up)).T
          + oracle.bf16_bits_to_f64(H.bits(L.bias)))
    H.assert_y_close(r["y"], lr, "low-rank only")
    H.assert_y_close(r["y_fold"], lr, "low-rank only, folded")


def test_output_row_stride():
    s = H.svdq()
    L = synth.make_layer(100, 256, 256, seed=17)
    d = H.to_dev(L)
    wt = s.repack_weights(d["wscales"])
    qact, asc, lr = s.quantize_act(d["x"], d["smooth"], d["proj_down"])
    ybig = torch.full((100, 320), 7.0, dtype=torch.bfloat16, device="cuda")
    s.w4a4_linear(qact, asc, lr, d["qweight"], wt, d["wcscales"], d["wtscale"], d["proj_up"],
                  d["bias"], y=ybig[:, :256])
    s.check_device_error()
    y_ref, *_ = H.oracle_y(L)
    H.assert_y_close(ybig[:, :256].cpu(), y_ref, "ldy")
    assert torch.all(ybig[:, 256:].cpu() == 7.0)


# ------------------------------------------------- full-size workloads ---

def _full_size_check(name):
    """Every code, scale, L value and output of the workload against the
    oracle (the fp64 product of the decoded operands)."""
    M, K, N = synth.WORKLOADS[name]
    L = synth.make_layer(M, K, N, seed=synth.workload_seed(name))
    r = H.gpu_layer(L)
    y_ref, q_ref, a_ref, L_ref = H.oracle_y(L)
    H.assert_quant_exact(r["qact"], r["ascales"], q_ref, a_ref, name)
    H.assert_y_close(r["y"], y_ref, name)
    H.assert_y_close(r["y_fold"], y_ref, f"{name} folded")
    H.assert_lowrank_close(r["lowrank"], L_ref, name)
    return L, r


def test_full_size_layer_m128():
    _full_size_check("layer_m128_k512_n512")


def test_full_size_qkv():
    _full_size_check("qkv_m4352_k3840_n11520")


@pytest.mark.parametrize("M", synth.OUT_PROJ_SWEEP_M)
def test_full_size_out_proj_sweep(M):
    _full_size_check(f"out_m{M}_k3840_n3840")


def test_full_size_ffn_chain():
    # w1, w3 on the block input, h = silu(y1) * y3 from the GPU's own bf16
    # outputs (bit for bit the oracle's silu_mul of those outputs), then w2
    # on h; the oracle for w2 takes that h as its input.
    s = H.svdq()
    L1, r1 = _full_size_check("ffn_w1_m4352_k3840_n10240")
    L3 = synth.make_layer(*synth.WORKLOADS["ffn_w3_m4352_k3840_n10240"],
                          seed=synth.workload_seed("ffn_w3_m4352_k3840_n10240"))
    L3.x = L1.x
    r3 = H.gpu_layer(L3)
    y3_ref, *_ = H.oracle_y(L3)
    H.assert_y_close(r3["y"], y3_ref, "w3")
    h = s.silu_mul(r1["y"].cuda(), r3["y"].cuda())
    s.check_device_error()
    hd = h.cpu()
    h_ref = oracle.silu_mul(H.bits(r1["y"]), H.bits(r3["y"]))
    assert np.array_equal(H.bits(hd), h_ref), "silu(y1) * y3 differs from the oracle"
    L2 = synth.make_layer(*synth.WORKLOADS["ffn_w2_m4352_k10240_n3840"],
                          seed=synth.workload_seed("ffn_w2_m4352_k10240_n3840"))
    r2 = H.gpu_layer(L2, x_override=h)
    y_ref, q_ref, a_ref, L_ref = H.oracle_y(L2, x=hd)
    H.assert_quant_exact(r2["qact"], r2["ascales"], q_ref, a_ref, "w2 quant")
    H.assert_y_close(r2["y"], y_ref, "w2")
    H.assert_lowrank_close(r2["lowrank"], L_ref, "w2 L")


@pytest.mark.parametrize("M,K,R", [(300, 512, 128), (64, 1024, 0), (1000, 2048, 128),
                                   (4352, 10240, 128)])
def test_fused_silu_mul_quantize(M, K, R):
    # quantize_act of x = silu(a) * b, with x formed on chip: codes and
    # scales equal, bit for bit, to oracle.quantize_act(oracle.silu_mul(a,
    # b)) on every row, and to the unfused path (svdq_silu_mul, then
    # svdq_quantize_act); L within tolerance of the oracle's on that x.
    s = H.svdq()
    g = torch.Generator().manual_seed(M + K + R)
    a = (torch.randn(M, K, generator=g) * 2).to(torch.bfloat16)
    b = torch.randn(M, K, generator=g).to(torch.bfloat16)
    sm = (torch.rand(K, generator=g) * 1.5 + 0.5).to(torch.bfloat16)
    pd = (torch.randn(K, 128, generator=g) * 0.02).to(torch.bfloat16) if R else None
    ad, bd, smd = a.cuda(), b.cuda(), sm.cuda()
    pdd = pd.cuda() if R else None
    q1, a1, l1 = s.silu_mul_quantize_act(ad, bd, smd, pdd)
    h = s.silu_mul(ad, bd)
    q2, a2, l2 = s.quantize_act(h, smd, pdd)
    s.check_device_error()
    h_ref = oracle.silu_mul(H.bits(a), H.bits(b))
    assert np.array_equal(H.bits(h.cpu()), h_ref), "silu(a) * b differs from the oracle"
    q_ref, a_ref = ref.quantize_act(h_ref, H.bits(sm))
    asc1 = s.unpack_scales(a1, M, K).cpu()
    H.assert_quant_exact(q1.cpu(), asc1, q_ref, a_ref, "fused silu quant vs oracle")
    assert torch.equal(q1, q2)
    assert torch.equal(asc1, s.unpack_scales(a2, M, K).cpu())
    if R:
        L_ref = ref.lowrank_down(h_ref, H.bits(pd))
        H.assert_lowrank_close(l1.cpu(), L_ref, "fused silu L")
    else:
        assert l1 is None


def test_full_size_ffn_chain_fused():
    # w1, w3, then w2 with its input formed on chip from their outputs;
    # the oracle forms that input with its own silu_mul.
    s = H.svdq()
    names = ("ffn_w1_m4352_k3840_n10240", "ffn_w3_m4352_k3840_n10240", "ffn_w2_m4352_k10240_n3840")
    L1, L3, L2 = (synth.make_layer(*synth.WORKLOADS[n], seed=synth.workload_seed(n)) for n in names)
    L3.x = L1.x
    r1, r3 = H.gpu_layer(L1), H.gpu_layer(L3)
    y1, y3 = r1["y"].cuda(), r3["y"].cuda()
    d = H.to_dev(L2)
    wt = s.repack_weights(d["wscales"])
    qa, asc, lr = s.silu_mul_quantize_act(y1, y3, d["smooth"], d["proj_down"])
    y = s.w4a4_linear(qa, asc, lr, d["qweight"], wt, d["wcscales"], d["wtscale"], d["proj_up"],
                      d["bias"])
    s.check_device_error()
    h_ref = oracle.silu_mul(H.bits(r1["y"]), H.bits(r3["y"]))
    h = torch.from_numpy(h_ref.view(np.int16)).view(torch.bfloat16)
    y_ref, q_ref, a_ref, L_ref = H.oracle_y(L2, x=h)
    H.assert_quant_exact(qa.cpu(), s.unpack_scales(asc, L2.M, L2.K).cpu(), q_ref, a_ref,
                         "fused w2 quant")
    H.assert_y_close(y.cpu(), y_ref, "fused w2")
    H.assert_lowrank_close(lr.cpu(), L_ref, "fused w2 L")


# ------------------------------------------------ seeded shape sweep ---

def _sweep_shapes(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        M = int(rng.integers(1, 700))
        K = 256 * int(rng.integers(1, 9))
        N = 32 * int(rng.integers(1, 33))
        out.append((M, K, N))
    return out


@pytest.mark.parametrize("M,K,N", _sweep_shapes(12, 2026))
def test_shape_sweep_all_paths(M, K, N):
    # Seeded shapes (ragged M, N and several K) through every path: the
    # layer, the layer without the low-rank branch (with and without
    # smooth), and w2's activation formed on chip; each against the oracle,
    # and each repeated bit for bit.
    s = H.svdq()
    L = synth.make_layer(M, K, N, seed=M * 7 + K + N)
    r = H.gpu_layer(L)
    y_ref, q_ref, a_ref, L_ref = H.oracle_y(L)
    H.assert_quant_exact(r["qact"], r["ascales"], q_ref, a_ref, f"layer {M}x{K}x{N}")
    H.assert_y_close(r["y"], y_ref, f"layer {M}x{K}x{N}")
    H.assert_y_close(r["y_fold"], y_ref, f"folded layer {M}x{K}x{N}")
    H.assert_lowrank_close(r["lowrank"], L_ref, f"layer {M}x{K}x{N}")
    again = H.gpu_layer(L)
    assert torch.equal(again["y"].view(torch.int16), r["y"].view(torch.int16))
    assert torch.equal(again["y_fold"].view(torch.int16), r["y_fold"].view(torch.int16))
    for with_smooth in (False, True):
        p = H.gpu_plain_layer(L, with_smooth)
        yp, qp, ap = H.oracle_plain_y(L, with_smooth)
        H.assert_quant_exact(p["qact"], p["ascales"], qp, ap, f"plain {M}x{K}x{N}")
        H.assert_y_close(p["y"], yp, f"plain {M}x{K}x{N}")
    g = torch.Generator().manual_seed(M + N)
    a = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    b = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    d = H.to_dev(L)
    q1, a1, l1 = s.silu_mul_quantize_act(a, b, d["smooth"], d["proj_down"])
    h = s.silu_mul(a, b)
    q2, a2, l2 = s.quantize_act(h, d["smooth"], d["proj_down"])
    s.check_device_error()
    assert torch.equal(q1, q2)
    assert torch.equal(s.unpack_scales(a1, M, K).cpu(), s.unpack_scales(a2, M, K).cpu())
    Lh = ref.lowrank_down(H.bits(h.cpu()), H.bits(L.proj_down))
    H.assert_lowrank_close(l1.cpu(), Lh, f"fused L {M}x{K}")


# ------------------------------------------------ few tokens (M <= 64) ---

@pytest.mark.parametrize("M,K,N", [(1, 256, 128), (7, 10240, 3840), (33, 1024, 416), (64, 512, 384),
                                   (64, 768, 11520), (64, 2048, 20480)])
def test_small_m_transposed_gemm(M, K, N):
    # M <= 64 runs the transposed GEMM (weights as the 128-row operand):
    # one token, ragged M and N, a long K, more 128-column tiles than SMs
    # (the persistent loop) -- with and without the low-rank branch,
    # against the oracle, and repeated bit for bit.
    L = synth.make_layer(M, K, N, seed=M * 3 + K + N)
    r = H.gpu_layer(L)
    y_ref, q_ref, a_ref, L_ref = H.oracle_y(L)
    H.assert_quant_exact(r["qact"], r["ascales"], q_ref, a_ref, f"{M}x{K}x{N}")
    H.assert_y_close(r["y"], y_ref, f"{M}x{K}x{N}")
    again = H.gpu_layer(L)
    assert torch.equal(again["y"].view(torch.int16), r["y"].view(torch.int16))
    p = H.gpu_plain_layer(L, True)
    yp, _, _ = H.oracle_plain_y(L, True)
    H.assert_y_close(p["y"], yp, f"plain {M}x{K}x{N}")


# --------------------------------- every bf16 amax through the quantizer ---

_E2M1_MIDPOINTS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def _amax_sweep_groups(random_smooth: bool, seed: int):
    """One 16-element group per positive finite bf16 value A: A itself (the
    group's amax, at a rotating position and with alternating sign) and
    the seven E2M1 midpoints of the group's scale d = e4m3(A / 6), both
    signs, so that every element quotient is a tie.  With random smooth the
    stored x is bf16(target / smooth), so v = x * smooth is a 16-bit product
    next to the target instead of on it (targets up to 2^126, so that x
    stays finite)."""
    amax_bits = np.arange(1, 0x7F80, dtype=np.uint16)
    A = nv.bf16_bits_to_f64(amax_bits)
    if random_smooth:
        # x = A / smooth must stay finite in bf16 and x * smooth in fp32
        A = A[A <= 2.0 ** 126]
    d = nv.decode_e4m3(nv.encode_e4m3_rne_satfinite(A / 6.0))
    n = len(A)
    G = np.zeros((n, 16))
    mids = np.array(_E2M1_MIDPOINTS)
    body = np.concatenate([mids[None, :] * d[:, None], -mids[None, :] * d[:, None],
                           np.zeros((n, 1))], axis=1)                   # 15 values
    body = np.minimum(np.abs(body), A[:, None]) * np.sign(body)         # keep A the amax
    pos = np.arange(n) % 16
    sign = np.where(np.arange(n) % 2 == 0, 1.0, -1.0)
    for i in range(n):
        row = list(body[i])
        row.insert(pos[i], sign[i] * A[i])
        G[i] = row
    K = 64
    rows = (n + 3) // 4
    X = np.zeros((rows * 4, 16))
    X[:n] = G
    X = X.reshape(rows, K)
    rng = np.random.default_rng(seed)
    if random_smooth:
        sm = torch.from_numpy(rng.uniform(0.5, 2.0, K)).to(torch.bfloat16)
        x = (torch.from_numpy(X) / sm.double()[None, :]).to(torch.bfloat16)
    else:
        sm = torch.ones(K, dtype=torch.bfloat16)
        x = torch.from_numpy(X).to(torch.bfloat16)
        assert torch.equal(x.double(), torch.from_numpy(X)), "planted values must be bf16"
    return x, sm


@pytest.mark.parametrize("random_smooth", [False, True])
def test_quantizer_every_bf16_amax_with_planted_ties(random_smooth):
    # The activation kernel's divisions (reciprocal + one residual step)
    # against the oracle's exact rounding, for every positive finite bf16
    # value as a group amax, on the chip that runs them.
    s = H.svdq()
    x, sm = _amax_sweep_groups(random_smooth, seed=41)
    M, K = x.shape
    for R in (128, 0):
        pd = torch.zeros(K, 128, dtype=torch.bfloat16).cuda() if R else None
        qact, asc, _ = s.quantize_act(x.cuda(), sm.cuda(), pd)
        s.check_device_error()
        q_ref, a_ref = H.oracle_quant(x, sm)
        H.assert_quant_exact(qact.cpu(), s.unpack_scales(asc, M, K).cpu(), q_ref, a_ref,
                             f"amax sweep, random smooth {random_smooth}, R={R}")


# ---------------------------- ragged K ranges and cluster-sum boundaries ---

@pytest.mark.parametrize("M,K", [(16, 64 * 37), (64, 64 * 45), (100, 64 * 41), (200, 64 * 23),
                                 (33, 64 * 161)])
def test_quantize_ragged_k_split(M, K):
    # K/64 not a multiple of the plan's split: the K ranges of a tile
    # differ by 64 k and the last stage of some ranges holds one chunk.
    s = H.svdq()
    bm, split = s.quantize_plan(M, K)
    assert split > 1 and (K // 64) % split != 0, (M, K, bm, split)
    L = synth.make_layer(M, K, 32, seed=M + K)
    qact, asc, lr = s.quantize_act(L.x.cuda(), L.smooth.cuda(), L.proj_down.cuda())
    s.check_device_error()
    q_ref, a_ref = H.oracle_quant(L.x, L.smooth)
    H.assert_quant_exact(qact.cpu(), s.unpack_scales(asc, M, K).cpu(), q_ref, a_ref,
                         f"ragged split M={M} K={K}")
    H.assert_lowrank_close(lr.cpu(), ref.lowrank_down(H.bits(L.x), H.bits(L.proj_down)),
                           f"ragged split L M={M} K={K}")


@pytest.mark.parametrize("M,K,N", [(16, 256 * 5, 1024), (64, 256 * 7, 896), (1, 256 * 11, 1280),
                                   (40, 256 * 13, 2048), (64, 256 * 37, 512)])
def test_few_token_gemm_ragged_k_split(M, K, N):
    # num_k = K/256 not a multiple of the few-token GEMM's cluster split:
    # ranks hold different numbers of K steps, and the rank-order sum of
    # the partials covers uneven ranges.
    s = H.svdq()
    kernel, split, grid = s.linear_plan(M, N, K)
    assert kernel == s.GEMM_FEW_TOKENS and split > 1 and (K // 256) % split != 0, \
        (M, N, K, kernel, split)
    L = synth.make_layer(M, K, N, seed=M * 5 + K + N)
    r = H.gpu_layer(L)
    y_ref, q_ref, a_ref, _ = H.oracle_y(L)
    H.assert_quant_exact(r["qact"], r["ascales"], q_ref, a_ref, f"{M}x{K}x{N}")
    H.assert_y_close(r["y"], y_ref, f"ragged few-token {M}x{K}x{N} split {split}")
    p = H.gpu_plain_layer(L, True)
    yp, _, _ = H.oracle_plain_y(L, True)
    H.assert_y_close(p["y"], yp, f"plain ragged few-token {M}x{K}x{N}")


def test_linear_plans_follow_their_rules():
    # The launch shapes the host picks (not a restatement of them): the
    # kernel by M (few tokens, single-SM tiles, CTA pairs), the few-token K
    # split within 1..8, at most one K step short per rank, the clusters of
    # a split in one wave.
    s = H.svdq()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for M in (1, 16, 63, 64, 65, 256, 4352):
        for N in (32, 416, 3840, 11520, 20480):
            for K in (256, 768, 1280, 3840, 10240):
                kernel, split, grid = s.linear_plan(M, N, K)
                if M <= 64:
                    assert kernel == s.GEMM_FEW_TOKENS
                    n_tiles = -(-N // 128)
                    assert split in (1, 2, 4, 8) and split <= K // 256
                    if split > 1:
                        assert grid == n_tiles * split <= sms
                    else:
                        assert grid == min(n_tiles, sms)
                elif M <= 128:
                    tiles = -(-M // 128) * -(-N // 256)
                    assert kernel == s.GEMM_TOKEN_MAJOR and split == 1
                    assert grid == min(tiles, sms)
                else:
                    # CTA pairs: an even grid, one pair per 256 x 256 tile
                    # up to the pairs the device co-schedules
                    tiles = -(-M // 256) * -(-N // 256)
                    assert kernel == s.GEMM_PAIRS and split == 1
                    assert grid % 2 == 0 and grid // 2 <= min(tiles, sms // 2)
                    assert grid // 2 == tiles or grid >= sms - 2


# ------------------------------------------------ concurrent repacks ---

def test_concurrent_repacks_report_their_own_bad_scales():
    # Two host threads repack at once on their own streams; one input has a
    # sign-bit scale byte.  The bad-scale counter is shared per device, so
    # the calls are serialized inside the library: the bad input must
    # always give SVDQ_ERR_INVALID_ARG and the good one SVDQ_OK.
    import threading
    s = H.svdq()
    good = torch.full((240, 3840), 0x38, dtype=torch.uint8).cuda()
    bad = good.clone()
    bad[117, 2000] = 0x80
    results = {"good": [], "bad": []}

    def worker(name, ws):
        st = torch.cuda.Stream()
        for _ in range(40):
            try:
                s.repack_weights(ws, stream=st)
                results[name].append(s.SVDQ_OK)
            except s.SvdqError as e:
                results[name].append(e.status)

    ts = [threading.Thread(target=worker, args=("good", good)),
          threading.Thread(target=worker, args=("bad", bad))]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert results["good"] == [s.SVDQ_OK] * 40
    assert results["bad"] == [s.SVDQ_ERR_INVALID_ARG] * 40
