"""Pins for the CPU oracle: checks against things other than the oracle.

* closed forms of the E2M1 / e4m3 bit layouts and library codecs
  (ml_dtypes, torch) for decode and in-range encode;
* hand-worked groups under tests/golden/ (each file cites its passages);
* an exact rational brute force of the whole layer on tiny shapes, written
  independently of the oracle (fractions.Fraction, candidate scan);
* special cases that reduce to a plain matmul, and the integer-grid
  invariant of the block-scaled product.

All of these run without a GPU.
"""

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import nvfp4 as nv
from oracle import svdq_ref as ref
from nvfp4_w4a4_quantized_smooth_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            out[key.strip()] = val.split()
    return out


def bf16_bits_of(values):
    """float values exactly representable in bf16 -> raw uint16 bits."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64)
    b = t.to(torch.bfloat16)
    assert torch.equal(b.to(torch.float64), t), "value not representable in bf16"
    return b.view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------- E2M1 ---

def test_e2m1_table_matches_golden_and_bit_layout():
    g = read_golden("e2m1_codes.txt")
    want = np.array([float(v) for v in g["values"]])
    got = nv.decode_e2m1(np.arange(16, dtype=np.uint8))
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), np.signbit(want))
    # closed form from the 1-2-1 bit fields, bias 1
    for c in range(16):
        s, e, m = c >> 3, (c >> 1) & 3, c & 1
        mag = m * 0.5 if e == 0 else (1 + m / 2) * 2.0 ** (e - 1)
        assert got[c] == (-mag if s else mag)


def test_e2m1_decode_matches_ml_dtypes():
    ml = pytest.importorskip("ml_dtypes")
    codes = np.arange(16, dtype=np.uint8)
    lib = codes.view(ml.float4_e2m1fn) if hasattr(codes, "view") else None
    # ml_dtypes stores float4 one per byte in the low nibble
    lib = np.array(codes, dtype=np.uint8).view(ml.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(nv.decode_e2m1(codes), lib)


def test_e2m1_encode_all_midpoints_and_saturation():
    mags = nv.E2M1_MAGNITUDES
    for i in range(7):
        lo, hi = mags[i], mags[i + 1]
        mid = (lo + hi) / 2
        want = i if i % 2 == 0 else i + 1           # tie -> even code
        assert nv.encode_e2m1_rne_sat(mid) == want
        assert nv.encode_e2m1_rne_sat(-mid) == want | 8
        assert nv.encode_e2m1_rne_sat(np.nextafter(mid, 0)) == i
        assert nv.encode_e2m1_rne_sat(np.nextafter(mid, 10)) == i + 1
    for big in (6.0, 6.5, 7.0, 1e9):
        assert nv.encode_e2m1_rne_sat(big) == 7
        assert nv.encode_e2m1_rne_sat(-big) == 0xF
    assert nv.encode_e2m1_rne_sat(-0.0) == 8
    assert nv.encode_e2m1_rne_sat(-0.1) == 8
    # every code round-trips
    for c in range(16):
        assert nv.encode_e2m1_rne_sat(nv.decode_e2m1(c)) == c


def test_e2m1_encode_matches_ml_dtypes_on_random_values():
    ml = pytest.importorskip("ml_dtypes")
    rng = np.random.default_rng(1)
    v = rng.uniform(-6, 6, 20000)
    lib = v.astype(ml.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(nv.encode_e2m1_rne_sat(v), lib)


# ---------------------------------------------------------------- e4m3 ---

def test_e4m3_decode_all_codes_matches_libraries():
    ml = pytest.importorskip("ml_dtypes")
    codes = np.arange(256, dtype=np.uint8)
    got = nv.decode_e4m3(codes)
    lib = codes.view(ml.float8_e4m3fn).astype(np.float64)
    tlib = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(got), nan)
    assert set(np.nonzero(nan)[0]) == {0x7F, 0xFF}
    assert np.array_equal(got[~nan], lib[~nan])
    assert np.array_equal(got[~nan], tlib[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6


def test_e4m3_encode_roundtrip_midpoints_and_saturation():
    vals = nv.decode_e4m3(np.arange(0x7F, dtype=np.uint8))
    for c in range(0x7F):
        assert nv.encode_e4m3_rne_satfinite(vals[c]) == c
        assert nv.encode_e4m3_rne_satfinite(-vals[c]) == c | 0x80
    for c in range(0x7E):
        mid = (vals[c] + vals[c + 1]) / 2
        want = c if c % 2 == 0 else c + 1
        assert nv.encode_e4m3_rne_satfinite(mid) == want
        assert nv.encode_e4m3_rne_satfinite(np.nextafter(mid, 0)) == c
        assert nv.encode_e4m3_rne_satfinite(np.nextafter(mid, 1e9)) == c + 1
    for big in (448.0, 449.0, 464.0, 480.0, 1e6):
        assert nv.encode_e4m3_rne_satfinite(big) == 0x7E
    assert nv.encode_e4m3_rne_satfinite(2.0 ** -10) == 0      # tie -> even 0
    assert nv.encode_e4m3_rne_satfinite(2.0 ** -10 * 1.0001) == 1
    assert nv.encode_e4m3_rne_satfinite(1e-9) == 0


def test_e4m3_encode_matches_libraries_in_range():
    ml = pytest.importorskip("ml_dtypes")
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.uniform(-448, 448, 20000),
                        np.exp(rng.uniform(-14, 6, 20000)) * rng.choice([-1, 1], 20000)])
    v = v[np.abs(v) <= 448]
    lib = v.astype(ml.float8_e4m3fn).view(np.uint8)
    tlib = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = nv.encode_e4m3_rne_satfinite(v)
    assert np.array_equal(got, lib)
    assert np.array_equal(got, tlib)


# --------------------------------------------------------------- bf16 ---

def test_bf16_codec_matches_torch():
    rng = np.random.default_rng(3)
    v = rng.standard_normal(50000) * np.exp(rng.uniform(-20, 20, 50000))
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(nv.f64_to_bf16_bits_rne(v), want)
    assert np.array_equal(nv.bf16_bits_to_f64(want),
                          torch.from_numpy(want.view(np.int16)).view(torch.bfloat16)
                          .to(torch.float64).numpy())
    # halfway cases straight from float64 (no float32 double rounding)
    one_ulp = 2.0 ** -7
    assert nv.f64_to_bf16_bits_rne(1 + one_ulp / 2) == 0x3F80        # tie -> even
    assert nv.f64_to_bf16_bits_rne(1 + 3 * one_ulp / 2) == 0x3F82    # tie -> even
    assert nv.f64_to_bf16_bits_rne(1 + one_ulp / 2 + 2.0 ** -40) == 0x3F81


# ------------------------------------------------------- nibble packing ---

def test_pack_nibbles_literal_and_roundtrip():
    assert nv.pack_nibbles(np.array([1, 2], dtype=np.uint8))[0] == 0x21
    rng = np.random.default_rng(4)
    codes = rng.integers(0, 16, (7, 64), dtype=np.uint8)
    packed = nv.pack_nibbles(codes)
    assert packed.shape == (7, 32)
    assert np.array_equal(nv.unpack_nibbles(packed), codes)
    assert np.array_equal(nv.unpack_nibbles(packed.view(np.int8)), codes)
    raw = rng.integers(0, 256, (5, 16), dtype=np.uint8)
    assert np.array_equal(nv.pack_nibbles(nv.unpack_nibbles(raw)), raw)


# ------------------------------------------------- golden NVFP4 groups ---

def _quantize_group(values):
    x = bf16_bits_of(values).reshape(1, 16)
    smooth = bf16_bits_of([1.0] * 16)
    return ref.quantize_act(x, smooth)


@pytest.mark.parametrize("name", ["nvfp4_block_a.txt", "nvfp4_block_b.txt"])
def test_golden_group(name):
    g = read_golden(name)
    qact, sc = _quantize_group(g["v"])
    assert sc[0, 0] == int(g["scale"][0], 16)
    codes = nv.unpack_nibbles(qact)[0]
    assert [int(c) for c in codes] == [int(c, 16) for c in g["codes"]]
    assert [int(b) for b in qact[0]] == [int(b, 16) for b in g["packed"]]


@pytest.mark.parametrize("case", ["c1", "c2", "c3", "c4", "c5", "c6"])
def test_golden_degenerate_groups(case):
    g = read_golden("nvfp4_block_c.txt")
    qact, sc = _quantize_group(g[case + "_v"])
    assert sc[0, 0] == int(g[case + "_scale"][0], 16)
    codes = nv.unpack_nibbles(qact)[0]
    assert [int(c) for c in codes] == [int(c, 16) for c in g[case + "_codes"]]


def test_smooth_multiplies():
    # Doubling smooth on a group must give the same codes and a scale one
    # binade up (the model card writes quant(x * smooth), a product).
    g = read_golden("nvfp4_block_a.txt")
    x = bf16_bits_of([float(v) / 2 for v in g["v"]]).reshape(1, 16)
    q1, s1 = ref.quantize_act(x, bf16_bits_of([2.0] * 16))
    q2, s2 = _quantize_group(g["v"])
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


# ------------------------------------------------ exact brute force -----
# An independent exact model: decode from bit fields with Fractions and
# round by scanning every candidate code.

def _frac_e2m1(c):
    s, e, m = (c >> 3) & 1, (c >> 1) & 3, c & 1
    mag = Fraction(m, 2) if e == 0 else (1 + Fraction(m, 2)) * Fraction(2) ** (e - 1)
    return -mag if s else mag


def _frac_e4m3(c):
    s, e, m = (c >> 7) & 1, (c >> 3) & 15, c & 7
    assert not (e == 15 and m == 7)
    mag = m * Fraction(1, 512) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
    return -mag if s else mag


def _frac_bf16(b):
    b = int(b)
    s, e, m = b >> 15, (b >> 7) & 0xFF, b & 0x7F
    assert e != 0xFF
    mag = m * Fraction(2) ** -133 if e == 0 else (1 + Fraction(m, 128)) * Fraction(2) ** (e - 127)
    return -mag if s else mag


def _nearest_code(value, candidates):
    """Scan (code, exact value) pairs; nearest, ties to the even code."""
    best = None
    for code, val in candidates:
        d = abs(value - val)
        key = (d, code % 2)
        if best is None or key < best[0]:
            best = (key, code)
    return best[1]


_E2M1_POS = [(c, _frac_e2m1(c)) for c in range(8)]
_E4M3_POS = [(c, _frac_e4m3(c)) for c in range(0x7F)]


def _exact_layer(xb, sb, pdb, qw, ws, wcb, wtb, pub, bb):
    M, K = xb.shape
    N = qw.shape[0]
    x = [[_frac_bf16(xb[m, k]) for k in range(K)] for m in range(M)]
    s = [_frac_bf16(sb[k]) for k in range(K)]
    codes = np.zeros((M, K), dtype=np.uint8)
    scales = np.zeros((M, K // 16), dtype=np.uint8)
    for m in range(M):
        for g in range(K // 16):
            v = [x[m][k] * s[k] for k in range(16 * g, 16 * g + 16)]
            a = max(abs(t) for t in v) / 6
            sc = 0x7E if a >= 448 else _nearest_code(a, _E4M3_POS)
            scales[m, g] = sc
            d = _frac_e4m3(sc)
            for i, t in enumerate(v):
                neg = t < 0 or (t == 0 and np.signbit(float(x[m][16 * g + i])))
                mag = 0 if d == 0 else abs(t) / d
                c = 7 if mag >= 6 else _nearest_code(mag, _E2M1_POS)
                codes[m, 16 * g + i] = c | (8 if neg else 0)
    y = [[Fraction(0)] * N for _ in range(M)]
    alpha = _frac_bf16(wtb[0])
    R = pdb.shape[1]
    for m in range(M):
        L = [sum(x[m][k] * _frac_bf16(pdb[k, r]) for k in range(K)) for r in range(R)]
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                w = _frac_e2m1(int(qw[n, k // 2] >> (4 * (k % 2))) & 0xF)
                acc += (_frac_e2m1(int(codes[m, k])) * _frac_e4m3(int(scales[m, k // 16]))
                        * w * _frac_e4m3(int(ws[k // 16, n])))
            lr = sum(L[r] * _frac_bf16(pub[n, r]) for r in range(R))
            y[m][n] = acc * alpha * _frac_bf16(wcb[n]) + lr + _frac_bf16(bb[n])
    return codes, scales, y


@pytest.mark.parametrize("M,N,K,seed", [(1, 1, 16, 0), (2, 3, 32, 1), (3, 2, 32, 2), (3, 3, 16, 3)])
def test_oracle_matches_exact_brute_force(M, N, K, seed):
    L = synth.make_layer(M, K, N, R=4, seed=seed, outliers=1)
    b = synth.bits
    args = (b(L.x), b(L.smooth), b(L.proj_down), b(L.qweight), b(L.wscales),
            b(L.wcscales), b(L.wtscale), b(L.proj_up), b(L.bias))
    codes, scales, y_exact = _exact_layer(*args)
    y, qact, ascales, _ = ref.svdq_linear_from_x(*args)
    assert np.array_equal(nv.unpack_nibbles(qact), codes)
    assert np.array_equal(ascales, scales)
    for m in range(M):
        for n in range(N):
            e = float(y_exact[m][n])
            assert abs(y[m, n] - e) <= 1e-13 * max(1.0, abs(e))


def test_quantizer_matches_brute_force_on_wide_range():
    # Many random groups spanning the e4m3 range (subnormal and saturated
    # scales), including exact ties planted on E2M1 midpoints.
    rng = np.random.default_rng(5)
    rows = []
    for i in range(48):
        e = rng.integers(-14, 14)
        v = rng.standard_normal(16) * 2.0 ** e
        rows.append(v)
    v = torch.tensor(np.array(rows)).to(torch.bfloat16)
    xb = v.view(torch.int16).numpy().view(np.uint16)
    sb = bf16_bits_of([1.0] * 16)
    qact, sc = ref.quantize_act(xb, sb)
    for m in range(xb.shape[0]):
        vals = [_frac_bf16(t) for t in xb[m]]
        a = max(abs(t) for t in vals) / 6
        want = 0x7E if a >= 448 else _nearest_code(a, _E4M3_POS)
        assert sc[m, 0] == want


def test_planted_ties_round_to_even():
    # Groups built so that v / scale lands exactly on every E2M1 midpoint.
    for scale_code in (0x38, 0x39, 0x3B, 0x44, 0x4D, 0x05):
        d = nv.decode_e4m3(scale_code)
        mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
        vals = [6 * d] + [m * d for m in mids] + [-m * d for m in mids] + [0.0]
        xb = bf16_bits_of(vals).reshape(1, 16)
        qact, sc = ref.quantize_act(xb, bf16_bits_of([1.0] * 16))
        assert sc[0, 0] == scale_code
        codes = nv.unpack_nibbles(qact)[0]
        want = [7, 0, 2, 2, 4, 4, 6, 6, 8, 10, 10, 12, 12, 14, 14, 0]
        assert list(codes) == want


def test_fp32_division_path_equals_exact_rounding_for_every_bf16_amax():
    # The CUDA quantizer divides in float32 before rounding to e4m3 / E2M1.
    # That double rounding agrees with exact rational rounding for every
    # positive finite bf16 amax (a product of two bf16 values has at most 16
    # significant bits; every e4m3 midpoint times 6 has few bits, so a
    # correctly rounded float32 quotient never crosses a midpoint).  This
    # checks the e4m3 half of the argument over all bf16 magnitudes below
    # the saturation bound.
    bits = np.arange(1, 0x7F80, dtype=np.uint32)
    a = (bits << 16).view(np.float32).astype(np.float64)
    a = a[a / 6 < 480]
    q32 = (a.astype(np.float32) / np.float32(6)).astype(np.float64)
    assert np.array_equal(nv.encode_e4m3_rne_satfinite(q32),
                          nv.encode_e4m3_rne_satfinite(a / 6))
    # and products of two bf16 values (16 significant bits) on a sample
    rng = np.random.default_rng(6)
    x = torch.from_numpy(rng.standard_normal(200000) * 8).to(torch.bfloat16).to(torch.float64)
    s = torch.from_numpy(rng.uniform(0.5, 2, 200000)).to(torch.bfloat16).to(torch.float64)
    p = (x * s).abs().numpy()
    q32 = (p.astype(np.float32) / np.float32(6)).astype(np.float64)
    assert np.array_equal(nv.encode_e4m3_rne_satfinite(q32),
                          nv.encode_e4m3_rne_satfinite(p / 6))


# ----------------------------------------------- special cases / laws ---

def _dec(bits16):
    return nv.bf16_bits_to_f64(bits16)


def test_zero_weights_reduce_to_lowrank_matmul():
    # qweight = 0 -> y = (x @ proj_down) @ proj_up^T + bias, a plain matmul.
    L = synth.make_layer(16, 64, 24, R=8, seed=7)
    b = synth.bits
    qw = np.zeros_like(b(L.qweight))
    y, *_ = ref.svdq_linear_from_x(b(L.x), b(L.smooth), b(L.proj_down), qw,
                                   b(L.wscales), b(L.wcscales), b(L.wtscale),
                                   b(L.proj_up), b(L.bias))
    want = (_dec(b(L.x)) @ _dec(b(L.proj_down))) @ _dec(b(L.proj_up)).T + _dec(b(L.bias))
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)


def test_single_code_product_closed_form():
    # One nonzero weight code per row and one active x group: y is a single
    # closed-form product alpha * c[n] * e2m1 * sa * e2m1 * sw.
    M, K, N = 2, 32, 2
    x = np.zeros((M, K)); x[0, 3] = 6.0; x[1, 20] = -3.0
    xb = bf16_bits_of(x.ravel()).reshape(M, K)
    sm = bf16_bits_of([1.0] * K)
    qw = np.zeros((N, K // 2), dtype=np.uint8)
    qw[0, 1] = 0x50        # k = 3 (odd -> high nibble) code 5 = 3.0
    qw[1, 10] = 0x0E       # k = 20 (even -> low nibble) code E = -4.0
    ws = np.full((K // 16, N), 0x38, dtype=np.uint8)   # 1.0
    ws[0, 0] = 0x40                                    # 2.0 for (g0, n0)
    wc = bf16_bits_of([0.5, 1.5])
    wt = bf16_bits_of([0.25])
    zeros_pd = bf16_bits_of([0.0] * (K * 4)).reshape(K, 4)
    zeros_pu = bf16_bits_of([0.0] * (N * 4)).reshape(N, 4)
    y, qact, asc, _ = ref.svdq_linear_from_x(xb, sm, zeros_pd, qw, ws, wc, wt, zeros_pu, None)
    # row 0: group 0 amax 6 -> scale 1 -> code 7 (6.0); times w 3.0 * 2.0
    assert y[0, 0] == 6.0 * 1.0 * 3.0 * 2.0 * 0.25 * 0.5
    assert y[0, 1] == 0.0
    # row 1: group 1 amax 3 -> scale 0.5 -> -3/0.5 = -6 (code F); times -4 * 1
    assert asc[1, 1] == 0x30
    assert y[1, 1] == (-6.0 * 0.5) * (-4.0 * 1.0) * 0.25 * 1.5
    assert y[1, 0] == 0.0


def test_integer_grid_invariant():
    # Unit scales, no low-rank branch, every x group on the E2M1 grid with
    # amax exactly 6: the layer is an exact integer-grid matmul of the codes.
    rng = np.random.default_rng(8)
    M, K, N = 5, 64, 7
    codes_x = rng.integers(0, 16, (M, K), dtype=np.uint8)
    codes_x[:, ::16] = 7                                  # amax 6 in every group
    x = nv.decode_e2m1(codes_x)
    xb = bf16_bits_of(x.ravel()).reshape(M, K)
    qw = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    ws = np.full((K // 16, N), 0x38, dtype=np.uint8)
    one = bf16_bits_of([1.0])
    y, qact, asc, _ = ref.svdq_linear_from_x(
        xb, bf16_bits_of([1.0] * K), bf16_bits_of([0.0] * K * 4).reshape(K, 4), qw, ws,
        bf16_bits_of([1.0] * N), one, bf16_bits_of([0.0] * N * 4).reshape(N, 4),
        bf16_bits_of([0.0] * N))
    assert np.all(asc == 0x38)
    assert np.array_equal(nv.unpack_nibbles(qact), codes_x)
    w = nv.decode_e2m1(nv.unpack_nibbles(qw))
    exact = np.array([[sum(Fraction(float(x[m, k])) * Fraction(float(w[n, k]))
                           for k in range(K)) for n in range(N)] for m in range(M)])
    assert np.array_equal(y, exact.astype(np.float64))
    assert np.all(np.mod(y * 4, 1) == 0)        # multiples of 0.25


def test_plain_layer_integer_grid_exact():
    # The layer without the low-rank branch and without smoothing: every x
    # group on the E2M1 grid with amax 6 and unit weight scales give an exact
    # rational matmul of the codes, scaled by wtscale * wcscales, plus bias.
    rng = np.random.default_rng(11)
    M, K, N = 4, 96, 6
    codes_x = rng.integers(0, 16, (M, K), dtype=np.uint8)
    codes_x[:, ::16] = 15                                 # amax 6 (as -6) in every group
    x = nv.decode_e2m1(codes_x)
    xb = bf16_bits_of(x.ravel()).reshape(M, K)
    qw = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    ws = np.full((K // 16, N), 0x38, dtype=np.uint8)      # 1.0
    wc = bf16_bits_of([0.5, 1.0, 2.0, 0.25, 4.0, 1.5])
    wt = bf16_bits_of([0.125])
    bias = bf16_bits_of([1.0, -2.0, 0.5, 0.0, 3.0, -0.25])
    y, qact, asc = ref.plain_linear_from_x(xb, qw, ws, wc, wt, bias)
    assert np.all(asc == 0x38)
    assert np.array_equal(nv.unpack_nibbles(qact), codes_x)
    w = nv.decode_e2m1(nv.unpack_nibbles(qw))
    cs = [0.5, 1.0, 2.0, 0.25, 4.0, 1.5]
    bs = [1.0, -2.0, 0.5, 0.0, 3.0, -0.25]
    exact = np.array([[sum(Fraction(float(x[m, k])) * Fraction(float(w[n, k])) for k in range(K))
                       * Fraction(1, 8) * Fraction(cs[n]) + Fraction(bs[n])
                       for n in range(N)] for m in range(M)])
    assert np.array_equal(y, exact.astype(np.float64))


def test_plain_layer_is_the_layer_with_unit_smooth_and_no_lowrank():
    # No smooth = a factor of 1 (x * 1 is exact); R = 0 = a zero low-rank term.
    L = synth.make_layer(6, 64, 10, R=4, seed=12)
    b = synth.bits
    K, N = 64, 10
    y0, q0, a0 = ref.plain_linear_from_x(b(L.x), b(L.qweight), b(L.wscales), b(L.wcscales),
                                         b(L.wtscale), b(L.bias))
    # the smoothed layer's quantizer on x * 1, and a zero low-rank product
    y1, q1, a1, _ = ref.svdq_linear_from_x(
        b(L.x), bf16_bits_of([1.0] * K), bf16_bits_of([0.0] * K * 4).reshape(K, 4),
        b(L.qweight), b(L.wscales), b(L.wcscales), b(L.wtscale),
        bf16_bits_of([0.0] * N * 4).reshape(N, 4), b(L.bias))
    assert np.array_equal(q0, q1) and np.array_equal(a0, a1)
    assert np.array_equal(y0, y1)
    # with a smooth factor given, the codes are those of x * smooth
    y2, q2, a2 = ref.plain_linear_from_x(b(L.x), b(L.qweight), b(L.wscales), b(L.wcscales),
                                         b(L.wtscale), b(L.bias), smooth_bits=b(L.smooth))
    q3, a3 = ref.quantize_act(b(L.x), b(L.smooth))
    assert np.array_equal(q2, q3) and np.array_equal(a2, a3)


def test_lowrank_uses_raw_x():
    # The low-rank branch is (x @ proj_down), not (x * smooth) @ proj_down.
    L = synth.make_layer(4, 32, 8, R=4, seed=9)
    b = synth.bits
    got = ref.lowrank_down(b(L.x), b(L.proj_down))
    np.testing.assert_array_equal(got, _dec(b(L.x)) @ _dec(b(L.proj_down)))


def test_quantize_shapes_and_dtypes():
    L = synth.make_layer(3, 48, 5, R=4, seed=10)
    qact, asc = ref.quantize_act(synth.bits(L.x), synth.bits(L.smooth))
    assert qact.shape == (3, 24) and qact.dtype == np.uint8
    assert asc.shape == (3, 3) and asc.dtype == np.uint8
    assert np.all((asc & 0x80) == 0)        # amax/6 >= 0 -> sign bit clear


# ------------------------------------------------ bf16 rounding extremes ---

def test_bf16_rounding_of_subnormals_and_overflow_matches_torch():
    # float32 inputs are exact in float64, so the oracle's single rounding
    # must agree with torch's float32 -> bfloat16 conversion (nearest-even
    # on the bit pattern) also for float32 subnormals, the smallest normals
    # and values near the float32 maximum.
    rng = np.random.default_rng(21)
    sub = rng.integers(1, 1 << 23, 20000, dtype=np.uint32)                 # float32 subnormals
    small = rng.integers(1 << 23, 3 << 23, 20000, dtype=np.uint32)         # binades 2^-126, 2^-125
    big = rng.integers(0x7F000000, 0x7F800000, 20000, dtype=np.uint32)     # up to the float32 max
    ties = (rng.integers(0, 1 << 15, 6000, dtype=np.uint32) << 16) | 0x8000  # exact bf16 midpoints
    u = np.concatenate([sub, small, big, ties])
    u = np.concatenate([u, u | np.uint32(0x80000000)])
    v32 = u.view(np.float32)
    v32 = v32[np.isfinite(v32)]
    want = torch.from_numpy(v32.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = nv.f64_to_bf16_bits_rne(v32.astype(np.float64))
    assert np.array_equal(got, want)
    # overflow threshold (2 - 2^-8) 2^127 and signed zeros, by hand
    thr = (2.0 - 2.0 ** -8) * 2.0 ** 127
    assert nv.f64_to_bf16_bits_rne(thr) == 0x7F80
    assert nv.f64_to_bf16_bits_rne(np.nextafter(thr, 0)) == 0x7F7F
    assert nv.f64_to_bf16_bits_rne(-2.0 ** -135) == 0x8000
    assert nv.f64_to_bf16_bits_rne(2.0 ** -134) == 0x0000                    # tie -> even (0)
    assert nv.f64_to_bf16_bits_rne(3 * 2.0 ** -134) == 0x0002                # tie -> even (2)


# --------------------------------------------------------- SiLU * mul ---

def _bf16_table():
    """Every non-negative finite bf16 value, indexed by its bit pattern."""
    u = (np.arange(0, 0x7F80, dtype=np.uint32) << 16).view(np.float32)
    return [float(v) for v in u]


def _silu_mul_bits_mp(a, b, mp, table):
    """bf16 bits of silu(a) * b from 50-digit mpmath arithmetic, rounded by
    searching the table of bf16 values (ties to the even bit pattern; at or
    above the overflow threshold, inf).  Written independently of the
    oracle.  For a > 0 the product is taken as P - c with P = a b exact and
    c = P exp(-a) / (1 + exp(-a)), and the side of the nearest midpoint is
    decided from (|P| - mid) - |c|, so that c is never lost to the working
    precision (mpmath's exponent range is unbounded)."""
    import bisect
    a, b = mp.mpf(a), mp.mpf(b)
    if a == 0 or b == 0:
        neg = (mp.sign(a) < 0) != (mp.sign(b) < 0)
        return None if (a == 0) else (0x8000 if neg else 0)
    if a > 0:
        P = a * b
        c = P * mp.exp(-a) / (1 + mp.exp(-a))
        x = P - c
        above = lambda mid: (abs(P) - mid) - abs(c)           # sign of |x| - mid
    else:
        e = mp.exp(a)
        x = a * e / (1 + e) * b
        above = lambda mid: abs(x) - mid
    sign = 0x8000 if x < 0 else 0
    if above(mp.mpf((2.0 - 2.0 ** -8) * 2.0 ** 127)) >= 0:
        return sign | 0x7F80
    i = max(bisect.bisect_right(table, float(abs(x))) - 1, 0)
    for _ in range(2):                       # float(|x|) may sit one entry low
        if i + 1 < len(table):
            d = above(mp.mpf(table[i]) / 2 + mp.mpf(table[i + 1]) / 2)
            if d > 0 or (d == 0 and i % 2 == 1):
                i += 1
                continue
        break
    return sign | i


def test_silu_mul_every_bf16_input_against_mpmath():
    # silu(a) for every finite bf16 a (b = 1 and b = -0.75), against 50-digit
    # mpmath arithmetic rounded by a table search.
    mp = pytest.importorskip("mpmath").mp
    mp.dps = 50
    table = _bf16_table()
    pos = np.arange(0, 0x7F80, dtype=np.uint16)
    a_bits = np.concatenate([pos, pos | np.uint16(0x8000)])
    a = nv.bf16_bits_to_f64(a_bits)
    for bv in (1.0, -0.75):
        b_bits = np.full(a_bits.shape, bf16_bits_of([bv])[0], dtype=np.uint16)
        got = oracle.silu_mul(a_bits, b_bits)
        want = np.array([_silu_mul_bits_mp(x, bv, mp, table)
                         if x != 0 else (0x8000 if (np.signbit(x) != (bv < 0)) else 0)
                         for x in a], dtype=np.uint16)
        bad = np.flatnonzero(got != want)
        assert bad.size == 0, (bv, [(a[i], hex(got[i]), hex(want[i])) for i in bad[:5]])


def test_silu_mul_random_products_against_mpmath():
    # Products spread over the whole bf16 range: outputs near the smallest
    # normal and in the subnormal range, large negative a where exp(-a) is
    # huge, and large outputs.
    mp = pytest.importorskip("mpmath").mp
    mp.dps = 50
    table = _bf16_table()
    rng = np.random.default_rng(22)
    n = 6000
    a = np.concatenate([rng.standard_normal(n) * 4, rng.uniform(-100, -80, n),
                        rng.uniform(-30, 30, n), np.exp(rng.uniform(-20, 40, n))])
    b = np.concatenate([rng.standard_normal(n), np.exp(rng.uniform(-60, 60, n)) * rng.choice([-1, 1], n),
                        np.exp(rng.uniform(-90, -80, n)) * rng.choice([-1, 1], n),
                        rng.standard_normal(n) * 1e-30])
    a_bits = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    b_bits = torch.from_numpy(b).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    av, bv = nv.bf16_bits_to_f64(a_bits), nv.bf16_bits_to_f64(b_bits)
    keep = np.isfinite(av) & np.isfinite(bv) & (av != 0) & (bv != 0)
    a_bits, b_bits, av, bv = a_bits[keep], b_bits[keep], av[keep], bv[keep]
    got = oracle.silu_mul(a_bits, b_bits)
    want = np.array([_silu_mul_bits_mp(x, y, mp, table) for x, y in zip(av, bv)],
                    dtype=np.uint16)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, [(av[i], bv[i], hex(got[i]), hex(want[i])) for i in bad[:5]]
    # the sample does reach the subnormal outputs and the region a < -87
    assert np.any((got & 0x7F80) == 0) and np.any(av < -87)


def test_silu_mul_closed_forms():
    # silu(0) = 0 with the sign of the product; silu(a) * b for large a is
    # a * b rounded, except where a * b is exactly a bf16 midpoint: silu(a)
    # is then just below a, so the product rounds toward zero; for large
    # negative a the product is a tiny value of the opposite sign to b.
    z = bf16_bits_of([0.0, -0.0, 0.0, -0.0])
    b = bf16_bits_of([1.0, 1.0, -2.0, -2.0])
    assert list(oracle.silu_mul(z, b)) == [0x0000, 0x8000, 0x8000, 0x0000]
    rng = np.random.default_rng(23)
    a = bf16_bits_of([float(v) for v in rng.integers(64, 128, 200)])       # silu(a) = a (1 - 2^-92..)
    bb = torch.from_numpy(rng.standard_normal(200)).to(torch.bfloat16)
    b_bits = bb.view(torch.int16).numpy().view(np.uint16)
    prod = nv.bf16_bits_to_f64(a) * nv.bf16_bits_to_f64(b_bits)          # exact (16 bits)
    pbits = (torch.from_numpy(prod.astype(np.float32)).view(torch.int32).numpy()
             .view(np.uint32))
    is_tie = (pbits & 0xFFFF) == 0x8000
    trunc = (pbits >> 16).astype(np.uint16)                                 # toward zero
    rne = torch.from_numpy(prod.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.silu_mul(a, b_bits)
    assert np.array_equal(got[~is_tie], rne[~is_tie])
    # planted ties: a = 1.5 * 2^k, b = 1 + 2^-7: a * b has 9 significant bits
    a_t = bf16_bits_of([48.0, 96.0, 192.0, 384.0, 1536.0, 3072.0])
    b_t = bf16_bits_of([1.0 + 2.0 ** -7] * 6)
    p = nv.bf16_bits_to_f64(a_t) * (1.0 + 2.0 ** -7)
    pu = p.astype(np.float32).view(np.uint32)
    assert np.all((pu & 0xFFFF) == 0x8000)
    assert np.array_equal(oracle.silu_mul(a_t, b_t), (pu >> 16).astype(np.uint16))
    assert np.array_equal(got[is_tie], trunc[is_tie])
    # large negative a: -a e^a b, tiny and of the opposite sign to b
    an = bf16_bits_of([-40.0, -60.0, -80.0])
    bn = bf16_bits_of([3.0, -3.0, 3.0])
    h = nv.bf16_bits_to_f64(oracle.silu_mul(an, bn))
    want = np.array([-40 * math.exp(-40) * 3, 60 * math.exp(-60) * 3, -80 * math.exp(-80) * 3])
    assert np.all(np.abs(h - want) <= 2.0 ** -8 * np.abs(want))
