"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test would fail for a plausible mistake in the oracle: a /16 instead of
/15, a sign flip of the zero point, rint taken after adding z, a swapped
nibble order, a transposed operand, a dropped bias, a wrong group index.
None of these tests calls the CUDA library.
"""
from fractions import Fraction
import os

import numpy as np
import pytest

import oracle
from gemv_w4a16_groupwise_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16(vals):
    return synth.f64_to_bf16_bits(np.asarray(vals, dtype=np.float64))


def f16_value(bits):
    return float(np.asarray(bits, dtype=np.uint16).view(np.float16))


def bf16_value(bits):
    return synth.bf16_bits_to_f32(np.asarray(bits, dtype=np.uint16)).astype(np.float64)


# ----------------------------------------------------------------------------
# Hand-derived closed-form examples (derivations in the comments).
# Reading of the quantizer (llm-quantization, Objective 1, no formula printed):
#   s = fp16((max-min)/15); z = clamp(rint(-min/s), 0, 15); q = clamp(rint(w/s) + z, 0, 15)
# ----------------------------------------------------------------------------
ROW_A = [-1.0, -0.5, 0.0, 0.5, 1.0, 2.0, 1.5, -0.25]
# min -1, max 2: (2+1)/15 = 0.2 -> fp16 1.599609375*2^-3 = 0.199951171875 (0x3266)
# z = rint(1/0.19995...) = rint(5.0012) = 5 (0x4500)
# w/s = -5.0012, -2.5006, 0, 2.5006, 5.0012, 10.0024, 7.5018, -1.2503
# rint + 5 = 0, 2, 5, 8, 10, 15, 13, 4
ROW_A_Q = [0, 2, 5, 8, 10, 15, 13, 4]
ROW_B = [-1.75, 2.0, 0.125, 0.375, -0.125, -0.375, 0.625, 1.125]
# min -1.75, max 2: 3.75/15 = 0.25 exactly (0x3400); z = 7 (0x4700)
# w/s = -7, 8, 0.5, 1.5, -0.5, -1.5, 2.5, 4.5 -> ties go to even: 0, 2, -0, -2, 2, 4
ROW_B_Q = [0, 15, 7, 9, 7, 5, 9, 11]


def test_golden_groupwise_example():
    q, s, z = oracle.quantize(bf16([ROW_A, ROW_B]), "groupwise", 8)
    assert q.tolist() == [ROW_A_Q, ROW_B_Q]
    assert s.ravel().tolist() == [0x3266, 0x3400]
    assert z.ravel().tolist() == [0x4500, 0x4700]
    p = oracle.pack(q)
    # nibble i of the word holds code i: A -> 4,D,F,A,8,5,2,0 ; B -> B,9,5,7,9,7,F,0
    assert p.ravel().tolist() == [0x4DFA8520, 0xB95797F0]


def test_golden_rowwise_and_global():
    W = bf16([ROW_A, ROW_B])
    q, s, z = oracle.quantize(W, "rowwise", 0)
    assert s.shape == (2, 1) and q.tolist() == [ROW_A_Q, ROW_B_Q]
    assert s.ravel().tolist() == [0x3266, 0x3400]
    # GLOBAL: one group over both rows -> min -1.75, max 2 -> s 0.25, z 7;
    # row A: w/s = -4, -2, 0, 2, 4, 8, 6, -1 -> +7 = 3, 5, 7, 9, 11, 15, 13, 6
    q, s, z = oracle.quantize(W, "global", 0)
    assert s.shape == (1, 1) and s[0, 0] == 0x3400 and z[0, 0] == 0x4700
    assert q.tolist() == [[3, 5, 7, 9, 11, 15, 13, 6], ROW_B_Q]


def test_golden_degenerate_groups():
    rows = [[0.5] * 8, [0.0] * 8, [-3.0] * 8, [1.0, 1.5, 2.0, 1.25, 1.75, 1.0, 2.0, 1.5]]
    q, s, z = oracle.quantize(bf16(rows), "groupwise", 8)
    # constant 0.5: s = 0 -> s = max(|min|, 2^-14) = 0.5; z = clamp(rint(-1)) = 0; q = 1
    assert (q[0] == 1).all() and s[0, 0] == 0x3800 and z[0, 0] == 0
    # all zero: s = 2^-14 (0x0400), z = 0, q = 0 -> w_hat = 0 exactly
    assert (q[1] == 0).all() and s[1, 0] == 0x0400 and z[1, 0] == 0
    # constant -3: s = 3 (0x4200), z = 1 (0x3C00), q = rint(-1) + 1 = 0 -> w_hat = -3
    assert (q[2] == 0).all() and s[2, 0] == 0x4200 and z[2, 0] == 0x3C00
    # all positive, min 1 max 2: s = fp16(1/15) = 0.066650390625 (0x2C44); z clamps to 0;
    # every w/s >= 15 so every code clamps to 15 (the clamped integer zero point cannot
    # reach a group that does not straddle zero)
    assert (q[3] == 15).all() and s[3, 0] == 0x2C44 and z[3, 0] == 0
    wh = oracle.dequant(oracle.pack(q), s, z, "groupwise", 8, 8)
    assert wh[0].tolist() == [0.5] * 8 and wh[1].tolist() == [0.0] * 8
    assert wh[2].tolist() == [-3.0] * 8 and wh[3].tolist() == [0.999755859375] * 8


def test_golden_matmul_example():
    W = bf16([ROW_A, ROW_B])
    p, s, z = oracle.quantize_pack(W, "groupwise", 8)
    X = bf16([[1, 0, 0, 0, 0, 0, 0, 0], [1] * 8, [0.5, -1, 2, 0, 0, 0, 0, 1]])
    y64, ybf = oracle.linear(X, p, s, z, "groupwise", 8, 2, 8)
    sA = 0.199951171875
    # row 0 picks w_hat[:,0]: (0-5)*sA and (0-7)*0.25
    # row 1 sums the codes: A: sum(q-z) = 17 -> 17*sA ; B: sum(q-z) = 7 -> 1.75
    # row 2: A: 0.5*(-5) - (-3) + 2*0 + (-1) = -0.5 -> -0.5*sA ; B: -3.5 - 8 + 4 = -7.5 -> -1.875
    expect = [[-5 * sA, -1.75], [17 * sA, 1.75], [-0.5 * sA, -1.875]]
    assert y64.tolist() == expect
    # bf16: -0.99976 -> -1.0 ; 3.39917 -> 218*2^-6 = 3.40625 ; -0.09998 -> -205*2^-11
    assert bf16_value(ybf).tolist() == [[-1.0, -1.75], [3.40625, 1.75], [-0.10009765625, -1.875]]
    # bias epilogue adds bias[n] once before the single rounding
    y64b, _ = oracle.linear(X, p, s, z, "groupwise", 8, 2, 8, bias=bf16([0.25, -1.0]))
    assert (y64b - y64).tolist() == [[0.25, -1.0]] * 3
    # transposed: one-hot dY rows return the dequantized rows, a sum returns their sum
    dY = bf16([[1, 0], [0, 1], [1, 1]])
    x64, _ = oracle.linear_t(dY, p, s, z, "groupwise", 8, 2, 8)
    wa = [(q - 5) * sA for q in ROW_A_Q]
    wb = [(q - 7) * 0.25 for q in ROW_B_Q]
    assert x64.tolist() == [wa, wb, [a + b for a, b in zip(wa, wb)]]


# ----------------------------------------------------------------------------
# bf16 rounding (used for every output)
# ----------------------------------------------------------------------------
def test_bf16_rounding_ties_and_cross_check():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to the even mantissa -> 1.0
    assert oracle.f64_to_bf16(1 + 2.0 ** -8) == 0x3F80
    # 1 + 3*2^-8 is halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even)
    assert oracle.f64_to_bf16(1 + 3 * 2.0 ** -8) == 0x3F82
    assert oracle.f64_to_bf16(-2.0) == 0xC000
    assert oracle.f64_to_bf16(0.0) == 0x0000 and oracle.f64_to_bf16(-0.0) == 0x8000
    # a value a hair above the tie rounds up (no fp32 double rounding)
    assert oracle.f64_to_bf16(1 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81
    # the C routine and the input generator's independent bit trick agree
    rng = np.random.default_rng(5)
    v = rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))
    ref = synth.f64_to_bf16_bits(v)
    got = np.array([oracle.f64_to_bf16(x) for x in v], np.uint16)
    assert (ref == got).all()


# ----------------------------------------------------------------------------
# Quantizer: exact round trip, brute force, error bound
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("g", [8, 16, 64])
def test_exact_round_trip_power_of_two_scales(g):
    """w = (q - z) * 2^-e is exactly representable; quantize must return q, z, 2^-e."""
    rng = np.random.default_rng(11 + g)
    N, G = 24, 5
    K = G * g
    q = rng.integers(0, 16, size=(N, K))
    q[:, ::g] = 0            # every group reaches both ends of the code range
    q[:, 1::g] = 15
    z = rng.integers(0, 16, size=(N, G))
    e = rng.integers(-3, 20, size=(N, G))
    zk = np.repeat(z, g, axis=1)
    ek = np.repeat(e, g, axis=1)
    w = (q - zk) * np.ldexp(1.0, -ek)
    W = bf16(w)
    assert (bf16_value(W) == w).all()
    q2, s2, z2 = oracle.quantize(W, "groupwise", g)
    assert (q2 == q).all()
    assert (z2.view(np.float16).astype(np.float64) == z).all()
    assert (s2.view(np.float16).astype(np.float64) == np.ldexp(1.0, -e)).all()
    wh = oracle.dequant(oracle.pack(q2), s2, z2, "groupwise", g, K)
    assert (wh == w).all()


def _brute_force_group(w_vals, s, z):
    """Nearest code by exact rational distance, ties to even (q - z)."""
    out = []
    sF = Fraction(s)
    for w in w_vals:
        t = Fraction(w) / sF
        best = None
        for cand in range(16):
            d = abs(t - (cand - z))
            key = (d, (cand - z) % 2)
            if best is None or key < best[0]:
                best = (key, cand)
        out.append(best[1])
    return out


def test_brute_force_codes_and_zero_point():
    rng = np.random.default_rng(3)
    g = 16
    W = synth.normal_bf16((40, 4 * g), 0.0, 0.02, seed=7, stream=2)
    W[5, :g] = bf16(rng.uniform(-1, 1, g) * 3)         # wider groups
    W[6, g:2 * g] = bf16(np.round(rng.uniform(-8, 8, g)) * 0.125)   # many exact ties
    q, s, z = oracle.quantize(W, "groupwise", g)
    wv = bf16_value(W)
    for n in range(W.shape[0]):
        for gi in range(4):
            sl = slice(gi * g, (gi + 1) * g)
            sv = f16_value(s[n, gi])
            zv = int(f16_value(z[n, gi]))
            mn = Fraction(float(wv[n, sl].min()))
            # z is the integer nearest -min/s (ties to even), clamped to [0, 15]
            t = -mn / Fraction(sv)
            zf = int(np.floor(t))
            rem = t - zf
            zr = zf + (1 if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and zf % 2) else 0)
            assert zv == min(max(zr, 0), 15)
            assert q[n, sl].tolist() == _brute_force_group(wv[n, sl], sv, zv)


@pytest.mark.parametrize("mode,g", [("groupwise", 32), ("groupwise", 128), ("rowwise", 0),
                                    ("global", 0)])
def test_error_bound_half_step(mode, g):
    """|w - w_hat| <= 0.51 s wherever the group straddles zero."""
    W = synth.normal_bf16((64, 512), 0.0, 0.02, seed=21, stream=2)
    q, s, z = oracle.quantize(W, mode, g)
    K = 512
    wh = oracle.dequant(oracle.pack(q), s, z, mode, g, K)
    sv = s.view(np.float16).astype(np.float64)
    gl = {"groupwise": g, "rowwise": K, "global": K}[mode]
    if mode == "global":
        sk = np.full(W.shape, sv[0, 0])
    else:
        sk = np.repeat(sv, gl, axis=1)
    err = np.abs(bf16_value(W) - wh)
    assert (err <= 0.51 * sk).all()
    # and the scale is the smallest that spans the group: max error is at least s/4 somewhere
    assert err.max() >= 0.25 * sk.min()


def test_groups_are_independent_and_row_local():
    """Quantizing a row subset gives the same codes as quantizing the full matrix."""
    W = synth.normal_bf16((32, 256), 0.0, 0.02, seed=4, stream=2)
    q, s, z = oracle.quantize(W, "groupwise", 64)
    q2, s2, z2 = oracle.quantize(W[10:20], "groupwise", 64)
    assert (q2 == q[10:20]).all() and (s2 == s[10:20]).all() and (z2 == z[10:20]).all()
    # each group only sees its own columns
    W3 = W.copy()
    W3[:, 64:128] = bf16(np.zeros((32, 64)))
    q3, s3, _ = oracle.quantize(W3, "groupwise", 64)
    assert (q3[:, :64] == q[:, :64]).all() and (s3[:, 2:] == s[:, 2:]).all()


def test_invalid_arguments():
    W = synth.normal_bf16((4, 64), 0.0, 0.02, seed=1, stream=2)
    with pytest.raises(ValueError):
        oracle.quantize(W, "groupwise", 48)   # K % g != 0
    with pytest.raises(ValueError):
        oracle.quantize(W, "groupwise", 0)


# ----------------------------------------------------------------------------
# Packing
# ----------------------------------------------------------------------------
def test_pack_golden_words_and_byte_view():
    q = np.array([[0, 1, 2, 3, 4, 5, 6, 7], [15, 0, 0, 0, 0, 0, 0, 0],
                  [0, 0, 0, 0, 0, 0, 0, 15]], np.uint8)
    p = oracle.pack(q)
    assert p.ravel().tolist() == [0x76543210, 0x0000000F, 0xF0000000]
    rng = np.random.default_rng(2)
    q = rng.integers(0, 16, size=(17, 96)).astype(np.uint8)
    p = oracle.pack(q)
    # two codes per byte, low nibble = even k (little-endian byte order of the words)
    by = p.view(np.uint8).reshape(17, 48)
    assert (by == (q[:, 0::2] | (q[:, 1::2] << 4))).all()
    assert (oracle.unpack(p, 96) == q).all()


# ----------------------------------------------------------------------------
# Matmul: brute force, one-hot rows, adjoint identity, bias, column subsets
# ----------------------------------------------------------------------------
@pytest.fixture(scope="module")
def tiny_case():
    """The tiny correctness workload: M=4, K=512, N=256, g=64, seed 0."""
    seed = 0
    X = synth.activations(4, 512, seed)
    W = synth.weights(256, 512, seed)
    dY = synth.grads(4, 256, seed)
    p, s, z = oracle.quantize_pack(W, "groupwise", 64)
    return X, W, dY, p, s, z


def test_matmul_matches_fp64_library_matmul(tiny_case):
    X, W, dY, p, s, z = tiny_case
    wh = oracle.dequant(p, s, z, "groupwise", 64, 512)
    y64, ybf = oracle.linear(X, p, s, z, "groupwise", 64, 256, 512)
    ref = bf16_value(X) @ wh.T
    assert np.allclose(y64, ref, rtol=1e-12, atol=1e-12)
    x64, _ = oracle.linear_t(dY, p, s, z, "groupwise", 64, 256, 512)
    assert np.allclose(x64, bf16_value(dY) @ wh, rtol=1e-12, atol=1e-12)
    assert (ybf == synth.f64_to_bf16_bits(y64)).all()


def test_one_hot_rows_reproduce_dequantized_weights(tiny_case):
    X, W, dY, p, s, z = tiny_case
    wh = oracle.dequant(p, s, z, "groupwise", 64, 512)
    ks = [0, 7, 63, 64, 200, 511]
    E = np.zeros((len(ks), 512))
    E[np.arange(len(ks)), ks] = 1.0
    y64, ybf = oracle.linear(bf16(E), p, s, z, "groupwise", 64, 256, 512)
    assert (y64 == wh[:, ks].T).all()
    assert (ybf == synth.f64_to_bf16_bits(wh[:, ks].T)).all()
    ns = [0, 1, 128, 255]
    D = np.zeros((len(ns), 256))
    D[np.arange(len(ns)), ns] = 1.0
    x64, _ = oracle.linear_t(bf16(D), p, s, z, "groupwise", 64, 256, 512)
    assert (x64 == wh[ns]).all()


def test_adjoint_identity(tiny_case):
    X, W, dY, p, s, z = tiny_case
    y64, _ = oracle.linear(X, p, s, z, "groupwise", 64, 256, 512)
    x64, _ = oracle.linear_t(dY, p, s, z, "groupwise", 64, 256, 512)
    lhs = float(np.sum(y64 * bf16_value(dY)))
    rhs = float(np.sum(bf16_value(X) * x64))
    assert abs(lhs - rhs) <= 1e-9 * (abs(lhs) + 1.0)


def test_bias_and_column_subsets(tiny_case):
    X, W, dY, p, s, z = tiny_case
    b = synth.bias(256, 0)
    y0, _ = oracle.linear(X, p, s, z, "groupwise", 64, 256, 512)
    yb, _ = oracle.linear(X, p, s, z, "groupwise", 64, 256, 512, bias=b)
    assert np.allclose(yb - y0, bf16_value(b)[None, :], rtol=0, atol=1e-12)
    cols = np.array([255, 3, 3, 100])
    ys, _ = oracle.linear(X, p, s, z, "groupwise", 64, 256, 512, bias=b, cols=cols)
    assert (ys == yb[:, cols]).all()
    bk = synth.bias(512, 1)
    x0, _ = oracle.linear_t(dY, p, s, z, "groupwise", 64, 256, 512)
    xb, _ = oracle.linear_t(dY, p, s, z, "groupwise", 64, 256, 512, bias=bk)
    assert np.allclose(xb - x0, bf16_value(bk)[None, :], rtol=0, atol=1e-12)
    kc = np.array([511, 0, 64])
    xs, _ = oracle.linear_t(dY, p, s, z, "groupwise", 64, 256, 512, bias=bk, cols=kc)
    assert (xs == xb[:, kc]).all()


@pytest.mark.parametrize("mode,g", [("groupwise", 64), ("rowwise", 0)])
def test_fused_qkv_equivalence(mode, g):
    """Fused Q/K/V weights concatenated along N (torchao "Add fused QKV HQQ
    triton_mm test"): forward is the concatenation, transposed is the sum."""
    K = 256
    parts = [synth.weights(n, K, 30 + i) for i, n in enumerate([64, 32, 32])]
    qs = [oracle.quantize_pack(Wp, mode, g) for Wp in parts]
    Wf = np.concatenate(parts, axis=0)
    pf, sf, zf = oracle.quantize_pack(Wf, mode, g)
    assert (pf == np.concatenate([t[0] for t in qs])).all()
    assert (sf == np.concatenate([t[1] for t in qs])).all()
    X = synth.activations(3, K, 5)
    yf, _ = oracle.linear(X, pf, sf, zf, mode, g, 128, K)
    ys = [oracle.linear(X, *t, mode, g, Wp.shape[0], K)[0] for t, Wp in zip(qs, parts)]
    assert (yf == np.concatenate(ys, axis=1)).all()
    dY = synth.grads(3, 128, 6)
    xf, _ = oracle.linear_t(dY, pf, sf, zf, mode, g, 128, K)
    offs = [0, 64, 96, 128]
    xs = [oracle.linear_t(dY[:, offs[i]:offs[i + 1]], *qs[i], mode, g, offs[i + 1] - offs[i], K)[0]
          for i in range(3)]
    assert np.allclose(xf, xs[0] + xs[1] + xs[2], rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------
# Soft band: the llm-quantization page's MAE column (not an exact pin)
# ----------------------------------------------------------------------------
def test_quantization_mae_soft_band():
    rows = []
    with open(os.path.join(GOLDEN, "llm_quantization_mae.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            mode, g, mae = line.split()
            rows.append((mode, int(g), float(mae)))
    W = synth.normal_bf16((2048, 2048), 0.0, 1.0, seed=8, stream=2)
    wv = bf16_value(W)
    for mode, g, page_mae in rows:
        # the page's ROWWISE row disagrees with its own 4096-long groups (0.0969 vs
        # 0.1189), so only GLOBAL and groups up to the row length are compared
        if mode == "ROWWISE" or g > 2048:
            continue
        m = mode.lower()
        q, s, z = oracle.quantize(W, m, g)
        wh = oracle.dequant(oracle.pack(q), s, z, m, g, 2048)
        mae = float(np.mean(np.abs(wv - wh)))
        assert 0.75 * page_mae <= mae <= 1.25 * page_mae, (mode, g, mae, page_mae)


# ----------------------------------------------------------------------------
# Variant: fractional zero point and bf16 scales / zeros (the HQQ-style
# quantizer of "Re-write HQQ Fused Gemm Transpose"; fp16 or bf16 metadata).
# Reading: s = meta((max - min) / 15); z = meta(-min / s), not rounded to an
# integer and not clamped to [0, 15]; q = clamp(rint(w / s + z), 0, 15).
# ----------------------------------------------------------------------------
def meta_value(bits, meta):
    b = np.asarray(bits, dtype=np.uint16)
    if meta == "bf16":
        return bf16_value(b)
    return b.view(np.float16).astype(np.float64)


ROW_C = [-0.15625, 0.78125, 0.0, 0.03125, 0.1, -0.1, 0.5, 0.25]
# bf16 inputs: 0.1 -> 0.10009765625 (= 205 * 2^-11), the rest exact.
# min -0.15625, max 0.78125: range 0.9375 = 15/16 -> s = 1/16 exactly (fp16 0x2C00,
# bf16 0x3D80); z = 0.15625 * 16 = 2.5 exactly (fp16 0x4100, bf16 0x4020).
# w/s + z = 0, 15, 2.5, 3, 4.1015625, 0.8984375, 10.5, 6.5 -> rint (ties to even):
ROW_C_Q = [0, 15, 2, 3, 4, 1, 10, 6]
# the integer-zero reading differs: z = rint(2.5) = 2, rint(w/s) + 2 = 0, 14, 2, 2, 4, 0, 10, 6
ROW_C_Q_INT = [0, 14, 2, 2, 4, 0, 10, 6]
ROW_D = [1.0, 1.5, 2.0, 1.25, 1.75, 1.0, 2.0, 1.5]
# all positive: s = fp16(1/15) = 0.066650390625 (0x2C44); -min/s = -15.00366...
# -> fp16 (step 2^-7 in [8, 16)) = -15.0 (0xCB80); w/s - 15 = 0.0037, 7.5055, 15.0073,
# 3.7546, 11.2564, ... -> q = 0, 8, 15, 4, 11, 0, 15, 8: the whole code range is used,
# where the clamped integer zero point maps every w to 15.
ROW_D_Q = [0, 8, 15, 4, 11, 0, 15, 8]


@pytest.mark.parametrize("meta,s_bits,z_bits", [("fp16", 0x2C00, 0x4100), ("bf16", 0x3D80, 0x4020)])
def test_golden_float_zero_example(meta, s_bits, z_bits):
    q, s, z = oracle.quantize(bf16([ROW_C]), "groupwise", 8, zero="float", meta=meta)
    assert q.tolist() == [ROW_C_Q]
    assert s.ravel().tolist() == [s_bits] and z.ravel().tolist() == [z_bits]
    assert oracle.pack(q).ravel().tolist() == [0x6A1432F0]
    wh = oracle.dequant(oracle.pack(q), s, z, "groupwise", 8, 8, meta=meta)
    assert wh.ravel().tolist() == [(c - 2.5) / 16 for c in ROW_C_Q]
    qi, _, zi = oracle.quantize(bf16([ROW_C]), "groupwise", 8, zero="int", meta=meta)
    assert qi.tolist() == [ROW_C_Q_INT] and meta_value(zi, meta).ravel().tolist() == [2.0]


def test_golden_float_zero_all_positive_group():
    q, s, z = oracle.quantize(bf16([ROW_D]), "groupwise", 8, zero="float")
    assert s.ravel().tolist() == [0x2C44] and z.ravel().tolist() == [0xCB80]
    assert q.tolist() == [ROW_D_Q]
    wh = oracle.dequant(oracle.pack(q), s, z, "groupwise", 8, 8)
    assert np.abs(wh - bf16_value(bf16([ROW_D]))).max() <= 0.5 * 0.066650390625 + 1e-12
    # constant groups reconstruct exactly: s = |w|, z = -sign(w)
    q, s, z = oracle.quantize(bf16([[0.5] * 8, [-3.0] * 8, [0.0] * 8]), "groupwise", 8, zero="float")
    wh = oracle.dequant(oracle.pack(q), s, z, "groupwise", 8, 8)
    assert wh.tolist() == [[0.5] * 8, [-3.0] * 8, [0.0] * 8]


@pytest.mark.parametrize("meta", ["fp16", "bf16"])
@pytest.mark.parametrize("g", [8, 16, 64])
def test_float_zero_exact_round_trip(meta, g):
    """w = (q - z) * 2^-e with a fractional z on a quarter grid: exactly representable;
    quantize must return q, z and 2^-e."""
    rng = np.random.default_rng(31 + g)
    N, G = 24, 5
    K = G * g
    q = rng.integers(0, 16, size=(N, K))
    q[:, ::g] = 0
    q[:, 1::g] = 15
    z = rng.integers(-60, 121, size=(N, G)) / 4.0          # -15 .. 30 in quarter steps
    e = rng.integers(-3, 20, size=(N, G))
    w = (q - np.repeat(z, g, axis=1)) * np.ldexp(1.0, -np.repeat(e, g, axis=1))
    W = bf16(w)
    assert (bf16_value(W) == w).all()
    q2, s2, z2 = oracle.quantize(W, "groupwise", g, zero="float", meta=meta)
    assert (q2 == q).all()
    assert (meta_value(z2, meta) == z).all()
    assert (meta_value(s2, meta) == np.ldexp(1.0, -e)).all()
    wh = oracle.dequant(oracle.pack(q2), s2, z2, "groupwise", g, K, meta=meta)
    assert (wh == w).all()


@pytest.mark.parametrize("meta", ["fp16", "bf16"])
def test_float_zero_brute_force_codes(meta):
    """Each code is the nearest of the 16 levels to u = fp32(fp32(w / s) + z), found by
    exhaustive search (ties to the even level), and z is within one rounding of -min/s."""
    g = 16
    W = synth.normal_bf16((40, 4 * g), 0.0, 0.02, seed=9, stream=2)
    W[3, :g] = bf16(np.abs(synth.bf16_bits_to_f32(W[3, :g])) + 0.05)     # all positive
    W[4, g:2 * g] = bf16(-np.abs(synth.bf16_bits_to_f32(W[4, g:2 * g])) - 0.05)
    q, s, z = oracle.quantize(W, "groupwise", g, zero="float", meta=meta)
    wv = synth.bf16_bits_to_f32(W)
    zrel = 2.0 ** -8 if meta == "bf16" else 2.0 ** -11          # half a step of the type
    for n in range(W.shape[0]):
        for gi in range(4):
            sl = slice(gi * g, (gi + 1) * g)
            sv = np.float32(meta_value(s[n, gi], meta))
            zv = np.float32(meta_value(z[n, gi], meta))
            exact = -Fraction(float(wv[n, sl].min())) / Fraction(float(sv))
            assert abs(Fraction(float(zv)) - exact) <= abs(exact) * Fraction(zrel) * Fraction(1001, 1000)
            for w, code in zip(wv[n, sl], q[n, sl]):
                u = np.float32(np.float32(w) / sv) + zv
                d = [abs(Fraction(float(u)) - lv) for lv in range(16)]
                best = min(range(16), key=lambda lv: (d[lv], lv % 2))
                assert code == best


@pytest.mark.parametrize("meta", ["fp16", "bf16"])
@pytest.mark.parametrize("mode,g", [("groupwise", 32), ("groupwise", 128), ("rowwise", 0), ("global", 0)])
def test_float_zero_error_bound(meta, mode, g):
    """|w - w_hat| <= (1/2 + |z - (-min/s)|) s: half a step plus the zero point's rounding,
    for every group, with or without zero inside it."""
    K = 512
    W = synth.normal_bf16((64, K), 0.0, 0.02, seed=22, stream=2)
    W[:8] = bf16(np.abs(synth.bf16_bits_to_f32(W[:8])) + 0.01)          # groups away from zero
    q, s, z = oracle.quantize(W, mode, g, zero="float", meta=meta)
    wh = oracle.dequant(oracle.pack(q), s, z, mode, g, K, meta=meta)
    w = bf16_value(W)
    gl = {"groupwise": g, "rowwise": K, "global": K}[mode]
    sv, zv = meta_value(s, meta), meta_value(z, meta)
    if mode == "global":
        sk, zk = np.full(W.shape, sv[0, 0]), np.full(W.shape, zv[0, 0])
        mn = np.full(W.shape, w.min())
    else:
        sk, zk = np.repeat(sv, gl, axis=1), np.repeat(zv, gl, axis=1)
        mn = np.repeat(w.reshape(64, -1, gl).min(axis=2), gl, axis=1)
    zerr = np.abs(zk + mn / sk)
    err = np.abs(w - wh)
    assert (err <= (0.5 + zerr + 2.0 ** -12) * sk).all()
    # the zero point follows the group: codes 0 and 15 are both used in most groups
    if mode == "groupwise":
        used = (q.reshape(64, -1, g).min(axis=2) == 0) & (q.reshape(64, -1, g).max(axis=2) == 15)
        assert used.mean() > 0.9


def test_float_zero_reduces_to_integer_zero_when_min_is_on_the_grid():
    """If -min/s is an integer in [0, 15] and no w/s sits on a half step, both readings
    give the same codes, scale and zero value."""
    rng = np.random.default_rng(17)
    g, G, N = 16, 4, 12
    zi = rng.integers(0, 16, size=(N, G))
    e = rng.integers(2, 12, size=(N, G))
    lev = rng.integers(0, 16, size=(N, G * g)).astype(np.float64)
    frac = rng.uniform(-0.4, 0.4, size=lev.shape)
    frac[:, ::g] = 0.0
    lev[:, ::g] = 0.0                      # the minimum sits on level 0 ...
    frac[:, 1::g] = 0.0
    lev[:, 1::g] = 15.0                    # ... and the maximum on level 15
    t = np.clip(lev + frac, 0.0, 15.0) - np.repeat(zi, g, axis=1)
    w = bf16_value(bf16(t * np.ldexp(1.0, -np.repeat(e, g, axis=1))))
    W = bf16(w)
    for meta in ("fp16", "bf16"):
        qf, sf, zf = oracle.quantize(W, "groupwise", g, zero="float", meta=meta)
        qi, si, zi2 = oracle.quantize(W, "groupwise", g, zero="int", meta=meta)
        assert (qf == qi).all() and (sf == si).all()
        assert (meta_value(zf, meta) == meta_value(zi2, meta)).all()
        assert (meta_value(zf, meta) == zi).all()


def test_bf16_metadata_matches_fp16_where_both_are_exact():
    """With power-of-two scales and integer zeros the bf16-metadata quantizer returns the
    same codes and values as the fp16 one (only the bit patterns differ)."""
    rng = np.random.default_rng(23)
    g, G, N = 32, 3, 10
    q = rng.integers(0, 16, size=(N, G * g))
    q[:, ::g] = 0
    q[:, 1::g] = 15
    z = rng.integers(0, 16, size=(N, G))
    e = rng.integers(-2, 14, size=(N, G))
    w = (q - np.repeat(z, g, axis=1)) * np.ldexp(1.0, -np.repeat(e, g, axis=1))
    W = bf16(w)
    q16, s16, z16 = oracle.quantize(W, "groupwise", g)
    qb, sb, zb = oracle.quantize(W, "groupwise", g, meta="bf16")
    assert (q16 == qb).all()
    assert (meta_value(s16, "fp16") == meta_value(sb, "bf16")).all()
    assert (meta_value(z16, "fp16") == meta_value(zb, "bf16")).all()
    # bf16 rounds the scale to 8 significant bits: a non-power-of-two range shows it
    qb, sb, _ = oracle.quantize(bf16([ROW_A]), "groupwise", 8, meta="bf16")
    assert sb.ravel().tolist() == [0x3E4D]          # 0.2 -> 205 * 2^-10 = 0.2001953125


@pytest.mark.parametrize("zero,meta", [("float", "fp16"), ("float", "bf16"), ("int", "bf16")])
def test_variant_matmul_one_hot_and_adjoint(zero, meta):
    """linear / linear_t read the variant's metadata: one-hot rows return the dequantized
    weights, and <X W^T, dY> = <X, dY W>."""
    seed = 0
    X = synth.activations(4, 512, seed)
    W = synth.weights(256, 512, seed)
    dY = synth.grads(4, 256, seed)
    p, s, z = oracle.quantize_pack(W, "groupwise", 64, zero=zero, meta=meta)
    wh = oracle.dequant(p, s, z, "groupwise", 64, 512, meta=meta)
    ks = [0, 63, 64, 511]
    E = np.zeros((len(ks), 512))
    E[np.arange(len(ks)), ks] = 1.0
    y64, _ = oracle.linear(bf16(E), p, s, z, "groupwise", 64, 256, 512, meta=meta)
    assert (y64 == wh[:, ks].T).all()
    y64, _ = oracle.linear(X, p, s, z, "groupwise", 64, 256, 512, meta=meta)
    x64, _ = oracle.linear_t(dY, p, s, z, "groupwise", 64, 256, 512, meta=meta)
    lhs = float(np.sum(y64 * bf16_value(dY)))
    rhs = float(np.sum(bf16_value(X) * x64))
    assert abs(lhs - rhs) <= 1e-9 * (abs(lhs) + 1.0)
    assert np.allclose(y64, bf16_value(X) @ wh.T, rtol=1e-12, atol=1e-12)


def test_act_order_reading_reduces_to_the_unpermuted_product():
    """Act-order: packed column j holds input channel perm[j].  Quantizing W[:, perm] and
    multiplying X[:, perm] equals the plain product with the dequantized weights put back in
    channel order (w_full[:, perm[j]] = w_hat[:, j]); the transposed product lands in
    dX[:, perm]."""
    N, K, g = 48, 256, 32
    W = synth.weights(N, K, 13)
    X = synth.activations(3, K, 13)
    dY = synth.grads(3, N, 13)
    perm = np.random.default_rng(13).permutation(K)
    p, s, z = oracle.quantize_pack(W[:, perm], "groupwise", g)
    wh = oracle.dequant(p, s, z, "groupwise", g, K)
    w_full = np.empty_like(wh)
    w_full[:, perm] = wh
    y64, _ = oracle.linear(X[:, perm], p, s, z, "groupwise", g, N, K)
    assert np.allclose(y64, bf16_value(X) @ w_full.T, rtol=1e-12, atol=1e-12)
    x64p, _ = oracle.linear_t(dY, p, s, z, "groupwise", g, N, K)
    x64 = np.empty_like(x64p)
    x64[:, perm] = x64p
    assert np.allclose(x64, bf16_value(dY) @ w_full, rtol=1e-12, atol=1e-12)
    # with the identity permutation it is the ordinary layer
    p0, s0, z0 = oracle.quantize_pack(W, "groupwise", g)
    pi = np.arange(K)
    pi_p, pi_s, pi_z = oracle.quantize_pack(W[:, pi], "groupwise", g)
    assert (pi_p == p0).all() and (pi_s == s0).all() and (pi_z == z0).all()
