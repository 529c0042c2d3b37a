"""GPU parity of the small-batch (M <= 4) GEMV paths on activations with a wide
dynamic range, against the CPU oracle at the stated tolerance.

LLM decode activations carry outliers: a handful of channels orders of
magnitude above the rest.  A kernel that brings a block of activations to one
common fixed-point scale rounds the small ones relative to the block's
largest, which shows when the large one meets a zero weight (its product
vanishes, the rounding of the others does not).  These cases plant exactly
that: one +-2^e activation in every 128 k (e = 8, 12, 16), with and without
an all-zero weight column under it; granules that mix 2^-20 and 2^4 values;
and, for the transposed product, dY outliers over all-zero weight rows and
weight rows whose quantization scales spread over 2^10.  Every output element
must satisfy |y - y_ref| <= 1e-2 rms(y_ref) + 2^-7 |y_ref|.
"""
import numpy as np
import pytest

import oracle
from gemv_w4a16_groupwise_b200 import synth

from gpu_helpers import assert_close, from_dev_bits, to_dev_bf16, to_dev_f16, to_dev_packed

pytestmark = pytest.mark.gpu

FWD_SHAPES = [
    # (N, K, mode, g): g = 128 and one group per row (the decode workloads),
    # g = 64 and 32 (the other word layouts), a long K
    (256, 4096, "groupwise", 128),
    (200, 2048, "rowwise", 0),
    (128, 1024, "groupwise", 64),
    (96, 1024, "groupwise", 32),
    (64, 16384, "groupwise", 128),
]


def _lib():
    import gemv_w4a16_groupwise_b200 as w4
    return w4


def _quantize(W, mode, g):
    return oracle.quantize_pack(W, mode, g)


def _forward(dev, X, W, mode, g):
    w4 = _lib()
    M, K = X.shape
    N = W.shape[0]
    p, s, z = _quantize(W, mode, g)
    Y = w4.w4a16_gemv(to_dev_bf16(X, dev), to_dev_packed(p, dev), to_dev_f16(s, dev), to_dev_f16(z, dev),
                      mode, g, N=N, K=K)
    ref, _ = oracle.linear(X, p, s, z, mode, g, N, K)
    return from_dev_bits(Y), ref


def _transposed(dev, dY, W, mode, g):
    w4 = _lib()
    M, N = dY.shape
    K = W.shape[1]
    p, s, z = _quantize(W, mode, g)
    dX = w4.w4a16_gemv(to_dev_bf16(dY, dev), to_dev_packed(p, dev), to_dev_f16(s, dev), to_dev_f16(z, dev),
                       mode, g, N=N, K=K, transposed=True)
    ref, _ = oracle.linear_t(dY, p, s, z, mode, g, N, K)
    return from_dev_bits(dX), ref


@pytest.mark.parametrize("zero_column", [False, True])
@pytest.mark.parametrize("exp", [8, 12, 16])
@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("N,K,mode,g", FWD_SHAPES)
def test_forward_activation_outliers(cuda_device, N, K, mode, g, M, exp, zero_column):
    seed = synth.config_seed("outlier_fwd", N, K, mode, g, M, exp, zero_column)
    X, pos = synth.outlier_activations(M, K, seed, exp)
    W = synth.weights(N, K, seed)
    if zero_column:
        W[:, pos] = 0          # w = 0 quantizes to q = z exactly: w_hat = 0 under every outlier
    y, ref = _forward(cuda_device, X, W, mode, g)
    assert_close(y, ref, f"fwd outliers 2^{exp} zero_col={zero_column} M={M} N={N} K={K} {mode} g={g}")


@pytest.mark.parametrize("zero_large", [False, True])
@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("N,K,mode,g", FWD_SHAPES)
def test_forward_mixed_range_granules(cuda_device, N, K, mode, g, M, zero_large):
    seed = synth.config_seed("mixed_fwd", N, K, mode, g, M, zero_large)
    X, pos = synth.mixed_range_activations(M, K, seed, lo_exp=-20, hi_exp=4)
    W = synth.weights(N, K, seed)
    if zero_large:
        W[:, pos] = 0          # only the 2^-20 values reach the output
    y, ref = _forward(cuda_device, X, W, mode, g)
    assert_close(y, ref, f"fwd mixed zero_large={zero_large} M={M} N={N} K={K} {mode} g={g}")


def test_forward_single_outlier_over_zero_column(cuda_device):
    """One 2^14 activation at k = 0 over an all-zero weight column, N(0, 1)
    elsewhere: a block fixed point per 128 k would round the other 127
    activations of that block to multiples of 2."""
    M, N, K = 1, 512, 4096
    X = synth.activations(M, K, 5)
    X[0, 0] = synth.f64_to_bf16_bits(np.array([2.0 ** 14]))[0]
    W = synth.weights(N, K, 5)
    W[:, 0] = 0
    y, ref = _forward(cuda_device, X, W, "groupwise", 128)
    assert_close(y, ref, "single outlier over a zero column")


T_SHAPES = [
    # (N, K, mode, g) with N the reduction length of the transposed product
    (2048, 1024, "groupwise", 128),
    (1024, 2048, "rowwise", 0),
    (4096, 512, "groupwise", 64),
    (28672, 256, "groupwise", 128),
]


@pytest.mark.parametrize("zero_rows", [False, True])
@pytest.mark.parametrize("exp", [8, 12, 16])
@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("N,K,mode,g", T_SHAPES)
def test_transposed_dy_outliers(cuda_device, N, K, mode, g, M, exp, zero_rows):
    seed = synth.config_seed("outlier_t", N, K, mode, g, M, exp, zero_rows)
    dY, pos = synth.outlier_activations(M, N, seed, exp, period=32, stream=synth.STREAM_DY)
    W = synth.weights(N, K, seed)
    if zero_rows:
        W[pos, :] = 0          # an all-zero row quantizes to w_hat = 0 exactly
    dx, ref = _transposed(cuda_device, dY, W, mode, g)
    assert_close(dx, ref, f"t outliers 2^{exp} zero_rows={zero_rows} M={M} N={N} K={K} {mode} g={g}")


@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("N,K,mode,g", T_SHAPES)
def test_transposed_row_scale_spread(cuda_device, N, K, mode, g, M):
    """Weight rows scaled by powers of two over 2^10, so that dY s spans ten
    binades more than dY alone, plus dY outliers on top."""
    seed = synth.config_seed("spread_t", N, K, mode, g, M)
    dY, _ = synth.outlier_activations(M, N, seed, 10, period=256, stream=synth.STREAM_DY)
    W = synth.spread_rows(synth.weights(N, K, seed), seed, binades=10)
    dx, ref = _transposed(cuda_device, dY, W, mode, g)
    assert_close(dx, ref, f"t spread M={M} N={N} K={K} {mode} g={g}")


@pytest.mark.parametrize("M", [1, 4])
@pytest.mark.parametrize("N,K,mode,g", T_SHAPES)
def test_transposed_mixed_range(cuda_device, N, K, mode, g, M):
    """dY mixing 2^-20 and 2^4 values, the large ones over all-zero weight rows."""
    seed = synth.config_seed("mixed_t", N, K, mode, g, M)
    dY, pos = synth.mixed_range_activations(M, N, seed, lo_exp=-20, hi_exp=4, stream=synth.STREAM_DY)
    W = synth.weights(N, K, seed)
    W[pos, :] = 0
    dx, ref = _transposed(cuda_device, dY, W, mode, g)
    assert_close(dx, ref, f"t mixed M={M} N={N} K={K} {mode} g={g}")
