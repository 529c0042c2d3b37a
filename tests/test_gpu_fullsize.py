"""Parity at the workloads' full sizes, in the launch configurations the bench
times, on sampled output columns the oracle computes one by one.

The rms of the tolerance is taken over the sampled columns (an estimate of
the full tensor's rms).  Quantize-and-pack is compared bit for bit on the
whole matrix.  GEMV results are also checked for run-to-run determinism.
"""
import numpy as np
import pytest

import oracle
from gemv_w4a16_groupwise_b200 import synth

from gpu_helpers import assert_close, from_dev_bits, to_dev_bf16, to_dev_f16, to_dev_packed

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def sample_cols(n, count, seed):
    rng = np.random.default_rng(seed)
    idx = rng.choice(n, size=min(count, n), replace=False)
    return np.unique(np.concatenate([idx, [0, n - 1]]))


def quantize_both(W, mode, g, dev):
    import gemv_w4a16_groupwise_b200 as w4
    p_ref, s_ref, z_ref = oracle.quantize_pack(W, mode, g)
    p, s, z = w4.w4_quantize_pack(to_dev_bf16(W, dev), mode, g)
    assert (p.cpu().numpy().view(np.uint32) == p_ref).all(), "packed not bit-exact"
    assert (from_dev_bits(s) == s_ref).all(), "scales not bit-exact"
    assert (from_dev_bits(z) == z_ref).all(), "zeros not bit-exact"
    return (p, s, z), (p_ref, s_ref, z_ref)


@pytest.mark.parametrize("N,K", [(16384, 16384), (12288, 12288), (24576, 2048)])
@pytest.mark.parametrize("mode,g", [("groupwise", 128), ("rowwise", 0)])
def test_decode_sweep_gemv(cuda_device, N, K, mode, g):
    """Decode GEMV sweep sizes (M = 1..4), multi-unit persistent CTAs, K split."""
    import gemv_w4a16_groupwise_b200 as w4
    dev = cuda_device
    seed = synth.config_seed("sweep", N, K)
    W = synth.weights(N, K, seed)
    (p, s, z), (p_ref, s_ref, z_ref) = quantize_both(W, mode, g, dev)
    cols = sample_cols(N, 192, seed)
    for M in (1, 2, 3, 4):
        X = synth.activations(M, K, seed + M)
        Xd = to_dev_bf16(X, dev)
        y1 = w4.w4a16_gemv(Xd, p, s, z, mode, g, N=N, K=K)
        y2 = w4.w4a16_gemv(Xd, p, s, z, mode, g, N=N, K=K)
        import torch
        assert torch.equal(y1, y2), "GEMV is not deterministic"
        ref, _ = oracle.linear(X, p_ref, s_ref, z_ref, mode, g, N, K, cols=cols)
        assert_close(from_dev_bits(y1)[:, cols], ref, f"sweep M={M} N={N} {mode}")
        dY = synth.grads(M, N, seed + M)
        x = w4.w4a16_gemv(to_dev_bf16(dY, dev), p, s, z, mode, g, N=N, K=K, transposed=True)
        kc = sample_cols(K, 96, seed + 1)
        ref_t, _ = oracle.linear_t(dY, p_ref, s_ref, z_ref, mode, g, N, K, cols=kc)
        assert_close(from_dev_bits(x)[:, kc], ref_t, f"sweep^T M={M} N={N} {mode}")
    assert w4.w4_device_error() == 0


@pytest.mark.parametrize("mode,g", [("groupwise", 64), ("rowwise", 0), ("global", 0)])
def test_llama32_1b_lm_head(cuda_device, mode, g):
    """Llama-3.2-1B shapes: quantize (128256 x 2048) bit-exact; GEMM at M = 2048."""
    import gemv_w4a16_groupwise_b200 as w4
    dev = cuda_device
    N, K = 128256, 2048
    seed = synth.config_seed("l32", N, K)
    W = synth.weights(N, K, seed)
    (p, s, z), (p_ref, s_ref, z_ref) = quantize_both(W, mode, g, dev)
    cols = sample_cols(N, 64, seed)
    for M in (128, 2048):
        X = synth.activations(M, K, seed + M)
        y = w4.w4a16_gemm(to_dev_bf16(X, dev), p, s, z, mode, g, N=N, K=K)
        ref, _ = oracle.linear(X, p_ref, s_ref, z_ref, mode, g, N, K, cols=cols)
        assert_close(from_dev_bits(y)[:, cols], ref, f"l32 M={M} {mode}")
    assert w4.w4_device_error() == 0


@pytest.mark.parametrize("N,K", [(12288, 4096), (4096, 11008)])
@pytest.mark.parametrize("mode,g", [("groupwise", 64), ("rowwise", 0)])
def test_llama2_7b_qlora(cuda_device, N, K, mode, g):
    """QLoRA shapes at M = 2048: forward and transposed from the same packed W."""
    import gemv_w4a16_groupwise_b200 as w4
    dev = cuda_device
    M = 2048
    seed = synth.config_seed("l27", N, K)
    W = synth.weights(N, K, seed)
    (p, s, z), (p_ref, s_ref, z_ref) = quantize_both(W, mode, g, dev)
    X = synth.activations(M, K, seed)
    y = w4.w4a16_gemm(to_dev_bf16(X, dev), p, s, z, mode, g, N=N, K=K)
    cols = sample_cols(N, 48, seed)
    ref, _ = oracle.linear(X, p_ref, s_ref, z_ref, mode, g, N, K, cols=cols)
    assert_close(from_dev_bits(y)[:, cols], ref, "qlora fwd")
    dY = synth.grads(M, N, seed)
    x = w4.w4a16_gemm(to_dev_bf16(dY, dev), p, s, z, mode, g, N=N, K=K, transposed=True)
    kc = sample_cols(K, 48, seed + 1)
    ref_t, _ = oracle.linear_t(dY, p_ref, s_ref, z_ref, mode, g, N, K, cols=kc)
    assert_close(from_dev_bits(x)[:, kc], ref_t, "qlora transposed")
    assert w4.w4_device_error() == 0


@pytest.mark.parametrize("M", [1, 4, 16, 64, 256, 1024])
def test_llama3_8b_serving_bias(cuda_device, M):
    """Serving shapes with the bias epilogue, g = 128 (gate_up N = 28672)."""
    import gemv_w4a16_groupwise_b200 as w4
    dev = cuda_device
    N, K = 28672, 4096
    seed = synth.config_seed("l38", N, K)
    W = synth.weights(N, K, seed)
    (p, s, z), (p_ref, s_ref, z_ref) = quantize_both(W, "groupwise", 128, dev)
    X = synth.activations(M, K, seed + M)
    b = synth.bias(N, seed)
    y = w4.w4a16_gemm(to_dev_bf16(X, dev), p, s, z, "groupwise", 128, N=N, K=K,
                      bias=to_dev_bf16(b, dev))
    cols = sample_cols(N, 96, seed)
    ref, _ = oracle.linear(X, p_ref, s_ref, z_ref, "groupwise", 128, N, K, bias=b, cols=cols)
    assert_close(from_dev_bits(y)[:, cols], ref, f"l38 M={M}")
    assert w4.w4_device_error() == 0


@pytest.mark.parametrize("mode,g", [("groupwise", 128), ("rowwise", 0), ("global", 0)])
def test_llama3_8b_transposed_gemv(cuda_device, mode, g):
    """Transposed GEMV (M = 1..4) at the gate_up shape N = 28672, K = 4096:
    every row split of the grid, sampled output columns, run to run equal."""
    import torch
    import gemv_w4a16_groupwise_b200 as w4
    dev = cuda_device
    N, K = 28672, 4096
    seed = synth.config_seed("l38t", N, K)
    W = synth.weights(N, K, seed)
    (p, s, z), (p_ref, s_ref, z_ref) = quantize_both(W, mode, g, dev)
    kc = sample_cols(K, 96, seed)
    for M in (1, 2, 3, 4):
        dY = synth.grads(M, N, seed + M)
        dYd = to_dev_bf16(dY, dev)
        x1 = w4.w4a16_gemv(dYd, p, s, z, mode, g, N=N, K=K, transposed=True)
        x2 = w4.w4a16_gemv(dYd, p, s, z, mode, g, N=N, K=K, transposed=True)
        assert torch.equal(x1, x2), "transposed GEMV is not deterministic"
        ref, _ = oracle.linear_t(dY, p_ref, s_ref, z_ref, mode, g, N, K, cols=kc)
        assert_close(from_dev_bits(x1)[:, kc], ref, f"l38^T M={M} {mode}")
    assert w4.w4_device_error() == 0
