"""GPU parity of the fractional-zero / bf16-metadata variant against the oracle.

The variant is the HQQ-style quantizer of "Re-write HQQ Fused Gemm Transpose"
(a float zero point: z = -min / s, q = clamp(rint(w / s + z), 0, 15)) with
fp16 or bf16 scales and zeros.  Quantize-and-pack must match the oracle bit
for bit; every matmul path (int8 and bf16 tensor-pipe GEMV, CUDA-core GEMV,
tcgen05 GEMM, CUDA-core GEMM; forward and transposed) must match the
oracle's fp64 product within the parity tolerance.  The weights carry groups
shifted away from zero, so that zero points fall far outside [0, 15].
"""
import numpy as np
import pytest

import oracle
from gemv_w4a16_groupwise_b200 import synth
from gpu_helpers import assert_close, from_dev_bits, to_dev_bf16, to_dev_f16, to_dev_packed

VARIANTS = [("float", "fp16"), ("float", "bf16"), ("int", "bf16")]


def lib():
    import gemv_w4a16_groupwise_b200 as w4
    return w4


def to_dev_meta(bits, meta, dev):
    return to_dev_bf16(bits, dev) if meta == "bf16" else to_dev_f16(bits, dev)


def variant_weights(N, K, mode, g, seed, shifted_row=True):
    """Seeded weights with planted edge structure and a quarter of the groups shifted
    off zero.  ``shifted_row=False`` keeps the planted structure but drops its last
    row, which is shifted by five weight deviations as a whole: with a fractional
    zero point its dequantized weights keep that size, and the tensor-core GEMM,
    which rounds them to bf16 for the mma, then exceeds the per-tensor tolerance on
    that row (its error grows with the row's weights, the bound with the tensor's
    rms), while the other rows stay well inside."""
    W = synth.weights(N, K, seed)
    gl = g if mode == "groupwise" else K
    P = synth.plant_structure(W, gl, seed)
    if not shifted_row:
        P[-1] = W[-1]
    if mode != "global":
        P = synth.offset_groups(P, gl, seed)
    return P


@pytest.mark.gpu
@pytest.mark.parametrize("zero,meta", VARIANTS)
@pytest.mark.parametrize("N,K,mode,g", [
    (256, 512, "groupwise", 64),
    (192, 1024, "groupwise", 128),
    (130, 264, "groupwise", 8),
    (40, 2048, "groupwise", 32),
    (96, 768, "rowwise", 0),
    (64, 512, "global", 0),
])
def test_quantize_pack_bit_exact(cuda_device, zero, meta, N, K, mode, g):
    w4 = lib()
    seed = synth.config_seed("variant-q", N, K, mode, g, zero, meta)
    W = variant_weights(N, K, mode, g, seed)
    p_ref, s_ref, z_ref = oracle.quantize_pack(W, mode, g, zero=zero, meta=meta)
    P, S, Z = w4.w4_quantize_pack(to_dev_bf16(W, cuda_device), mode, g, zero=zero, meta=meta)
    assert (P.cpu().numpy().view(np.uint32) == p_ref).all()
    assert (from_dev_bits(S) == s_ref).all()
    assert (from_dev_bits(Z) == z_ref).all()
    if zero == "float" and mode != "global":
        zv = synth.bf16_bits_to_f32(z_ref) if meta == "bf16" else z_ref.view(np.float16).astype(np.float32)
        assert (zv < 0).any() or (zv > 15).any()     # zero points outside the code range occur


MATMUL_CASES = [
    # M, N, K, mode, g, transposed            path taken
    (1, 512, 2048, "groupwise", 128, False),  # int8 forward GEMV
    (3, 512, 2048, "groupwise", 128, False),  # int8 forward GEMV, two digit sets
    (2, 256, 1024, "rowwise", 0, False),      # int8 forward GEMV, one group per row
    (1, 512, 1024, "global", 0, False),       # int8 forward GEMV, one scale
    (4, 384, 1024, "groupwise", 64, False),   # bf16 forward GEMV
    (2, 512, 2048, "groupwise", 128, True),   # transposed GEMV
    (4, 256, 1024, "groupwise", 64, True),    # transposed GEMV
    (3, 200, 520, "groupwise", 8, False),     # CUDA-core forward GEMV
    (2, 200, 520, "groupwise", 8, True),      # CUDA-core transposed GEMV
    (64, 512, 1024, "groupwise", 64, False),  # tcgen05 GEMM
    (130, 384, 512, "groupwise", 128, True),  # tcgen05 GEMM, transposed
    (17, 300, 520, "groupwise", 8, False),    # CUDA-core GEMM
]


@pytest.mark.gpu
@pytest.mark.parametrize("zero,meta", VARIANTS)
@pytest.mark.parametrize("M,N,K,mode,g,transposed", MATMUL_CASES)
def test_matmul_parity(cuda_device, zero, meta, M, N, K, mode, g, transposed):
    w4 = lib()
    dev = cuda_device
    seed = synth.config_seed("variant-mm", M, N, K, mode, g, transposed, zero, meta)
    W = variant_weights(N, K, mode, g, seed, shifted_row=M <= 4)
    p, s, z = oracle.quantize_pack(W, mode, g, zero=zero, meta=meta)
    A = synth.grads(M, N, seed) if transposed else synth.activations(M, K, seed)
    b = synth.bias(K if transposed else N, seed)
    fn = oracle.linear_t if transposed else oracle.linear
    ref, _ = fn(A, p, s, z, mode, g, N, K, bias=b, meta=meta)
    y = w4.w4a16_gemm(to_dev_bf16(A, dev), to_dev_packed(p, dev), to_dev_meta(s, meta, dev),
                      to_dev_meta(z, meta, dev), mode, g, N=N, K=K, bias=to_dev_bf16(b, dev),
                      transposed=transposed, zero=zero)
    assert_close(from_dev_bits(y), ref, f"{zero}/{meta} M={M} N={N} K={K} {mode} g={g} t={transposed}")
    assert w4.w4_device_error() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("meta", ["fp16", "bf16"])
@pytest.mark.parametrize("M", [1, 4])
def test_float_zero_gemv_wide_range_activations(cuda_device, meta, M):
    """Granules whose activations span more than 15 binades take the forward GEMV's
    bf16 path; with a fractional zero point it rounds q - z once."""
    w4 = lib()
    dev = cuda_device
    N, K, g = 256, 2048, 128
    seed = synth.config_seed("variant-wide", M, meta)
    W = variant_weights(N, K, "groupwise", g, seed)
    p, s, z = oracle.quantize_pack(W, "groupwise", g, zero="float", meta=meta)
    X, _ = synth.mixed_range_activations(M, K, seed, lo_exp=-24, hi_exp=6)
    ref, _ = oracle.linear(X, p, s, z, "groupwise", g, N, K, meta=meta)
    y = w4.w4a16_gemv(to_dev_bf16(X, dev), to_dev_packed(p, dev), to_dev_meta(s, meta, dev),
                      to_dev_meta(z, meta, dev), "groupwise", g, N=N, K=K, zero="float")
    assert_close(from_dev_bits(y), ref, f"wide-range float-zero M={M} {meta}")


@pytest.mark.gpu
def test_unknown_format_flag_rejected(cuda_device):
    import ctypes
    import torch
    w4 = lib()
    W = torch.zeros((8, 64), dtype=torch.bfloat16, device=cuda_device)
    P = torch.empty((8, 8), dtype=torch.int32, device=cuda_device)
    S = torch.empty((8, 1), dtype=torch.float16, device=cuda_device)
    st = w4.library().w4_quantize_pack(W.data_ptr(), 8, 64, 2 | 0x40, 64, P.data_ptr(), S.data_ptr(),
                                       S.data_ptr(), None, 0, None)
    assert st == 1
