"""Act-order weights and the two-per-byte view on the GPU, against the oracle.

Act-order (the GPTQ variant the TensorRT-LLM page "Modify small-batched weight
only quantization" sets beside channel-wise and group-wise kernels): the packed
column j holds input channel perm[j], so the forward product is
X[:, perm] . w_hat^T and the transposed one lands in dX[:, perm].  The oracle
reference is the plain product on the permuted operands.  The byte view is the
packed words' own bytes (two codes per byte, even k in the low nibble)."""
import numpy as np
import pytest

import oracle
from gemv_w4a16_groupwise_b200 import synth
from gpu_helpers import assert_close, from_dev_bits, to_dev_bf16


def lib():
    import gemv_w4a16_groupwise_b200 as w4
    return w4


def _perm(K, seed):
    return np.random.default_rng([seed, 31]).permutation(K).astype(np.int32)


@pytest.mark.gpu
@pytest.mark.parametrize("M,L,C", [(1, 7, 9), (4, 512, 512), (33, 1000, 1024), (2048, 4096, 4096)])
def test_gather_scatter_bit_exact(cuda_device, M, L, C):
    import torch
    w4 = lib()
    rng = np.random.default_rng([M, L, C])
    A = synth.normal_bf16((M, C), 0.0, 1.0, seed=M + L, stream=1)
    idx = rng.choice(C, size=L, replace=False).astype(np.int32)
    g = w4.w4_gather_columns(to_dev_bf16(A, cuda_device), torch.from_numpy(idx).to(cuda_device))
    assert (from_dev_bits(g) == A[:, idx]).all()
    B = synth.normal_bf16((M, L), 0.0, 1.0, seed=M + L + 1, stream=1)
    s = w4.w4_scatter_columns(to_dev_bf16(B, cuda_device), torch.from_numpy(idx).to(cuda_device), C)
    ref = np.zeros((M, C), np.uint16)
    ref[:, idx] = B
    assert (from_dev_bits(s) == ref).all()
    assert w4.w4_device_error() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("n", [1, 777, 4096, 28672])
def test_invert_permutation(cuda_device, n):
    import torch
    w4 = lib()
    perm = _perm(n, n)
    inv = w4.w4_invert_permutation(torch.from_numpy(perm).to(cuda_device)).cpu().numpy()
    assert (inv[perm] == np.arange(n)).all()
    assert w4.w4_device_error() == 0


@pytest.mark.gpu
def test_out_of_range_index_is_reported_not_read(cuda_device):
    import torch
    w4 = lib()
    A = synth.normal_bf16((3, 16), 0.0, 1.0, seed=2, stream=1)
    idx = np.array([0, 5, 16, 3, -1], np.int32)           # 16 and -1 are outside [0, 16)
    g = w4.w4_gather_columns(to_dev_bf16(A, cuda_device), torch.from_numpy(idx).to(cuda_device))
    out = from_dev_bits(g)
    assert (out[:, [0, 1, 3]] == A[:, [0, 5, 3]]).all() and (out[:, [2, 4]] == 0).all()
    assert w4.w4_device_error() == 5
    assert w4.w4_device_error() == 0                     # read and cleared


CASES = [
    # M, N, K, mode, g, zero
    (1, 512, 2048, "groupwise", 128, "int"),      # int8 GEMV
    (4, 384, 1024, "groupwise", 64, "float"),     # bf16 GEMV, fractional zero
    (3, 256, 1024, "rowwise", 0, "int"),
    (64, 512, 1024, "groupwise", 64, "int"),      # tcgen05 GEMM
    (130, 256, 512, "groupwise", 128, "float"),
]


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K,mode,g,zero", CASES)
def test_act_order_matches_oracle(cuda_device, M, N, K, mode, g, zero):
    import torch
    w4 = lib()
    dev = cuda_device
    seed = synth.config_seed("act-order", M, N, K, mode, g, zero)
    W = synth.weights(N, K, seed)
    perm = _perm(K, seed)
    tp = torch.from_numpy(perm).to(dev)
    # quantizing with perm = quantizing W[:, perm]
    p_ref, s_ref, z_ref = oracle.quantize_pack(W[:, perm], mode, g, zero=zero)
    P, S, Z = w4.w4_quantize_pack(to_dev_bf16(W, dev), mode, g, zero=zero, perm=tp)
    assert (P.cpu().numpy().view(np.uint32) == p_ref).all()
    assert (from_dev_bits(S) == s_ref).all() and (from_dev_bits(Z) == z_ref).all()
    X = synth.activations(M, K, seed)
    bN = synth.bias(N, seed)
    ref, _ = oracle.linear(X[:, perm], p_ref, s_ref, z_ref, mode, g, N, K, bias=bN)
    y = w4.w4a16_gemm(to_dev_bf16(X, dev), P, S, Z, mode, g, N=N, K=K, bias=to_dev_bf16(bN, dev),
                      zero=zero, perm=tp)
    assert_close(from_dev_bits(y), ref, f"act-order forward M={M} {mode} g={g} {zero}")
    dY = synth.grads(M, N, seed)
    bK = synth.bias(K, seed + 1)
    ref_p, _ = oracle.linear_t(dY, p_ref, s_ref, z_ref, mode, g, N, K, bias=bK[perm])
    ref_t = np.empty_like(ref_p)
    ref_t[:, perm] = ref_p
    x = w4.w4a16_gemm(to_dev_bf16(dY, dev), P, S, Z, mode, g, N=N, K=K, bias=to_dev_bf16(bK, dev),
                      transposed=True, zero=zero, perm=tp)
    assert_close(from_dev_bits(x), ref_t, f"act-order transposed M={M} {mode} g={g} {zero}")
    assert w4.w4_device_error() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("M", [2, 64])
def test_two_per_byte_view_gives_identical_results(cuda_device, M):
    import torch
    w4 = lib()
    dev = cuda_device
    N, K, g = 256, 1024, 128
    W = synth.weights(N, K, 11)
    P, S, Z = w4.w4_quantize_pack(to_dev_bf16(W, dev), "groupwise", g)
    P8 = P.view(torch.uint8)                              # [N, K / 2], two codes per byte
    q = oracle.unpack(P.cpu().numpy().view(np.uint32), K)
    b = P8.cpu().numpy()
    assert (b == (q[:, 0::2] | (q[:, 1::2] << 4))).all()  # even k in the low nibble
    X = to_dev_bf16(synth.activations(M, K, 11), dev)
    y32 = w4.w4a16_gemm(X, P, S, Z, "groupwise", g, N=N, K=K)
    y8 = w4.w4a16_gemm(X, P8, S, Z, "groupwise", g, N=N, K=K)
    assert torch.equal(y32, y8)
