"""Failure detection on the GPU without a GPU fault, and the debug-mode input check.

Every wait of the library's kernels is bounded.  These tests make one run
out on purpose: the wait limit is shortened to 1 ms and the GEMV producers
are told to skip one stage (its copy is never issued, so nothing is left in
flight).  The kernel must give up, report W4_ERR_TIMEOUT through
w4_device_error, and leave the context usable: the next normal call must
match the oracle.  The vLLM "Adding bias epilogue support for
cutlass_scaled_mm" thread (an opaque "Error Internal") is why failures come
back as distinct statuses.
"""
import numpy as np
import pytest

import oracle
from gemv_w4a16_groupwise_b200 import synth

from gpu_helpers import assert_close, from_dev_bits, quantized_case, to_dev_bf16, to_dev_f16, to_dev_packed

pytestmark = pytest.mark.gpu


def _lib():
    import gemv_w4a16_groupwise_b200 as w4
    return w4


@pytest.mark.parametrize("transposed", [False, True])
def test_bounded_wait_runs_out_and_the_context_recovers(cuda_device, transposed):
    import torch
    w4 = _lib()
    dev = cuda_device
    N, K, M, mode, g = 4096, 4096, 2, "groupwise", 128
    W, p, s, z = quantized_case(N, K, mode, g, 31)
    A = synth.activations(M, N if transposed else K, 31)
    args = (to_dev_bf16(A, dev), to_dev_packed(p, dev), to_dev_f16(s, dev), to_dev_f16(z, dev), mode, g)
    assert w4.w4_device_error() == 0
    try:
        w4.w4_debug_set_wait_limit(1_000_000)          # 1 ms
        w4.w4_debug_withhold_stage(1)                  # every CTA has at least two stages here
        w4.w4a16_gemv(*args, N=N, K=K, transposed=transposed)
        torch.cuda.synchronize()
        code = w4.w4_device_error()
    finally:
        w4.w4_debug_withhold_stage(-1)
        w4.w4_debug_set_wait_limit(0)
    assert code in (1, 3), code                        # a consumer (1) or the producer (3) gave up
    assert w4.w4_device_error() == 0                   # the word was cleared
    y = w4.w4a16_gemv(*args, N=N, K=K, transposed=transposed)
    if transposed:
        ref, _ = oracle.linear_t(A, p, s, z, mode, g, N, K)
    else:
        ref, _ = oracle.linear(A, p, s, z, mode, g, N, K)
    assert_close(from_dev_bits(y), ref, f"after a timeout, t={transposed}")
    assert w4.w4_device_error() == 0


def test_debug_checks_reject_nonfinite_weights(cuda_device):
    w4 = _lib()
    dev = cuda_device
    W = synth.weights(64, 256, 3)
    nan_w = W.copy()
    nan_w[5, 17] = 0x7FC0                              # a quiet NaN
    inf_w = W.copy()
    inf_w[63, 255] = 0xFF80                            # -Inf
    try:
        w4.w4_set_debug_checks(True)
        for bad in (nan_w, inf_w):
            with pytest.raises(w4.W4Error) as ei:
                w4.w4_quantize_pack(to_dev_bf16(bad, dev), "groupwise", 64)
            assert ei.value.status == 1
        p, s, z = w4.w4_quantize_pack(to_dev_bf16(W, dev), "groupwise", 64)   # finite: accepted
        p_ref, s_ref, z_ref = oracle.quantize_pack(W, "groupwise", 64)
        assert (p.cpu().numpy().view(np.uint32) == p_ref).all()
    finally:
        w4.w4_set_debug_checks(False)
    w4.w4_quantize_pack(to_dev_bf16(nan_w, dev), "groupwise", 64)   # release mode: no check
