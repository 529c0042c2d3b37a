"""The allocation-free forward GEMV (w4a16_gemv_noalloc) against w4a16_gemv.

Collected last on purpose.  Some callers cannot allocate device memory (an
engine that owns all GPU memory through its own pool, a plugin given only
its inputs and outputs); this entry point serves them from the library's
built-in 8 MiB scratch.  The test calls it through the C ABI twice in a row
on problems that need split-K scratch and compares each output with the
regular entry point, which takes a caller workspace.
"""
import ctypes

import numpy as np
import pytest

from gemv_w4a16_groupwise_b200 import synth

from gpu_helpers import assert_close, from_dev_bits, quantized_case, to_dev_bf16, to_dev_f16, to_dev_packed

pytestmark = pytest.mark.gpu


def _lib():
    import gemv_w4a16_groupwise_b200 as w4
    lib = w4.library()
    f = lib.w4a16_gemv_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, I, I, I, P, P, P, I, I, P, P, P]
    f.restype = I
    return w4, lib


def _case(M, N, K, mode, g, seed, dev):
    W, p, s, z = quantized_case(N, K, mode, g, seed)
    X = synth.activations(M, K, seed)
    b = synth.bias(N, seed)
    return (to_dev_bf16(X, dev), to_dev_packed(p, dev), to_dev_f16(s, dev), to_dev_f16(z, dev),
            to_dev_bf16(b, dev))


def test_noalloc_matches_workspace_entry_point_twice(cuda_device):
    import torch
    w4, lib = _lib()
    dev = cuda_device
    cases = [(4, 4096, 16384, "groupwise", 128, 1), (3, 2048, 8192, "rowwise", 0, 2)]
    for M, N, K, mode, g, seed in cases:
        assert w4.w4_workspace_bytes(M, N, K, False) > 0   # the scratch is really used
    outs = []
    stream = torch.cuda.current_stream(dev).cuda_stream
    for M, N, K, mode, g, seed in cases:          # two calls in a row on the shared scratch
        X, P, S, Z, B = _case(M, N, K, mode, g, seed, dev)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        st = lib.w4a16_gemv_noalloc(X.data_ptr(), M, N, K, P.data_ptr(), S.data_ptr(),
                                    Z.data_ptr(), w4.MODES[mode], g, B.data_ptr(), Y.data_ptr(),
                                    stream)
        assert st == 0, lib.w4_status_string(st)
        outs.append((Y, X, P, S, Z, B, M, N, K, mode, g))
    torch.cuda.synchronize()
    for Y, X, P, S, Z, B, M, N, K, mode, g in outs:
        ref = w4.w4a16_gemv(X, P, S, Z, mode, g, N=N, K=K, bias=B)
        ref64 = synth.bf16_bits_to_f32(from_dev_bits(ref)).astype(np.float64)
        assert_close(from_dev_bits(Y), ref64, f"noalloc M={M} N={N} K={K}")
    assert w4.w4_device_error() == 0


def test_noalloc_rejects_problems_beyond_the_scratch(cuda_device):
    w4, lib = _lib()
    M, N, K = 4, 1 << 20, 65536      # K split into slices: fp32 partials of 4 x M x N
    need = w4.w4_workspace_bytes(M, N, K, False)
    assert need > (8 << 20)
    fake = 1 << 20          # never dereferenced: the size check comes before any launch
    st = lib.w4a16_gemv_noalloc(fake, M, N, K, fake, fake, fake, 2, 128, None, fake, None)
    assert st == 4
    assert lib.w4a16_gemv_noalloc(fake, 5, 64, 256, fake, fake, fake, 2, 64, None, fake, None) == 1
