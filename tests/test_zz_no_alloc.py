"""The allocation-free forward GEMV (w4a16_gemv_noalloc) against w4a16_gemv
and the CPU oracle.

Collected last on purpose.  Some callers cannot allocate device memory (an
engine that owns all GPU memory through its own pool, a plugin given only
its inputs and outputs); this entry point serves them from the library's
built-in 8 MiB scratch.  The test calls it through the C ABI twice in a row
on problems whose plan splits K (so the scratch really holds the fp32
partials), checks that each output equals the regular entry point's bit for
bit (both run the same plan and kernels, only the workspace differs), and
that it meets the parity tolerance against the oracle.
"""
import ctypes

import pytest

import oracle
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
    ref, _ = oracle.linear(X, p, s, z, mode, g, N, K, bias=b)
    return (to_dev_bf16(X, dev), to_dev_packed(p, dev), to_dev_f16(s, dev), to_dev_f16(z, dev),
            to_dev_bf16(b, dev)), ref


def test_noalloc_matches_workspace_entry_point_twice(cuda_device):
    import torch
    w4, lib = _lib()
    dev = cuda_device
    # few rows and a long K: the plan splits K to give every SM work
    cases = [(4, 512, 16384, "groupwise", 128, 1), (3, 1024, 8192, "rowwise", 0, 2)]
    for M, N, K, mode, g, seed in cases:
        assert w4.w4_workspace_bytes(M, N, K, False) > 0   # the scratch is really used
    outs = []
    stream = torch.cuda.current_stream(dev).cuda_stream
    for M, N, K, mode, g, seed in cases:          # two calls in a row on the shared scratch
        (X, P, S, Z, B), ref64 = _case(M, N, K, mode, g, seed, dev)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        st = lib.w4a16_gemv_noalloc(X.data_ptr(), M, N, K, P.data_ptr(), S.data_ptr(),
                                    Z.data_ptr(), w4.MODES[mode], g, B.data_ptr(), Y.data_ptr(),
                                    stream)
        assert st == 0, lib.w4_status_string(st)
        outs.append((Y, X, P, S, Z, B, M, N, K, mode, g, ref64))
    torch.cuda.synchronize()
    for Y, X, P, S, Z, B, M, N, K, mode, g, ref64 in outs:
        same = w4.w4a16_gemv(X, P, S, Z, mode, g, N=N, K=K, bias=B)
        assert torch.equal(Y, same), f"noalloc M={M} N={N} K={K}: differs from w4a16_gemv"
        assert_close(from_dev_bits(Y), ref64, f"noalloc M={M} N={N} K={K} vs oracle")
    assert w4.w4_device_error() == 0


def test_noalloc_rejects_problems_beyond_the_scratch(cuda_device):
    w4, lib = _lib()
    # g = 64 with K = 65536 at M = 4: the activations of all of K do not fit
    # in shared memory, so K is split into slices with fp32 partials of
    # slices x M x N floats, far beyond the scratch
    M, N, K = 4, 1 << 20, 65536
    need = w4.w4_workspace_bytes(M, N, K, False)
    assert need > (8 << 20)
    fake = 1 << 20          # never dereferenced: the size check comes before any launch
    st = lib.w4a16_gemv_noalloc(fake, M, N, K, fake, fake, fake, 2, 64, None, fake, None)
    assert st == 4
    assert lib.w4a16_gemv_noalloc(fake, 5, 64, 256, fake, fake, fake, 2, 64, None, fake, None) == 1
