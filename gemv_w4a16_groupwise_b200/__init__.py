"""B200-native W4A16 weight-only matmul: thin Python binding of ``libw4a16.so``.

Every step of the computation runs in the library's sm_100a kernels; this
module only checks tensor metadata, passes device pointers and the current
CUDA stream, and turns status codes into exceptions.  PyTorch provides
device memory and streams.  There is no CPU fallback: without a CUDA device
or without the built library every call raises.

Entry points (same names as the C ABI in ``include/w4a16.h``):

* :func:`w4_quantize_pack` -- bf16 W [N, K] -> packed int4 (int32 [N, K/8]),
  fp16 scales and zeros (``zero="float"``: fractional zero point;
  ``meta="bf16"``: bf16 scales and zeros)
* :func:`w4a16_gemm` -- Y = X . dequant(W)^T (or dX = dY . dequant(W) with
  ``transposed=True``), optional bias
* :func:`w4a16_gemv` -- the same for M <= 4 (TMA-streamed weights, exact
  products on the tensor pipe, fp32 sums)
* :func:`w4_gather_columns` / :func:`w4_scatter_columns` -- the column
  permutations of act-order weights (``perm=`` on the calls above)
* :func:`w4_workspace_bytes`, :func:`w4_device_error`

:mod:`gemv_w4a16_groupwise_b200.tp` shards one layer over torch.distributed
ranks (column-parallel over N, row-parallel over K) on top of these calls.

``packed`` may also be given as its two-per-byte view, uint8 [N, K/2] (the
same bytes; the even k in the low nibble).
"""
from __future__ import annotations

import ctypes
import os
import threading

from . import build as _build

W4_MODE_GLOBAL = 0
W4_MODE_ROWWISE = 1
W4_MODE_GROUPWISE = 2
MODES = {"global": W4_MODE_GLOBAL, "rowwise": W4_MODE_ROWWISE, "groupwise": W4_MODE_GROUPWISE}
W4_ZERO_FLOAT = 0x10
W4_META_BF16 = 0x20

_lock = threading.Lock()
_lib = None


class W4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = f"{what}: {library().w4_status_string(status).decode()}"
        if status == 5:
            msg += f" ({library().w4_last_cuda_error().decode()})"
        super().__init__(msg)


def library_path() -> str:
    return _build.LIB


def library():
    """Load (building first if needed) the in-tree CUDA library."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            lib = ctypes.CDLL(path)
            P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
            lib.w4_status_string.argtypes = [I]
            lib.w4_status_string.restype = ctypes.c_char_p
            lib.w4_quantize_workspace_bytes.argtypes = [I, I, I]
            lib.w4_quantize_workspace_bytes.restype = Z
            lib.w4_quantize_pack.argtypes = [P, I, I, I, I, P, P, P, P, Z, P]
            lib.w4_quantize_pack.restype = I
            lib.w4_workspace_bytes.argtypes = [I, I, I, I]
            lib.w4_workspace_bytes.restype = Z
            for name in ("w4a16_gemm", "w4a16_gemv"):
                f = getattr(lib, name)
                f.argtypes = [P, I, I, I, P, P, P, I, I, P, I, P, P, Z, P]
                f.restype = I
            lib.w4_device_error.argtypes = [ctypes.POINTER(I)]
            lib.w4_device_error.restype = I
            lib.w4_last_cuda_error.argtypes = []
            lib.w4_last_cuda_error.restype = ctypes.c_char_p
            lib.w4_launch_count.argtypes = []
            lib.w4_launch_count.restype = ctypes.c_uint64
            lib.w4_set_debug_checks.argtypes = [I]
            lib.w4_set_debug_checks.restype = I
            lib.w4_debug_set_wait_limit.argtypes = [ctypes.c_ulonglong]
            lib.w4_debug_set_wait_limit.restype = I
            lib.w4_debug_withhold_stage.argtypes = [I]
            lib.w4_debug_withhold_stage.restype = I
            lib.w4_gather_columns.argtypes = [P, I, I, P, I, P, P]
            lib.w4_gather_columns.restype = I
            lib.w4_scatter_columns.argtypes = [P, I, I, P, I, P, P]
            lib.w4_scatter_columns.restype = I
            lib.w4_invert_permutation.argtypes = [P, I, P, P]
            lib.w4_invert_permutation.restype = I
            _lib = lib
    return _lib


def _torch():
    import torch
    return torch


def _mode(mode, zero: str = "int", meta: str = "fp16") -> int:
    """The C mode argument: base mode or-ed with the format flags."""
    m = MODES[mode] if isinstance(mode, str) else int(mode)
    if zero not in ("int", "float") or meta not in ("fp16", "bf16"):
        raise ValueError(f"zero must be 'int' or 'float' and meta 'fp16' or 'bf16', got {zero!r}, {meta!r}")
    return m | (W4_ZERO_FLOAT if zero == "float" else 0) | (W4_META_BF16 if meta == "bf16" else 0)


def _meta_dtype(meta: str):
    torch = _torch()
    return torch.bfloat16 if meta == "bf16" else torch.float16


def _check_cuda(t, name, dtype, shape=None):
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must live on a CUDA device (no CPU path exists)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _packed_words(packed, N: int, K: int):
    """The packed codes as int32 [N, K/8]; a uint8 [N, K/2] two-per-byte view is
    reinterpreted (same bytes), anything else is passed on for the checks."""
    torch = _torch()
    if isinstance(packed, torch.Tensor) and packed.dtype == torch.uint8:
        if tuple(packed.shape) != (N, K // 2) or not packed.is_contiguous():
            raise ValueError(f"uint8 packed codes must be contiguous [{N}, {K // 2}]")
        return packed.view(torch.int32)
    return packed


def _check_perm(perm, K: int, dev):
    torch = _torch()
    _check_cuda(perm, "perm", torch.int32, (K,))
    if perm.device != dev:
        raise ValueError("perm must be on the activations' device")


def _device_index(device) -> int:
    torch = _torch()
    if isinstance(device, int):
        return device
    return device.index if device.index is not None else torch.cuda.current_device()


def _stream_ptr(device):
    """The current stream of `device` as a raw handle.  PyTorch's own raw
    accessor (what its compiled kernels use) costs a tenth of building the
    Stream object; the public call is the fallback."""
    torch = _torch()
    idx = _device_index(device)
    raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
    if raw is not None:
        return ctypes.c_void_p(raw(idx))
    return ctypes.c_void_p(torch.cuda.current_stream(idx).cuda_stream)


class _OnDevice:
    """Make `idx` the current device for a library call and restore the
    previous one, switching only when they differ (the library launches on
    the current device)."""

    __slots__ = ("idx", "prev", "_get", "_set")

    def __init__(self, device):
        torch = _torch()
        self.idx = _device_index(device)
        self._get = getattr(torch._C, "_cuda_getDevice", None)
        self._set = getattr(torch._C, "_cuda_setDevice", None)
        self.prev = None

    def __enter__(self):
        if self._get is None or self._set is None:
            self.prev = _torch().cuda.device(self.idx)
            self.prev.__enter__()
            return self
        self.prev = self._get()
        if self.prev != self.idx:
            self._set(self.idx)
        return self

    def __exit__(self, *exc):
        if self._get is None or self._set is None:
            return self.prev.__exit__(*exc)
        if self.prev != self.idx:
            self._set(self.prev)
        return False


# w4_workspace_bytes by (device, M, N, K, transposed): a pure function of
# the shape and the device's SM count
_ws_cache: dict = {}


def meta_shape(N: int, K: int, mode, group_size: int):
    m = _mode(mode) & 0x0F
    if m == W4_MODE_GLOBAL:
        return (1, 1)
    if m == W4_MODE_ROWWISE:
        return (N, 1)
    if group_size <= 0 or K % group_size:
        raise ValueError(f"group_size {group_size} must divide K={K}")
    return (N, K // group_size)


def w4_quantize_workspace_bytes(N: int, K: int, mode) -> int:
    return int(library().w4_quantize_workspace_bytes(N, K, _mode(mode)))


def w4_workspace_bytes(M: int, N: int, K: int, transposed: bool = False) -> int:
    return int(library().w4_workspace_bytes(M, N, K, int(bool(transposed))))


def w4_quantize_pack(W, mode="groupwise", group_size: int = 128, out=None, zero: str = "int",
                     meta: str = "fp16", perm=None):
    """Quantize bf16 W [N, K] (CUDA) -> (packed int32 [N, K/8], scales, zeros).

    ``zero="float"`` keeps a fractional zero point (the HQQ-style quantizer);
    ``meta="bf16"`` stores scales and zeros as bf16 instead of fp16;
    ``perm`` (int32 [K], a permutation) quantizes W[:, perm] (act-order).
    """
    torch = _torch()
    _check_cuda(W, "W", torch.bfloat16)
    N, K = W.shape
    if perm is not None:
        _check_perm(perm, K, W.device)
        W = w4_gather_columns(W, perm)
    shape = meta_shape(N, K, mode, group_size)
    dev = W.device
    mdt = _meta_dtype(meta)
    if out is None:
        packed = torch.empty((N, K // 8), dtype=torch.int32, device=dev)
        scales = torch.empty(shape, dtype=mdt, device=dev)
        zeros = torch.empty(shape, dtype=mdt, device=dev)
    else:
        packed, scales, zeros = out
        _check_cuda(scales, "scales", mdt, shape)
        _check_cuda(zeros, "zeros", mdt, shape)
    nws = w4_quantize_workspace_bytes(N, K, mode)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        st = library().w4_quantize_pack(W.data_ptr(), N, K, _mode(mode, zero, meta), int(group_size),
                                        packed.data_ptr(), scales.data_ptr(), zeros.data_ptr(),
                                        ws.data_ptr(), nws, _stream_ptr(dev))
    if st != 0:
        raise W4Error(st, "w4_quantize_pack")
    return packed, scales, zeros


def _matmul(fname, A, packed, scales, zeros, mode, group_size, N, K, bias, transposed, out, zero,
            perm=None):
    torch = _torch()
    packed = _packed_words(packed, N, K)
    if perm is not None:
        # act-order: forward gathers X's columns; transposed scatters dX's
        _check_cuda(A, "A", torch.bfloat16)
        _check_perm(perm, K, A.device)
        if not transposed:
            return _matmul(fname, w4_gather_columns(A, perm), packed, scales, zeros, mode, group_size, N, K,
                           bias, False, out, zero)
        bias_p = None if bias is None else w4_gather_columns(bias.view(1, -1), perm).view(-1)
        part = _matmul(fname, A, packed, scales, zeros, mode, group_size, N, K, bias_p, True, None, zero)
        # dX[:, perm[j]] = part[:, j]: a gather by the inverse permutation
        return w4_gather_columns(part, w4_invert_permutation(perm), out=out)
    _check_cuda(A, "A", torch.bfloat16)
    _check_cuda(packed, "packed", torch.int32, (N, K // 8))
    # the metadata type follows the scales' dtype (fp16 or bf16)
    meta = "bf16" if isinstance(scales, torch.Tensor) and scales.dtype == torch.bfloat16 else "fp16"
    _check_cuda(scales, "scales", _meta_dtype(meta), meta_shape(N, K, mode, group_size))
    _check_cuda(zeros, "zeros", _meta_dtype(meta), meta_shape(N, K, mode, group_size))
    if A.dim() != 2:
        raise ValueError("A must be 2-D")
    M = A.shape[0]
    in_len, out_len = (N, K) if transposed else (K, N)
    if A.shape[1] != in_len:
        raise ValueError(f"A must have {in_len} columns, got {A.shape[1]}")
    if bias is not None:
        _check_cuda(bias, "bias", torch.bfloat16, (out_len,))
    dev = A.device
    if out is None:
        out = torch.empty((M, out_len), dtype=torch.bfloat16, device=dev)
    else:
        _check_cuda(out, "out", torch.bfloat16, (M, out_len))
    with _OnDevice(dev) as on:
        key = (on.idx, M, N, K, bool(transposed))
        nws = _ws_cache.get(key)
        if nws is None:
            nws = w4_workspace_bytes(M, N, K, transposed)
            if len(_ws_cache) > 4096:
                _ws_cache.clear()
            _ws_cache[key] = nws
        ws = torch.empty(nws, dtype=torch.uint8, device=dev) if nws else None
        st = getattr(library(), fname)(
            A.data_ptr(), M, N, K, packed.data_ptr(), scales.data_ptr(), zeros.data_ptr(),
            _mode(mode, zero, meta), int(group_size), None if bias is None else bias.data_ptr(),
            int(bool(transposed)), out.data_ptr(), None if ws is None else ws.data_ptr(), nws,
            _stream_ptr(on.idx))
    if st != 0:
        raise W4Error(st, fname)
    return out


def w4a16_gemm(A, packed, scales, zeros, mode="groupwise", group_size: int = 128, *, N: int,
               K: int, bias=None, transposed: bool = False, out=None, zero: str = "int", perm=None):
    """Y = A . dequant(W)^T  (A [M, K])  or, transposed, dX = A . dequant(W)  (A [M, N]).

    ``zero`` must name the quantizer's zero point ("int" or "float"); bf16 scales
    and zeros are recognised by their dtype; ``perm`` (int32 [K]) marks act-order
    weights whose packed column j is input channel perm[j]."""
    return _matmul("w4a16_gemm", A, packed, scales, zeros, mode, group_size, N, K, bias,
                   transposed, out, zero, perm)


def w4a16_gemv(A, packed, scales, zeros, mode="groupwise", group_size: int = 128, *, N: int,
               K: int, bias=None, transposed: bool = False, out=None, zero: str = "int", perm=None):
    """Small-batch (M <= 4) path of :func:`w4a16_gemm`: TMA-streamed weights, exact
    products on the tensor pipe with fp32 sums, forward and transposed."""
    return _matmul("w4a16_gemv", A, packed, scales, zeros, mode, group_size, N, K, bias,
                   transposed, out, zero, perm)


def w4_gather_columns(A, idx, out=None):
    """out[m, j] = A[m, idx[j]]: bf16 A [M, C] (CUDA), int32 idx [L] -> bf16 [M, L]."""
    torch = _torch()
    _check_cuda(A, "A", torch.bfloat16)
    _check_cuda(idx, "idx", torch.int32)
    if A.dim() != 2 or idx.dim() != 1:
        raise ValueError("A must be 2-D and idx 1-D")
    M, C = A.shape
    L = idx.shape[0]
    if out is None:
        out = torch.empty((M, L), dtype=torch.bfloat16, device=A.device)
    else:
        _check_cuda(out, "out", torch.bfloat16, (M, L))
    with torch.cuda.device(A.device):
        st = library().w4_gather_columns(A.data_ptr(), M, C, idx.data_ptr(), L, out.data_ptr(),
                                         _stream_ptr(A.device))
    if st != 0:
        raise W4Error(st, "w4_gather_columns")
    return out


def w4_invert_permutation(perm, out=None):
    """inv [n] with inv[perm[j]] = j (int32, CUDA; perm a permutation of [0, n))."""
    torch = _torch()
    _check_cuda(perm, "perm", torch.int32)
    n = perm.shape[0]
    inv = torch.empty_like(perm) if out is None else out
    with torch.cuda.device(perm.device):
        st = library().w4_invert_permutation(perm.data_ptr(), n, inv.data_ptr(), _stream_ptr(perm.device))
    if st != 0:
        raise W4Error(st, "w4_invert_permutation")
    return inv


def w4_scatter_columns(A, idx, dst_cols: int, out=None):
    """out[m, idx[j]] = A[m, j]: bf16 A [M, L], int32 idx [L] (no repeats) -> bf16
    [M, dst_cols] (a fresh tensor, zero where no index lands, unless `out` is given)."""
    torch = _torch()
    _check_cuda(A, "A", torch.bfloat16)
    _check_cuda(idx, "idx", torch.int32)
    M, L = A.shape
    if idx.shape != (L,):
        raise ValueError(f"idx must have shape ({L},)")
    if out is None:
        out = torch.zeros((M, dst_cols), dtype=torch.bfloat16, device=A.device)
    else:
        _check_cuda(out, "out", torch.bfloat16, (M, dst_cols))
    with torch.cuda.device(A.device):
        st = library().w4_scatter_columns(A.data_ptr(), M, L, idx.data_ptr(), dst_cols, out.data_ptr(),
                                          _stream_ptr(A.device))
    if st != 0:
        raise W4Error(st, "w4_scatter_columns")
    return out


def w4_launch_count() -> int:
    """Kernel launches issued by the library in this process (host counter)."""
    return int(library().w4_launch_count())


def w4_set_debug_checks(on: bool) -> None:
    """Debug mode: w4_quantize_pack rejects NaN / Inf weights (W4_ERR_INVALID_ARG)."""
    library().w4_set_debug_checks(1 if on else 0)


def w4_debug_set_wait_limit(ns: int) -> None:
    """Limit of a kernel's bounded waits on the current device (0 = the default 2 s)."""
    st = library().w4_debug_set_wait_limit(int(ns))
    if st != 0:
        raise W4Error(st, "w4_debug_set_wait_limit")


def w4_debug_withhold_stage(stage: int) -> None:
    """Failure injection: the GEMV producers skip stage `stage` (-1: none)."""
    st = library().w4_debug_withhold_stage(int(stage))
    if st != 0:
        raise W4Error(st, "w4_debug_withhold_stage")


def w4_device_error() -> int:
    """Read and clear the device error word (synchronizes); 0 = no kernel gave up."""
    code = ctypes.c_int(0)
    st = library().w4_device_error(ctypes.byref(code))
    if st not in (0, 1, 6) or (st == 1 and code.value == 0):
        raise W4Error(st, "w4_device_error")
    return int(code.value)
