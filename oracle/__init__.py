"""CPU oracle for the W4A16 weight-only matmul -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The library in
``gemv_w4a16_groupwise_b200`` never does, and the two share no code: this
package wraps ``w4a16_oracle.c`` (plain C, compiled with gcc) through ctypes
and exchanges numpy arrays.  bf16 and fp16 values are numpy ``uint16`` bit
patterns.

Functions, in the order the method applies them (each follows the page and
section named in its docstring):

* :func:`quantize`  -- bf16 W -> uint4 codes, fp16 scales and zeros (or, with
  ``zero="float"`` / ``meta="bf16"``, a fractional zero point / bf16 scales and
  zeros: the HQQ-style variant)
* :func:`pack` / :func:`unpack` -- eight codes per uint32 along K
* :func:`dequant`   -- w_hat = (q - z) * s in fp64
* :func:`linear`    -- Y = X @ w_hat^T (+ bias), fp64 accumulation
* :func:`linear_t`  -- dX = dY @ w_hat (+ bias), the transposed mode

Parity status: every function is pinned by tests in ``tests/test_oracle.py``
(brute force, exact round trips, closed forms, invariants, hand-derived
golden values).  The quantization-error statistics of the
llm-quantization page's mode table are a soft band only.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

MODE_GLOBAL = 0
MODE_ROWWISE = 1
MODE_GROUPWISE = 2
MODES = {"global": MODE_GLOBAL, "rowwise": MODE_ROWWISE, "groupwise": MODE_GROUPWISE}
# format flags or-ed into the mode (see w4a16_oracle.c)
FLAG_FLOAT_ZERO = 0x10
FLAG_META_BF16 = 0x20

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "w4a16_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FP contraction)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            L = ctypes.c_long
            I = ctypes.c_int
            lib.oracle_quantize.argtypes = [P, L, L, I, L, P, P, P]
            lib.oracle_quantize.restype = I
            lib.oracle_pack.argtypes = [P, L, L, P]
            lib.oracle_unpack.argtypes = [P, L, L, P]
            lib.oracle_dequant.argtypes = [P, P, P, L, L, I, L, P]
            lib.oracle_linear.argtypes = [P, L, L, P, P, P, L, I, L, P, P, L, P, P]
            lib.oracle_linear_t.argtypes = [P, L, L, P, P, P, L, I, L, P, P, L, P, P]
            lib.oracle_groups_per_row.argtypes = [L, I, L]
            lib.oracle_groups_per_row.restype = L
            lib.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
            lib.oracle_f64_to_bf16.restype = ctypes.c_uint16
            lib.oracle_num_threads.argtypes = []
            lib.oracle_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _mode(mode, zero: str = "int", meta: str = "fp16"):
    m = MODES[mode] if isinstance(mode, str) else int(mode)
    if zero not in ("int", "float") or meta not in ("fp16", "bf16"):
        raise ValueError(f"zero must be 'int' or 'float' and meta 'fp16' or 'bf16', got {zero!r}, {meta!r}")
    return m | (FLAG_FLOAT_ZERO if zero == "float" else 0) | (FLAG_META_BF16 if meta == "bf16" else 0)


def groups_per_row(K: int, mode, g: int) -> int:
    return int(_load().oracle_groups_per_row(K, _mode(mode), g))


def meta_shape(N: int, K: int, mode, g: int):
    """Shape of the scale / zero arrays: [N,G], [N,1] or [1,1]."""
    m = _mode(mode) & 0x0F
    if m == MODE_GLOBAL:
        return (1, 1)
    if m == MODE_ROWWISE:
        return (N, 1)
    if g <= 0 or K % g:
        raise ValueError(f"group size {g} must be positive and divide K={K}")
    return (N, K // g)


def num_threads() -> int:
    """OpenMP threads the oracle's parallel loops use."""
    return int(_load().oracle_num_threads())


def f64_to_bf16(x: float) -> int:
    """Round one double to bf16 bits, ties to even."""
    return int(_load().oracle_f64_to_bf16(float(x)))


def quantize(W_bf16: np.ndarray, mode, g: int = 0, zero: str = "int", meta: str = "fp16"):
    """Quantize bf16 W [N,K] -> (codes uint8 [N,K], s bits, z bits).

    Asymmetric min-max to uint4 per group (llm-quantization, Objective 1:
    GLOBAL / ROWWISE / GROUPWISE modes), integer zero point, fp16 s and z.
    ``zero="float"``: fractional zero point z = -min / s and
    q = clamp(rint(w / s + z), 0, 15) (the HQQ-style quantizer of "Re-write
    HQQ Fused Gemm Transpose"); ``meta="bf16"``: s and z stored as bf16.
    """
    W = _c(W_bf16, np.uint16)
    N, K = W.shape
    shape = meta_shape(N, K, mode, g)
    q = np.empty((N, K), np.uint8)
    s = np.empty(shape, np.uint16)
    z = np.empty(shape, np.uint16)
    rc = _load().oracle_quantize(_ptr(W), N, K, _mode(mode, zero, meta), int(g), _ptr(q), _ptr(s), _ptr(z))
    if rc != 0:
        raise ValueError(f"oracle_quantize: bad arguments N={N} K={K} mode={mode} g={g}")
    return q, s, z


def pack(q: np.ndarray) -> np.ndarray:
    """Codes uint8 [N,K] -> uint32 [N,K/8]; code i of word j at bits 4i..4i+3."""
    q = _c(q, np.uint8)
    N, K = q.shape
    if K % 8:
        raise ValueError("K must be a multiple of 8")
    out = np.empty((N, K // 8), np.uint32)
    _load().oracle_pack(_ptr(q), N, K, _ptr(out))
    return out


def unpack(packed: np.ndarray, K: int) -> np.ndarray:
    p = _c(packed, np.uint32)
    N = p.shape[0]
    out = np.empty((N, K), np.uint8)
    _load().oracle_unpack(_ptr(p), N, K, _ptr(out))
    return out


def dequant(packed, s, z, mode, g: int, K: int, meta: str = "fp16") -> np.ndarray:
    """w_hat [N,K] fp64 = (q - z) * s (s, z read as fp16, or bf16 with meta="bf16")."""
    p = _c(packed, np.uint32)
    N = p.shape[0]
    out = np.empty((N, K), np.float64)
    _load().oracle_dequant(_ptr(p), _ptr(_c(s, np.uint16)), _ptr(_c(z, np.uint16)), N, K,
                           _mode(mode, "int", meta), int(g), _ptr(out))
    return out


def linear(X_bf16, packed, s, z, mode, g: int, N: int, K: int, bias=None, cols=None, meta: str = "fp16"):
    """Y = X @ w_hat^T (+ bias), fp64 accumulation -> (y64, y_bf16_bits).

    With ``cols`` (output column indices n) only those columns are computed.
    """
    X = _c(X_bf16, np.uint16)
    M = X.shape[0]
    assert X.shape[1] == K
    c = None if cols is None else _c(cols, np.int64)
    nc = N if c is None else c.shape[0]
    y64 = np.empty((M, nc), np.float64)
    ybf = np.empty((M, nc), np.uint16)
    b = None if bias is None else _c(bias, np.uint16)
    _load().oracle_linear(_ptr(X), M, K, _ptr(_c(packed, np.uint32)), _ptr(_c(s, np.uint16)),
                          _ptr(_c(z, np.uint16)), N, _mode(mode, "int", meta), int(g), _ptr(b), _ptr(c), nc,
                          _ptr(y64), _ptr(ybf))
    return y64, ybf


def linear_t(dY_bf16, packed, s, z, mode, g: int, N: int, K: int, bias=None, cols=None, meta: str = "fp16"):
    """dX = dY @ w_hat (+ bias) from the same packed weights -> (x64, x_bf16_bits).

    With ``cols`` (output column indices k) only those columns are computed.
    """
    dY = _c(dY_bf16, np.uint16)
    M = dY.shape[0]
    assert dY.shape[1] == N
    c = None if cols is None else _c(cols, np.int64)
    nc = K if c is None else c.shape[0]
    y64 = np.empty((M, nc), np.float64)
    ybf = np.empty((M, nc), np.uint16)
    b = None if bias is None else _c(bias, np.uint16)
    _load().oracle_linear_t(_ptr(dY), M, N, _ptr(_c(packed, np.uint32)), _ptr(_c(s, np.uint16)),
                            _ptr(_c(z, np.uint16)), K, _mode(mode, "int", meta), int(g), _ptr(b), _ptr(c), nc,
                            _ptr(y64), _ptr(ybf))
    return y64, ybf


def quantize_pack(W_bf16, mode, g: int = 0, zero: str = "int", meta: str = "fp16"):
    """quantize then pack: -> (packed uint32 [N,K/8], s, z)."""
    q, s, z = quantize(W_bf16, mode, g, zero, meta)
    return pack(q), s, z
