"""Shared helpers of the GPU parity tests (not a test module)."""
import numpy as np

import oracle
from gemv_w4a16_groupwise_b200 import synth

MODE_ARG = {"groupwise": "groupwise", "rowwise": "rowwise", "global": "global"}


def to_dev_bf16(bits, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


def to_dev_f16(bits, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.float16).to(dev)


def to_dev_packed(p, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(p).view(np.int32)).to(dev)


def from_dev_bits(t):
    import torch
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def assert_close(y_bits, y_ref64, what=""):
    """The parity tolerance: |y - y_ref| <= 1e-2 rms(y_ref) + 2^-7 |y_ref| per element."""
    y = bf16_to_f64(y_bits)
    ref = np.asarray(y_ref64, dtype=np.float64)
    assert y.shape == ref.shape, (y.shape, ref.shape)
    assert np.isfinite(y).all(), f"{what}: non-finite output"
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    err = np.abs(y - ref)
    bound = 1e-2 * rms + 2.0 ** -7 * np.abs(ref)
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; rms={rms:.4g}; "
            f"first {idx.tolist()} got {y[tuple(idx[0])]:.6g} want {ref[tuple(idx[0])]:.6g}; "
            f"max err/bound {float((err / np.maximum(bound, 1e-30)).max()):.3f}")
    return float((err / np.maximum(bound, 1e-30)).max())


def quantized_case(N, K, mode, g, seed, structure=False):
    W = synth.weights(N, K, seed)
    if structure:
        W = synth.plant_structure(W, g if mode == "groupwise" else K, seed)
    p, s, z = oracle.quantize_pack(W, mode, g)
    return W, p, s, z
