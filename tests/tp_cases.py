"""Shared body of the tensor-parallel tests (not a test module): each rank of a
two-rank gloo group shards one layer, runs the column- and row-parallel
products and their transposed forms, and rank 0 checks them against the
oracle's unsharded results.  ``device`` selects where the local products run:
"cpu" drives the sharding and collective logic with the oracle as the local
product, "cuda" runs the library's kernels."""
import os
import sys

import numpy as np

CASES = [
    # N, K, mode, g, zero, meta
    (96, 512, "groupwise", 64, "int", "fp16"),
    (80, 768, "groupwise", 128, "float", "bf16"),
    (64, 256, "rowwise", 0, "int", "fp16"),
    (72, 384, "global", 0, "float", "fp16"),
]


def _bits_to_torch(bits, dtype):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dtype)


def _torch_to_bits(t):
    import torch
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_matmul(A, packed, scales, zeros, mode, g, *, N, K, bias=None, transposed=False, zero="int"):
    """The oracle with the library's matmul signature (CPU torch tensors in and out)."""
    import torch
    import oracle
    meta = "bf16" if scales.dtype == torch.bfloat16 else "fp16"
    p = packed.contiguous().numpy().view(np.uint32)
    s, z = _torch_to_bits(scales), _torch_to_bits(zeros)
    b = None if bias is None else _torch_to_bits(bias)
    fn = oracle.linear_t if transposed else oracle.linear
    _, ybf = fn(_torch_to_bits(A), p, s, z, mode, g, N, K, bias=b, meta=meta)
    return _bits_to_torch(ybf, torch.bfloat16)


def run_rank(rank, world, port, device, q):
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    import torch
    import torch.distributed as dist
    import oracle
    from gemv_w4a16_groupwise_b200 import synth, tp
    from gpu_helpers import assert_close
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    results = []
    try:
        dev = torch.device("cuda", 0) if device == "cuda" else torch.device("cpu")
        matmul = None if device == "cuda" else oracle_matmul
        for (N, K, mode, g, zero, meta) in CASES:
            seed = synth.config_seed("tp", N, K, mode, g, zero, meta)
            W = synth.weights(N, K, seed)
            p, s, z = oracle.quantize_pack(W, mode, g, zero=zero, meta=meta)
            mdt = torch.bfloat16 if meta == "bf16" else torch.float16
            P = torch.from_numpy(p.view(np.int32)).to(dev)
            S, Z = _bits_to_torch(s, mdt).to(dev), _bits_to_torch(z, mdt).to(dev)
            M = 3
            X = synth.activations(M, K, seed)
            dY = synth.grads(M, N, seed)
            bN, bK = synth.bias(N, seed), synth.bias(K, seed + 1)
            Xd, dYd = _bits_to_torch(X, torch.bfloat16).to(dev), _bits_to_torch(dY, torch.bfloat16).to(dev)
            bNd, bKd = _bits_to_torch(bN, torch.bfloat16).to(dev), _bits_to_torch(bK, torch.bfloat16).to(dev)
            col = tp.ColumnParallelW4A16(P, S, Z, mode, g, N, K, bias=bNd, zero=zero, matmul=matmul)
            row = tp.RowParallelW4A16(P, S, Z, mode, g, N, K, bias=bNd, zero=zero, matmul=matmul)
            y_col = col.forward(Xd)
            y_col_local = col.forward(Xd, gather=False)
            dx_col = col.backward_input(dYd)
            y_row = row.forward(Xd)
            dx_row = row.backward_input(dYd)
            dx_row_local = row.backward_input(dYd, gather=False)
            if rank == 0:
                ref_y, _ = oracle.linear(X, p, s, z, mode, g, N, K, bias=bN, meta=meta)
                ref_dx, _ = oracle.linear_t(dY, p, s, z, mode, g, N, K, meta=meta)
                tag = f"{N}x{K} {mode} g={g} {zero}/{meta}"
                assert_close(_torch_to_bits(y_col), ref_y, "column forward " + tag)
                assert_close(_torch_to_bits(dx_col), ref_dx, "column transposed " + tag)
                assert_close(_torch_to_bits(y_row), ref_y, "row forward " + tag)
                assert_close(_torch_to_bits(dx_row), ref_dx, "row transposed " + tag)
                lo, hi = col.shard.lo, col.shard.hi
                assert tuple(y_col_local.shape) == (M, hi - lo)
                assert (_torch_to_bits(y_col_local) == _torch_to_bits(y_col)[:, lo:hi]).all()
                klo, khi = row.shard.lo, row.shard.hi
                assert tuple(dx_row_local.shape) == (M, khi - klo)
                assert (_torch_to_bits(dx_row_local) == _torch_to_bits(dx_row)[:, klo:khi]).all()
                results.append(tag)
        dist.barrier()
        q.put((rank, "ok", results))
    except BaseException as e:   # report to the parent, then leave the group
        q.put((rank, f"{type(e).__name__}: {e}", results))
    finally:
        dist.destroy_process_group()
