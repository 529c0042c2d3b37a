"""Tensor-parallel sharding of one layer on two gloo ranks (CPU): the column-
(over N) and row-parallel (over K) forms of the forward and transposed products
equal the oracle's unsharded layer.  The local products are the oracle's, so
this covers the sharding and collective logic; tests/test_gpu_tp.py runs the
same cases with the library's kernels.  The pages have no parallelism; the
split along N is the one the fused-QKV page ("Add fused QKV HQQ triton_mm
test") uses to concatenate Q, K and V."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def run_two_ranks(device):
    import tp_cases
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=tp_cases.run_rank, args=(r, 2, port, device, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    for rank, status, _ in res:
        assert status == "ok", f"rank {rank}: {status}"
    for p in procs:
        assert p.exitcode == 0
    done = [r for r in res if r[0] == 0][0][2]
    assert len(done) == len(tp_cases.CASES)


def test_two_rank_column_and_row_parallel_match_oracle():
    run_two_ranks("cpu")


def test_split_ranges():
    from gemv_w4a16_groupwise_b200 import tp
    assert [tp.split_range(100, 3, r) for r in range(3)] == [(0, 33), (33, 66), (66, 100)]
    assert [tp.split_range(512, 2, r, 64) for r in range(2)] == [(0, 256), (256, 512)]
    assert [tp.split_range(384, 2, r, 128) for r in range(2)] == [(0, 128), (128, 384)]
    with pytest.raises(ValueError):
        tp.split_range(100, 2, 0, 64)            # not a whole number of groups
    with pytest.raises(ValueError):
        tp.split_range(128, 4, 0, 64)            # fewer groups than ranks


def test_shards_reassemble_the_layer():
    import numpy as np
    import torch
    import oracle
    from gemv_w4a16_groupwise_b200 import synth, tp
    N, K, g = 40, 256, 32
    W = synth.weights(N, K, 3)
    p, s, z = oracle.quantize_pack(W, "groupwise", g)
    P = torch.from_numpy(p.view(np.int32))
    S = torch.from_numpy(s.view(np.int16)).view(torch.float16)
    Z = torch.from_numpy(z.view(np.int16)).view(torch.float16)
    cols = [tp.shard_columns(P, S, Z, "groupwise", g, N, K, r, 3) for r in range(3)]
    assert torch.equal(torch.cat([c.packed for c in cols]), P)
    assert torch.equal(torch.cat([c.scales for c in cols]), S)
    rows = [tp.shard_rows(P, S, Z, "groupwise", g, N, K, r, 2) for r in range(2)]
    assert torch.equal(torch.cat([r.packed for r in rows], dim=1), P)
    assert torch.equal(torch.cat([r.zeros for r in rows], dim=1), Z)
    # the shards are self-contained layers: their dequantized weights tile the whole
    wh = oracle.dequant(p, s, z, "groupwise", g, K)
    r1 = rows[1]
    wh1 = oracle.dequant(r1.packed.numpy().view(np.uint32), r1.scales.view(torch.int16).numpy().view(np.uint16),
                         r1.zeros.view(torch.int16).numpy().view(np.uint16), "groupwise", g, r1.K)
    assert (wh1 == wh[:, r1.lo:r1.hi]).all()
