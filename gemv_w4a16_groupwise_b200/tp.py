"""Tensor-parallel sharding of one W4A16 layer over torch.distributed ranks.

The packed layout shards along both of its axes without repacking:

* column-parallel (over N, the output rows of W): rank r holds packed rows
  [N0, N1) with their scale / zero rows.  The forward product of each rank
  is its own slice of Y; a consumer that is itself sharded needs nothing
  more, else one all-gather along N rebuilds Y.  The transposed product
  dX = dY . w_hat is then a sum over N, i.e. row-parallel: each rank
  multiplies its slice of dY by its rows and one all-reduce adds them.
* row-parallel (over K): rank r holds packed columns [K0 / 8, K1 / 8) and
  the groups [K0 / g, K1 / g) of every row, so K1 - K0 must be a multiple of
  the group length (and of 8); per-row and global scales are shared.  The
  forward product is a sum over K: each rank multiplies its slice of X and
  one all-reduce adds the partial outputs (the bias once, after it).  The
  transposed product gives each rank its own slice of dX (an all-gather
  rebuilds the whole).

This is how the fused QKV weight of the torchao page "Add fused QKV HQQ
triton_mm test" is built as well: concatenation along N is the same split
as column parallelism, its equivalence test (forward = concatenation,
transposed = sum) is this module's column-parallel identity.

The local products run the library's kernels through ``matmul`` (by default
:func:`gemv_w4a16_groupwise_b200.w4a16_gemm`; any callable with its
signature works, which is how the CPU tests drive the sharding logic).
The partial outputs are summed in fp32 and rounded to bf16 once.  With the
gloo backend, CUDA tensors go through host memory for the collectives; with
NCCL they stay on the device.
"""
from __future__ import annotations

from dataclasses import dataclass


def _torch():
    import torch
    return torch


def split_range(total: int, world: int, rank: int, quantum: int = 1) -> tuple[int, int]:
    """[lo, hi) of `rank` when `total` is cut into `world` contiguous parts whose
    sizes are multiples of `quantum` (the parts differ by at most one quantum)."""
    if total % quantum:
        raise ValueError(f"{total} is not a multiple of the shard quantum {quantum}")
    units = total // quantum
    if units < world:
        raise ValueError(f"cannot split {units} units of {quantum} over {world} ranks")
    lo = rank * units // world
    hi = (rank + 1) * units // world
    return lo * quantum, hi * quantum


def _own(t):
    """A copy of a slice in storage of its own: slices of the full layer can start off
    the 16-byte alignment the library requires, fresh allocations do not."""
    return t.clone(memory_format=_torch().contiguous_format)


def _mode_base(mode) -> str:
    if isinstance(mode, str):
        return mode
    return {0: "global", 1: "rowwise", 2: "groupwise"}[int(mode) & 0x0F]


@dataclass
class Shard:
    """One rank's part of a packed layer (tensors in the layout of the full one)."""
    packed: object          # int32 [N_local, K_local / 8]
    scales: object
    zeros: object
    N: int                  # rows of this shard
    K: int                  # reduction length of this shard
    lo: int                 # first row (column-parallel) or first k (row-parallel)
    hi: int


def shard_columns(packed, scales, zeros, mode, group_size: int, N: int, K: int, rank: int,
                  world: int) -> Shard:
    """Rows [N0, N1) of W (column parallelism over N)."""
    lo, hi = split_range(N, world, rank)
    base = _mode_base(mode)
    if base == "global":
        s, z = scales, zeros
    else:
        s, z = scales[lo:hi], zeros[lo:hi]
    return Shard(_own(packed[lo:hi]), _own(s), _own(z), hi - lo, K, lo, hi)


def shard_rows(packed, scales, zeros, mode, group_size: int, N: int, K: int, rank: int,
               world: int) -> Shard:
    """Reduction range [K0, K1) of W (row parallelism over K); K1 - K0 is a
    multiple of the group length for groupwise weights, of 8 otherwise."""
    base = _mode_base(mode)
    quantum = group_size if base == "groupwise" else 8
    if quantum % 8:
        raise ValueError("the group length must be a multiple of 8")
    lo, hi = split_range(K, world, rank, quantum)
    p = _own(packed[:, lo // 8:hi // 8])
    if base == "groupwise":
        s = _own(scales[:, lo // group_size:hi // group_size])
        z = _own(zeros[:, lo // group_size:hi // group_size])
    else:
        s, z = scales, zeros
    return Shard(p, s, z, N, hi - lo, lo, hi)


def _default_matmul():
    from . import w4a16_gemm
    return w4a16_gemm


class _Comm:
    """The two collectives of the layer, fp32 payloads, on the group's device kind."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.backend = dist.get_backend(group)
        self.world = dist.get_world_size(group)

    def _staged(self, t):
        # gloo takes host tensors; NCCL device tensors
        return t.cpu() if (self.backend == "gloo" and t.is_cuda) else t

    def all_reduce_sum(self, t):
        x = self._staged(t.float().contiguous())
        self.dist.all_reduce(x, op=self.dist.ReduceOp.SUM, group=self.group)
        return x.to(t.device)

    def all_gather_cols(self, t, sizes):
        """Concatenate each rank's [M, n_r] along dim 1 (n_r = sizes[r])."""
        torch = _torch()
        x = self._staged(t.float().contiguous())
        M = x.shape[0]
        width = max(sizes)
        pad = torch.zeros((M, width), dtype=x.dtype, device=x.device)
        pad[:, :x.shape[1]] = x
        bufs = [torch.empty_like(pad) for _ in range(self.world)]
        self.dist.all_gather(bufs, pad, group=self.group)
        return torch.cat([b[:, :n] for b, n in zip(bufs, sizes)], dim=1).to(t.device)


class ColumnParallelW4A16:
    """Y[:, N0:N1] = X . w_hat[N0:N1]^T on each rank; see the module notes."""

    def __init__(self, packed, scales, zeros, mode, group_size: int, N: int, K: int, *, bias=None,
                 zero: str = "int", group=None, matmul=None):
        import torch.distributed as dist
        self.comm = _Comm(group)
        self.rank = dist.get_rank(group)
        self.mode, self.g, self.N, self.K, self.zero = mode, group_size, N, K, zero
        self.shard = shard_columns(packed, scales, zeros, mode, group_size, N, K, self.rank, self.comm.world)
        self.sizes = [split_range(N, self.comm.world, r) for r in range(self.comm.world)]
        self.bias = None if bias is None else _own(bias[self.shard.lo:self.shard.hi])
        self.matmul = matmul or _default_matmul()

    def forward(self, X, gather: bool = True):
        """X [M, K] (whole) -> Y [M, N] (gather) or this rank's Y [M, N1 - N0]."""
        sh = self.shard
        y = self.matmul(X, sh.packed, sh.scales, sh.zeros, self.mode, self.g, N=sh.N, K=self.K,
                        bias=self.bias, zero=self.zero)
        if not gather:
            return y
        full = self.comm.all_gather_cols(y, [hi - lo for lo, hi in self.sizes])
        return full.to(y.dtype)

    def backward_input(self, dY):
        """dY [M, N] (whole, or this rank's [M, N1 - N0]) -> dX [M, K], summed over ranks."""
        torch = _torch()
        sh = self.shard
        d = _own(dY[:, sh.lo:sh.hi]) if dY.shape[1] == self.N and self.comm.world > 1 else dY
        part = self.matmul(d, sh.packed, sh.scales, sh.zeros, self.mode, self.g, N=sh.N, K=self.K,
                           transposed=True, zero=self.zero)
        return self.comm.all_reduce_sum(part).to(torch.bfloat16)


class RowParallelW4A16:
    """Y = sum over ranks of X[:, K0:K1] . w_hat[:, K0:K1]^T; see the module notes."""

    def __init__(self, packed, scales, zeros, mode, group_size: int, N: int, K: int, *, bias=None,
                 zero: str = "int", group=None, matmul=None):
        import torch.distributed as dist
        self.comm = _Comm(group)
        self.rank = dist.get_rank(group)
        self.mode, self.g, self.N, self.K, self.zero = mode, group_size, N, K, zero
        self.shard = shard_rows(packed, scales, zeros, mode, group_size, N, K, self.rank, self.comm.world)
        quantum = group_size if _mode_base(mode) == "groupwise" else 8
        self.sizes = [split_range(K, self.comm.world, r, quantum) for r in range(self.comm.world)]
        self.bias = bias
        self.matmul = matmul or _default_matmul()

    def forward(self, X):
        """X [M, K] (whole) or this rank's X [M, K1 - K0] -> Y [M, N] (all-reduced, + bias once)."""
        torch = _torch()
        sh = self.shard
        x = _own(X[:, sh.lo:sh.hi]) if X.shape[1] == self.K and self.comm.world > 1 else X
        part = self.matmul(x, sh.packed, sh.scales, sh.zeros, self.mode, self.g, N=self.N, K=sh.K,
                           zero=self.zero)
        y = self.comm.all_reduce_sum(part)
        if self.bias is not None:
            y = y + self.bias.float()
        return y.to(torch.bfloat16)

    def backward_input(self, dY, gather: bool = True):
        """dY [M, N] -> dX [M, K] (gather) or this rank's dX [M, K1 - K0]."""
        sh = self.shard
        part = self.matmul(dY, sh.packed, sh.scales, sh.zeros, self.mode, self.g, N=self.N, K=sh.K,
                           transposed=True, zero=self.zero)
        if not gather:
            return part
        return self.comm.all_gather_cols(part, [hi - lo for lo, hi in self.sizes]).to(part.dtype)
