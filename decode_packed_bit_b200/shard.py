"""Row-sharded products across the GPUs of one node.

Every weight matrix W_r [N][K] of a group is split by output rows: rank q of
a world of G holds rows [n0_q, n1_q) of every matrix (contiguous blocks of
32-row tiles, the tile the product kernels stream), x is replicated, and each
rank computes its rows of y with the library's group call on its own memory
only.  One all-gather over the process group then gives every rank all of y.
There is no split over K, so no partial sums cross GPUs and nothing is
reduced: the exchange is the gather of M x N / G outputs per matrix.

The gathered buffer is rank-major: rank q's segment holds, for each matrix r,
that rank's [M][n1_q - n0_q] outputs at the start of a slot of M x rows_max
floats rounded up to a multiple of 4 (rows_max = the largest shard).
`assemble` turns it into dense [R][M][N].

Communication goes through torch.distributed (NCCL on GPUs, gloo on CPU in
the tests); no kernel reads another GPU's memory.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Sequence

TILE = 32


def row_shard(N: int, world: int, rank: int, tile: int = TILE) -> tuple[int, int]:
    """Rows [n0, n1) of `rank`: the ceil(N / tile) tiles are dealt out in
    contiguous runs whose lengths differ by at most one (the first N_tiles %
    world ranks take one more); the last run ends at N.  A rank may get an
    empty range when there are fewer tiles than ranks."""
    if N < 0 or world < 1 or not 0 <= rank < world or tile < 1:
        raise ValueError(f"row_shard: bad arguments N={N} world={world} rank={rank} tile={tile}")
    tiles = -(-N // tile)
    per, extra = divmod(tiles, world)
    t0 = rank * per + min(rank, extra)
    t1 = t0 + per + (1 if rank < extra else 0)
    return min(N, t0 * tile), min(N, t1 * tile)


def shard_sizes(N: int, world: int, tile: int = TILE) -> list[int]:
    return [b - a for a, b in (row_shard(N, world, q, tile) for q in range(world))]


@dataclass
class ShardLayout:
    """Where each rank's outputs sit in the gathered buffer."""
    R: int
    M: int
    N: int
    world: int
    tile: int = TILE

    @property
    def rows_max(self) -> int:
        return max(shard_sizes(self.N, self.world, self.tile))

    @property
    def slot(self) -> int:
        """floats per (rank, matrix) slot, rounded up to 4 so that every y_r
        a rank writes starts on a 16-byte boundary"""
        return -(-self.M * self.rows_max // 4) * 4

    @property
    def segment(self) -> int:
        """floats per rank"""
        return self.R * self.slot

    def bounds(self, rank: int) -> tuple[int, int]:
        return row_shard(self.N, self.world, rank, self.tile)


def assemble(gathered, layout: ShardLayout, out=None):
    """Dense y [R][M][N] from the rank-major gathered buffer (a torch tensor
    or numpy array of world * segment floats).  Rank q's matrix r occupies
    floats [q * segment + r * slot, ... + M * (n1_q - n0_q)) as [M][n1_q - n0_q]."""
    import numpy as np
    is_np = isinstance(gathered, np.ndarray)
    if out is None:
        if is_np:
            out = np.empty((layout.R, layout.M, layout.N), dtype=gathered.dtype)
        else:
            import torch
            out = torch.empty((layout.R, layout.M, layout.N), dtype=gathered.dtype, device=gathered.device)
    flat = gathered.reshape(-1)
    for q in range(layout.world):
        n0, n1 = layout.bounds(q)
        w = n1 - n0
        if w == 0:
            continue
        for r in range(layout.R):
            base = q * layout.segment + r * layout.slot
            out[r, :, n0:n1] = flat[base:base + layout.M * w].reshape(layout.M, w)
    return out


LocalProduct = Callable[[Sequence, Sequence, object, Sequence], None]


class RowShardedGroup:
    """R matrices of one shape [N][K], row-sharded over a process group.

    local_bits / local_scales: this rank's rows [n0, n1) of every matrix, in
    the packed layout of `fmt` ("q1": uint8 [rows][K/8] and fp16 bits
    [rows][K/128]; "int4": uint8 [rows][K/2] and fp16 bits [rows][K/64]).
    step(x) computes this rank's outputs into its segment of the gathered
    buffer with the library's group call, then all-gathers the segments.
    `local_product(bits, scales, x, ys)` replaces the library call (the CPU
    tests pass one that runs on the host)."""

    def __init__(self, fmt: str, local_bits, local_scales, N: int, K: int, M: int, group=None, device=None,
                 local_product: LocalProduct | None = None, stream=None):
        import torch
        import torch.distributed as dist
        self.fmt = fmt
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.layout = ShardLayout(len(local_bits), M, N, self.world)
        self.n0, self.n1 = self.layout.bounds(self.rank)
        self.rows = self.n1 - self.n0
        for b in local_bits:
            if b.shape[0] != self.rows:
                raise ValueError(f"rank {self.rank}: shard has {b.shape[0]} rows, expected {self.rows}")
        self.bits, self.scales = list(local_bits), list(local_scales)
        self.N, self.K, self.M = N, K, M
        self.device = device if device is not None else (local_bits[0].device if local_bits else "cpu")
        lay = self.layout
        self.local = torch.zeros(lay.segment, dtype=torch.float32, device=self.device)
        self.gathered = (self.local if lay.world == 1 else
                         torch.zeros(lay.world * lay.segment, dtype=torch.float32, device=self.device))
        # this rank's y_r: [M][rows] at the start of its slot (contiguous views)
        self.ys = [self.local[r * lay.slot: r * lay.slot + M * self.rows].view(M, self.rows)
                   for r in range(lay.R)]
        self.stream = stream
        self.workspace = None
        if local_product is None and fmt == "q1" and self.rows > 0:
            from . import lowbit as lb
            need = lb.lowbit_q1g128_group_workspace_bytes(lay.R, M, self.rows, K)
            if need:
                self.workspace = torch.zeros(need, dtype=torch.uint8, device=self.device)
        self.local_product = local_product or self._library_product

    def _library_product(self, bits, scales, x, ys):
        from . import lowbit as lb
        if self.fmt == "q1":
            lb.lowbit_q1g128_gemv_group(bits, scales, x, ys, workspace=self.workspace, stream=self.stream)
        elif self.fmt == "int4":
            lb.lowbit_int4g64_gemm_group(bits, scales, x, ys, stream=self.stream)
        else:
            raise ValueError(f"unknown format {self.fmt!r}")

    def compute(self, x):
        """This rank's rows of every y_r (no communication)."""
        if self.rows > 0:
            self.local_product(self.bits, self.scales, x, self.ys)

    def gather(self):
        """All-gather every rank's segment into self.gathered (rank-major)."""
        import torch.distributed as dist
        if self.world > 1:  # with one rank the local segment is the whole buffer
            dist.all_gather_into_tensor(self.gathered, self.local, group=self.group)
        return self.gathered

    def step(self, x):
        self.compute(x)
        return self.gather()

    def dense(self, out=None):
        return assemble(self.gathered, self.layout, out)
