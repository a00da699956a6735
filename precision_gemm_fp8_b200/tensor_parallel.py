"""Tensor-parallel FP8 linear layers over several GPUs of one node.

"C++ and FP8" §4.2 deploys the quantised model with a tensor-parallel size
(--tp_size) and §5.2 sums the partial results of a split layer with an
all-reduce over NVLink.  One process per GPU; torch.distributed (NCCL over
NVLink / NVSwitch) carries the collectives; every arithmetic step runs in the
library's kernels (`Fp8Ops`).

Column-parallel (the weight split along N): rank r holds the channels
[r N/R, (r+1) N/R) with their per-channel scales.  The per-token scale is
the amax over the whole activation row, which every rank holds, so every
rank quantises identically and computes its channels with no exchange; the
full output, when wanted, is an all-gather of the ranks' column blocks.

Row-parallel (the weight split along K): rank r holds columns
[r K/R, (r+1) K/R) of every weight row and the same slice of every
activation row.  The per-token scale must still come from the whole row
("7B on an RTX 4060 with FP8" §2.2 dynamic per-token scale, §6.1 scale =
amax / 448), so each rank takes the amax of its slice, an all-reduce MAX
makes it the row's amax, and the codes are formed from it: bit-identical to
quantising the unsplit row.  Each rank's f32 partial product (scaled by
sa[m] sw[n]; sw belongs to the unsplit weight row) is summed by an all-reduce
SUM in f32 and rounded to bf16 once.

No TMA multicast is used anywhere (each kernel reads only this GPU's memory).
"""
from __future__ import annotations

import dataclasses

import torch
import torch.distributed as dist


class Fp8Ops:
    """The arithmetic steps of a tensor-parallel layer: the library's kernels."""

    def __init__(self):
        import precision_gemm_fp8_b200 as pg
        self.pg = pg

    def row_amax(self, x):
        return self.pg.fp8_row_amax(x)

    def quantize_rows_amax(self, x, amax):
        return self.pg.fp8_quantize_rows_amax(x, amax)

    def quantize_rows(self, x):
        return self.pg.fp8_quantize_rows(x)

    def linear_partial(self, aq, sa, wq, sw):
        return self.pg.fp8_linear_partial(aq, sa, wq, sw)

    def round_bf16(self, y):
        return self.pg.round_bf16(y)

    def linear_dynamic(self, x, wq, sw):
        return self.pg.fp8_linear_dynamic(x, wq, sw)


@dataclasses.dataclass
class TPGroup:
    rank: int
    world: int
    group: object = None     # torch.distributed process group (None: the default group)

    @staticmethod
    def current(group=None) -> "TPGroup":
        if not dist.is_initialized():
            return TPGroup(0, 1, group)
        return TPGroup(dist.get_rank(group), dist.get_world_size(group), group)


def split_range(total: int, world: int, rank: int, align: int = 16) -> tuple[int, int]:
    """Rank's contiguous block [start, stop) of `total`, in equal blocks that
    are multiples of `align` (the kernels' 16-element K / N granularity)."""
    if total % (align * world) != 0:
        raise ValueError(f"{total} does not split into {world} blocks of a multiple of {align}")
    b = total // world
    return rank * b, (rank + 1) * b


class ColumnParallelFP8Linear:
    """y[:, block r] = FP8 linear of x with the rank's channels; gather=True
    all-gathers the blocks into the full [M, N] output on every rank."""

    def __init__(self, wq, sw, tp: TPGroup, ops: Fp8Ops | None = None):
        """wq [N, K] E4M3 codes and sw [N] of the unsplit layer (quantised per
        channel once, offline); this rank keeps its block of channels."""
        self.tp = tp
        self.ops = ops if ops is not None else Fp8Ops()
        N = wq.shape[0]
        self.n0, self.n1 = split_range(N, tp.world, tp.rank)
        self.wq = wq[self.n0:self.n1].contiguous()
        self.sw = sw[self.n0:self.n1].contiguous()
        self.N = N

    def forward(self, x, gather=False):
        y = self.ops.linear_dynamic(x, self.wq, self.sw)
        if not gather or self.tp.world == 1:
            return y
        parts = [torch.empty_like(y) for _ in range(self.tp.world)]
        dist.all_gather(parts, y.contiguous(), group=self.tp.group)
        return torch.cat(parts, dim=1)


class RowParallelFP8Linear:
    """y [M, N] (bf16, on every rank) of the full layer from the rank's slice
    of K: all-reduce MAX of the per-token amax, codes from the row amax, f32
    partial product, all-reduce SUM, one rounding to bf16."""

    def __init__(self, wq, sw, tp: TPGroup, ops: Fp8Ops | None = None):
        """wq [N, K] E4M3 codes and sw [N] of the unsplit layer (each channel's
        scale comes from its whole row); this rank keeps its slice of K."""
        self.tp = tp
        self.ops = ops if ops is not None else Fp8Ops()
        K = wq.shape[1]
        self.k0, self.k1 = split_range(K, tp.world, tp.rank)
        self.wq = wq[:, self.k0:self.k1].contiguous()
        self.sw = sw.contiguous()
        self.K = K

    def slice_input(self, x):
        """This rank's slice [M, K/R] of full activation rows x [M, K]."""
        return x[:, self.k0:self.k1].contiguous()

    def quantize(self, x_r):
        """Codes of this rank's slice and the per-token scales of the whole
        rows (identical on every rank)."""
        amax = self.ops.row_amax(x_r)
        if self.tp.world > 1:
            dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=self.tp.group)
        return self.ops.quantize_rows_amax(x_r, amax)

    def forward(self, x_r):
        aq, sa = self.quantize(x_r)
        y = self.ops.linear_partial(aq, sa, self.wq, self.sw)
        if self.tp.world > 1:
            dist.all_reduce(y, op=dist.ReduceOp.SUM, group=self.tp.group)
        return self.ops.round_bf16(y)
