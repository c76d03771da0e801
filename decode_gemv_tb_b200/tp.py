"""Tensor-parallel sharding of a decoder layer's projections over the ranks
of a torch.distributed process group (one process per GPU).

The packed format splits without repacking: a row of W is a run of
independent 128-group blocks (32 bytes per group for the 2-bit container,
48 bytes for 3 bits: tb.h's layout), and each group has its own scale.  So
  * column-parallel (q, k, v, gate, up): rank r keeps the contiguous output
    rows [N r / R, N (r+1) / R) -- a slice of rows of the packed array and of
    the scales -- and computes its part of y with no exchange (all_gather
    only if every rank needs the whole y);
  * row-parallel (o, down): rank r keeps the contiguous 128-groups
    [G r / R, G (r+1) / R) of every row -- a slice of bytes of each packed row
    and of its scales -- multiplies them with its slice of x, and one
    all_reduce(SUM) of the fp32 partial y gives y.
The shard products are whatever `product(packed, grid, scales, x, N, K)`
computes; on a GPU that is tb.tb_gemv.  The all_reduce adds R fp32 partials,
each within the products' bound of its exact value, so the sum stays within
|y - y_exact| <= 1e-5 sum_k |x_k c_k s_k| plus R fp32 roundings of at most
sum_k |x_k c_k s_k| each.

Only the method's format facts are used here (group size, bytes per group);
the arithmetic runs in the product and the collective.
"""
from __future__ import annotations

import torch

GROUP = 128
INT3 = 2


def group_bytes(grid: int) -> int:
    """Packed bytes of one 128-group of one row (32 for the 2-bit container, 48 for 3 bits)."""
    return 48 if grid == INT3 else 32


def column_range(N: int, rank: int, world: int) -> tuple[int, int]:
    return N * rank // world, N * (rank + 1) // world


def group_range(K: int, rank: int, world: int) -> tuple[int, int]:
    G = K // GROUP
    return G * rank // world, G * (rank + 1) // world


def column_shard(packed: torch.Tensor, scales: torch.Tensor, grid: int, N: int, K: int, rank: int, world: int):
    """(packed rows, scales rows, n0, n1) of rank's output rows."""
    n0, n1 = column_range(N, rank, world)
    rb = K // GROUP * group_bytes(grid)
    p = packed.view(N, rb)[n0:n1].contiguous().view(-1)
    return p, scales.view(N, K // GROUP)[n0:n1].contiguous(), n0, n1


def row_shard(packed: torch.Tensor, scales: torch.Tensor, grid: int, N: int, K: int, rank: int, world: int):
    """(packed, scales, g0, g1) of rank's 128-groups of every row: a packed
    N x (g1 - g0) * 128 matrix of the same layout."""
    g0, g1 = group_range(K, rank, world)
    gb = group_bytes(grid)
    p = packed.view(N, K // GROUP * gb)[:, g0 * gb:g1 * gb].contiguous().view(-1)
    return p, scales.view(N, K // GROUP)[:, g0:g1].contiguous(), g0, g1


class ShardedLinear:
    """One projection split over the ranks of `group` (torch.distributed),
    column- or row-parallel."""

    def __init__(self, packed, scales, grid, N, K, kind, dist, group=None):
        if kind not in ("column", "row"):
            raise ValueError(kind)
        self.kind, self.grid, self.N, self.K, self.dist, self.group = kind, grid, N, K, dist, group
        self.rank, self.world = dist.get_rank(group), dist.get_world_size(group)
        if kind == "column":
            self.packed, self.scales, self.n0, self.n1 = column_shard(packed, scales, grid, N, K, self.rank,
                                                                      self.world)
        else:
            self.packed, self.scales, self.g0, self.g1 = row_shard(packed, scales, grid, N, K, self.rank, self.world)

    def local(self, x, product):
        """This rank's product: y rows [n0, n1) (column) or the partial y (row)."""
        if self.kind == "column":
            return product(self.packed, self.grid, self.scales, x, self.n1 - self.n0, self.K)
        xs = x[self.g0 * GROUP:self.g1 * GROUP].contiguous()
        return product(self.packed, self.grid, self.scales, xs, self.N, (self.g1 - self.g0) * GROUP)

    def forward(self, x, product, gather=True):
        """y = W x: the row-parallel partials are summed with one all_reduce;
        column-parallel rows are gathered when `gather` (else the local rows)."""
        y = self.local(x, product).float()
        if self.kind == "row":
            self.dist.all_reduce(y, op=self.dist.ReduceOp.SUM, group=self.group)
            return y
        if not gather:
            return y
        sizes = [column_range(self.N, r, self.world) for r in range(self.world)]
        parts = [torch.empty(b - a, dtype=y.dtype, device=y.device) for a, b in sizes]
        if max(b - a for a, b in sizes) == min(b - a for a, b in sizes):
            self.dist.all_gather(parts, y, group=self.group)
        else:  # uneven splits: pad to the largest, then trim
            m = max(b - a for a, b in sizes)
            buf = [torch.empty(m, dtype=y.dtype, device=y.device) for _ in sizes]
            pad = torch.zeros(m, dtype=y.dtype, device=y.device)
            pad[:y.numel()] = y
            self.dist.all_gather(buf, pad, group=self.group)
            parts = [b_[:hi - lo] for b_, (lo, hi) in zip(buf, sizes)]
        return torch.cat(parts)
