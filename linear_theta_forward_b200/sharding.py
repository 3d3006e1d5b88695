"""The theta path split across GPUs: one process per GPU, torch.distributed.

Every tensor of the theta bundle is indexed by output row ("The theta bundle"
-- component table: W0 [out, in], s [out], U [out, rank]; only V [in, rank]
is indexed by input), and every step of the path works row by row: band
mean, row scale, residual and reconstruct touch one row of each tensor at a
time, the relative Frobenius error is a ratio of two sums over rows, and the
forward's output column o needs only row o of W0, s and U. So a family's O
rows split into contiguous blocks, one per rank:

  * rank k holds rows [o0, o1) of every W_l, W0, s, U and R, and the whole of
    V and X;
  * band mean, row scale, residual and reconstruct run on the block with no
    exchange at all;
  * the forward gives Y[:, o0:o1] on each rank; when the consumer wants all
    of Y, one all-gather of the column blocks assembles it (gather_columns);
  * the relative Frobenius error all-reduces the two sums of every rank
    (theta_frob_partials), then takes the ratio of their square roots
    (frob_from_sums).

A projection whose input is itself split by columns -- the down projection
after gate and up projections split by rows -- is split along I instead: rank
k holds W0[:, i0:i1], V[i0:i1] and the whole of s and U, and the forward is
linear in that split,

  Y = s * (X.W0^T) + (X.V).U^T = sum_k [ s * (X_k.W0_k^T) + (X_k.V_k).U^T ],

so each rank's forward of its block is a partial Y and one all-reduce sums
them (allreduce_partials).

Blocks start on multiples of `align` rows (8: the bf16 kernels need 16-byte
aligned rows and row counts that are multiples of 8); earlier ranks take the
remainder, as earlier bands do. The functions here are host logic over
torch.distributed (NCCL between GPUs, gloo on the CPU); the arithmetic of
each block is the library's.
"""
from __future__ import annotations

import math

__all__ = ["row_blocks", "block_of", "gather_columns", "gather_rows", "allreduce_partials", "frob_from_sums",
           "sharded_frob_error", "forward_rows", "forward_k"]


def row_blocks(n: int, world: int, align: int = 8) -> list[tuple[int, int]]:
    """[(o0, o1)] for each rank: n rows in contiguous blocks of whole
    `align`-row units, as equal as possible, earlier blocks taking the
    remainder; the last block also takes the n % align tail rows."""
    if world < 1 or n < 0 or align < 1:
        raise ValueError(f"row_blocks: bad arguments n={n}, world={world}, align={align}")
    units = n // align
    q, m = divmod(units, world)
    out, start = [], 0
    for k in range(world):
        size = (q + (1 if k < m else 0)) * align
        out.append((start, start + size))
        start += size
    o0, _ = out[-1]
    out[-1] = (o0, n)
    return out


def block_of(n: int, rank: int, world: int, align: int = 8) -> tuple[int, int]:
    return row_blocks(n, world, align)[rank]


def _dist():
    import torch.distributed as dist
    return dist


def gather_columns(Y_local, n_cols: int, group=None, align: int = 8):
    """Assembles Y [M, n_cols] on every rank from each rank's column block
    Y_local [M, o1 - o0] (row_blocks(n_cols, world, align)): blocks are padded
    to the widest one, all-gathered, and placed side by side."""
    import torch
    dist = _dist()
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    blocks = row_blocks(n_cols, world, align)
    o0, o1 = blocks[rank]
    M = Y_local.shape[0]
    if tuple(Y_local.shape) != (M, o1 - o0):
        raise ValueError(f"gather_columns: rank {rank} holds {tuple(Y_local.shape)}, expected {(M, o1 - o0)}")
    wmax = max(b - a for a, b in blocks)
    pad = Y_local.new_zeros((M, wmax))
    pad[:, :o1 - o0] = Y_local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad.contiguous(), group=group)
    return torch.cat([p[:, :b - a] for p, (a, b) in zip(parts, blocks)], dim=1)


def gather_rows(T_local, n_rows: int, group=None, align: int = 8):
    """Assembles a row-split tensor (W0, R, s: [n_rows, ...]) on every rank
    from each rank's row block."""
    return gather_columns(T_local.reshape(T_local.shape[0], -1).T.contiguous(), n_rows, group, align).T.reshape(
        (n_rows,) + tuple(T_local.shape[1:]))


def allreduce_partials(t, group=None):
    """Sums a tensor over ranks in place (the K-split forward's partial
    outputs, the Frobenius sums) and returns it."""
    dist = _dist()
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return t


def frob_from_sums(num: float, den: float) -> float:
    """sqrt(num) / sqrt(den): 0 when both are 0, +inf when only den is."""
    if den == 0.0:
        return 0.0 if num == 0.0 else math.inf
    return math.sqrt(num) / math.sqrt(den)


def sharded_frob_error(A_block, B_block, workspace, group=None, stream=None) -> float:
    """relative_frobenius_error of a matrix whose rows are split across the
    ranks: each rank passes its row block of the original and of the
    reconstruction."""
    import torch
    import linear_theta_forward_b200 as theta
    sums = torch.empty(2, dtype=torch.float64, device=A_block.device)
    theta.theta_frob_partials(A_block, B_block, sums, workspace, stream=stream)
    allreduce_partials(sums, group)
    num, den = sums.tolist()
    return frob_from_sums(num, den)


def forward_rows(X, W0_block, s_block, U_block, V, workspace, n_cols, group=None, gather=True, stream=None):
    """The forward of a projection split by output rows: this rank's column
    block s*(X.W0_k^T) + (X.V).U_k^T, and (gather=True) all of Y."""
    import torch
    import linear_theta_forward_b200 as theta
    Y_local = torch.empty(X.shape[0], W0_block.shape[0], dtype=X.dtype, device=X.device)
    theta.theta_linear_forward(X, W0_block, s_block, U_block, V, Y_local, workspace, stream=stream)
    return gather_columns(Y_local, n_cols, group) if gather else Y_local


def forward_k(X_block, W0_block, s, U, V_block, workspace, group=None, stream=None):
    """The forward of a projection split along its input: this rank's partial
    s*(X_k.W0_k^T) + (X_k.V_k).U^T, summed over ranks. Each partial comes out
    of the forward in the activation dtype; the sum over ranks is taken in
    fp32 and rounded once more to that dtype."""
    import torch
    import linear_theta_forward_b200 as theta
    part = torch.empty(X_block.shape[0], W0_block.shape[0], dtype=X_block.dtype, device=X_block.device)
    theta.theta_linear_forward(X_block, W0_block, s, U, V_block, part, workspace, stream=stream)
    acc = part.float()
    allreduce_partials(acc, group)
    return acc.to(X_block.dtype)
