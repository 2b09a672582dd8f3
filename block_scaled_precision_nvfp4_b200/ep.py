"""Expert parallelism around the grouped W4A4 product (page 2's MegaMoE dispatch
and combine, across GPUs): the E experts are split into contiguous ranges over
the ranks of a process group, each token row goes to the ranks that own its
top-k experts, and the expert outputs come back to combine.

The exchange is torch.distributed's all-to-all (NCCL over NVLink between GPUs);
every local step runs in this package's kernels:

  dispatch  route (expert offsets, stable order) -> permute the token rows
            into that order -> exchange the per-expert row counts -> exchange
            the rows (codes and scales) -> regroup the received rows by local
            expert (a second row permutation);
  compute   the caller's grouped product over the local experts;
  combine   undo the regroup -> exchange the output rows back -> weighted
            combine per token.

`LocalOps` names the three local steps; the default is the CUDA library (route,
permute_rows, combine).  A rank takes every collective in the same order.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


def expert_range(E: int, world: int, rank: int) -> tuple[int, int]:
    """Experts [e0, e1) owned by `rank`: contiguous, E // world each (E % world == 0)."""
    if E % world != 0:
        raise ValueError(f"E ({E}) must be a multiple of the world size ({world})")
    per = E // world
    return rank * per, (rank + 1) * per


class LocalOps:
    """The local steps on CUDA tensors, through the library's kernels."""

    def route(self, ids, E):
        from . import moe_route
        return moe_route(ids, E)

    def permute(self, x, src, k):
        from . import moe_permute_rows
        return moe_permute_rows(x, src, k)

    def combine(self, Yg, dest, weights, T, k):
        from . import moe_combine
        return moe_combine(Yg, dest, weights, T, k)


@dataclass
class Dispatched:
    """What a rank holds after dispatch: its local experts' rows, grouped."""
    codes: object            # uint8 [R, K/2], grouped by local expert
    scales: object           # uint8 [R, K/16]
    local_offsets: list      # host ints [E_local + 1]
    # bookkeeping for the way back
    dest: object             # int32 [T*k]: each local pair's row in the sent order
    inv: object              # int32 [R]: received row -> its row in the regrouped order
    send_splits: list
    recv_splits: list
    T: int
    k: int


def _regroup_index(recv_counts: np.ndarray) -> np.ndarray:
    """Rows received as [source][local expert] blocks -> [local expert][source] order:
    the received row that lands on each regrouped row."""
    W, El = recv_counts.shape
    start = np.zeros((W, El), dtype=np.int64)        # first received row of block (s, e)
    run = 0
    for s in range(W):
        for e in range(El):
            start[s, e] = run
            run += int(recv_counts[s, e])
    idx = [np.arange(start[s, e], start[s, e] + recv_counts[s, e], dtype=np.int64)
           for e in range(El) for s in range(W)]
    return np.concatenate(idx) if idx else np.zeros(0, dtype=np.int64)


def dispatch(codes, scales, expert_ids, E, group=None, ops=None) -> Dispatched:
    """codes uint8 [T, K/2], scales uint8 [T, K/16], expert_ids int32 [T, k] (one
    rank's tokens) -> this rank's experts' rows from every rank, grouped."""
    import torch
    import torch.distributed as dist
    ops = ops or LocalOps()
    W = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    T, k = expert_ids.shape
    dev = codes.device
    off, dest, src = ops.route(expert_ids.reshape(-1).contiguous(), E)
    g_codes = ops.permute(codes, src, k)
    g_scales = ops.permute(scales, src, k)
    counts = (off[1:] - off[:-1]).to(torch.int64)                 # rows per expert, all E
    e0, e1 = expert_range(E, W, rank)
    El = e1 - e0
    if W > 1:
        recv = torch.empty_like(counts)
        dist.all_to_all_single(recv, counts, group=group)         # E/W counts per peer
    else:
        recv = counts
    recv_counts = recv.cpu().numpy().reshape(W, El)
    send_splits = [int(x) for x in counts.cpu().numpy().reshape(W, El).sum(axis=1)]
    recv_splits = [int(x) for x in recv_counts.sum(axis=1)]
    R = sum(recv_splits)
    if W > 1:
        r_codes = torch.empty((R, g_codes.shape[1]), dtype=g_codes.dtype, device=dev)
        r_scales = torch.empty((R, g_scales.shape[1]), dtype=g_scales.dtype, device=dev)
        dist.all_to_all_single(r_codes, g_codes, recv_splits, send_splits, group=group)
        dist.all_to_all_single(r_scales, g_scales, recv_splits, send_splits, group=group)
    else:
        r_codes, r_scales = g_codes, g_scales
    regroup = _regroup_index(recv_counts)
    src2 = torch.from_numpy(regroup.astype(np.int32)).to(dev)
    inv_np = np.empty(R, dtype=np.int32)
    inv_np[regroup] = np.arange(R, dtype=np.int32)
    loc_counts = recv_counts.sum(axis=0)
    local_offsets = [0] + [int(x) for x in np.cumsum(loc_counts)]
    return Dispatched(codes=ops.permute(r_codes, src2, 1) if R else r_codes,
                      scales=ops.permute(r_scales, src2, 1) if R else r_scales,
                      local_offsets=local_offsets, dest=dest,
                      inv=torch.from_numpy(inv_np).to(dev), send_splits=send_splits,
                      recv_splits=recv_splits, T=T, k=k)


def combine(Yg_local, state: Dispatched, weights, group=None, ops=None):
    """Yg_local BF16 [R, N] in the regrouped order (the grouped product over the local
    experts) -> this rank's tokens, Y BF16 [T, N] = sum_j w[t, j] * row of (t, j)."""
    import torch
    import torch.distributed as dist
    ops = ops or LocalOps()
    W = dist.get_world_size(group) if dist.is_initialized() else 1
    R, N = Yg_local.shape
    rows_u8 = Yg_local.view(torch.uint8) if R else Yg_local.view(torch.uint8)
    back = ops.permute(rows_u8, state.inv, 1) if R else rows_u8          # received order
    P = state.T * state.k
    if W > 1:
        out = torch.empty((P, rows_u8.shape[1]), dtype=torch.uint8, device=Yg_local.device)
        dist.all_to_all_single(out, back.contiguous(), state.send_splits, state.recv_splits,
                               group=group)
    else:
        out = back
    Yg = out.view(Yg_local.dtype).reshape(P, N)
    return ops.combine(Yg, state.dest, weights, state.T, state.k)
