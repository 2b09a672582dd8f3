"""Oracle for the MoE steps around the grouped product (test infrastructure only).

Page 2 (the MegaMoE swap-AB kernel) dispatches each token to its top-k experts,
runs one grouped GEMM over the expert-grouped rows, and combines each token's k
expert outputs with its routing weights.  The pages fix no order inside an
expert; the reading used here is the stable one, pairs (token t, slot j),
p = t*k + j, in ascending p inside each expert.

Only tests/, __graft_entry__.smoke() and bench.py's CPU baseline use this
module.  It shares nothing with the CUDA library: plain numpy, FP64 for the
weighted sums.
"""
import numpy as np


def route(expert_ids, E):
    """expert_ids [P] (or [T, k]) -> (offsets [E+1], dest [P], src [P]), int64.

    offsets[e] = number of pairs routed to experts < e; the pairs of expert e
    take rows offsets[e] .. offsets[e+1]-1 in ascending p; dest[p] is pair p's row
    and src[r] the pair on row r.  Ids outside [0, E) are placed nowhere
    (dest = -1) and do not count."""
    ids = np.asarray(expert_ids, dtype=np.int64).reshape(-1)
    P = ids.size
    valid = (ids >= 0) & (ids < E)
    counts = np.bincount(ids[valid], minlength=E)[:E]
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    dest = np.full(P, -1, dtype=np.int64)
    src = np.full(P, -1, dtype=np.int64)
    filled = np.zeros(E, dtype=np.int64)
    for p in range(P):          # ascending p: stable inside each expert
        if valid[p]:
            e = ids[p]
            r = offsets[e] + filled[e]
            filled[e] += 1
            dest[p] = r
            src[r] = p
    return offsets, dest, src


def permute_rows(x, src, k):
    """out[r] = x[src[r] // k] (rows of bytes in token order -> grouped order)."""
    x = np.asarray(x)
    src = np.asarray(src, dtype=np.int64)
    out = np.zeros((src.size,) + x.shape[1:], dtype=x.dtype)
    for r, p in enumerate(src):
        if p >= 0:
            out[r] = x[p // k]
    return out


def combine(Yg, dest, weights, T, k):
    """Y[t] = sum_j weights[t, j] * Yg[dest[t*k + j]], in FP64 (weights None: 1)."""
    Yg = np.asarray(Yg, dtype=np.float64)
    dest = np.asarray(dest, dtype=np.int64).reshape(T, k)
    w = np.ones((T, k)) if weights is None else np.asarray(weights, dtype=np.float64).reshape(T, k)
    Y = np.zeros((T, Yg.shape[1]), dtype=np.float64)
    for t in range(T):
        for j in range(k):
            r = dest[t, j]
            if 0 <= r < Yg.shape[0]:
                Y[t] += w[t, j] * Yg[r]
    return Y
