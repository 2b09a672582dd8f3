"""Expert-parallel dispatch and combine across two ranks (gloo on CPU).

The exchange logic of block_scaled_precision_nvfp4_b200.ep: per-expert count
exchange, row all-to-all, regrouping by local expert, and the way back. It is
checked with the oracle's route/permute/combine standing in for the CUDA
kernels, and with a marker function standing in for the grouped product: row i
of expert e becomes f(row bytes, e). Each rank's output must equal the
weighted sum, over its own tokens' top-k experts, of f of the token's row."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import moe as om

E, K2, KS, N = 8, 32, 4, 6          # experts, code bytes, scale bytes per row, output width


class OracleOps:
    def route(self, ids, E):
        off, dest, src = om.route(ids.numpy(), E)
        return (torch.from_numpy(off.astype(np.int32)), torch.from_numpy(dest.astype(np.int32)),
                torch.from_numpy(src.astype(np.int32)))

    def permute(self, x, src, k):
        return torch.from_numpy(om.permute_rows(x.numpy(), src.numpy(), k))

    def combine(self, Yg, dest, weights, T, k):
        w = None if weights is None else weights.numpy()
        return torch.from_numpy(om.combine(Yg.numpy(), dest.numpy(), w, T, k))


def f(codes_row, scales_row, e):
    """The stand-in expert: N floats from the row's bytes and the expert id."""
    c = codes_row.astype(np.float64)
    return (c[:N] + 3.0 * c[N:2 * N] + scales_row.astype(np.float64).sum()) * (e + 1)


def _tokens(rank):
    rng = np.random.default_rng(100 + rank)
    T, k = (37, 53)[rank], 2
    ids = rng.integers(0, E, size=(T, k)).astype(np.int32)
    ids[:, 1] = np.where(ids[:, 1] == 2, 7, ids[:, 1])        # expert 2 only ever as slot 0
    codes = rng.integers(0, 256, size=(T, K2), dtype=np.uint8)
    scales = rng.integers(0, 0x7F, size=(T, KS), dtype=np.uint8)
    w = rng.random((T, k)).astype(np.float32)
    return ids, codes, scales, w


def _rank(rank, world, port, q):
    from block_scaled_precision_nvfp4_b200 import ep
    os.environ["MASTER_ADDR"], os.environ["MASTER_PORT"] = "127.0.0.1", str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ids, codes, scales, w = _tokens(rank)
        ops = OracleOps()
        st = ep.dispatch(torch.from_numpy(codes), torch.from_numpy(scales), torch.from_numpy(ids),
                         E, ops=ops)
        e0, e1 = ep.expert_range(E, world, rank)
        # the stand-in grouped product over this rank's experts
        R = st.codes.shape[0]
        Yl = np.zeros((R, N), dtype=np.float64)
        off = st.local_offsets
        for le in range(e1 - e0):
            for r in range(off[le], off[le + 1]):
                Yl[r] = f(st.codes[r].numpy(), st.scales[r].numpy(), e0 + le)
        Y = ep.combine(torch.from_numpy(Yl), st, torch.from_numpy(w), ops=ops).numpy()
        T, k = ids.shape
        want = np.array([sum(w[t, j] * f(codes[t], scales[t], ids[t, j]) for j in range(k))
                         for t in range(T)])
        q.put((rank, bool(np.allclose(Y, want, rtol=1e-12, atol=1e-9)), st.local_offsets,
               st.send_splits, st.recv_splits))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_rank_dispatch_and_combine():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok, loc_off, send, recv in res:
        assert ok, f"rank {rank}: combined output differs"
    # what rank 0 sends to rank 1 is what rank 1 receives from rank 0, and back
    (_, _, off0, send0, recv0), (_, _, off1, send1, recv1) = res
    assert send0[1] == recv1[0] and send1[0] == recv0[1]
    # every pair of both ranks lands on exactly one expert owner
    assert off0[-1] + off1[-1] == 2 * (37 + 53)


def test_expert_range_and_regroup_index():
    from block_scaled_precision_nvfp4_b200 import ep
    assert [ep.expert_range(8, 4, r) for r in range(4)] == [(0, 2), (2, 4), (4, 6), (6, 8)]
    with pytest.raises(ValueError):
        ep.expert_range(6, 4, 0)
    # received as [source][expert] blocks of sizes [[1, 2], [2, 1]]:
    #   s0: e0 -> row 0, e1 -> rows 1, 2;  s1: e0 -> rows 3, 4, e1 -> row 5
    # regrouped expert-major, sources in order inside an expert
    idx = ep._regroup_index(np.array([[1, 2], [2, 1]]))
    assert idx.tolist() == [0, 3, 4, 1, 2, 5]
    assert ep._regroup_index(np.zeros((2, 3), dtype=np.int64)).size == 0
