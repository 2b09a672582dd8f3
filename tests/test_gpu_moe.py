"""MoE route / permute / combine on the GPU against the oracle's MoE steps, through
the C ABI; then one whole MoE layer (quantise, route, permute, pack, grouped W4A4,
combine) against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from oracle import moe as om
import block_scaled_precision_nvfp4_b200 as nv
from block_scaled_precision_nvfp4_b200 import workloads as wl

from parity import bf16_to_f64, check

pytestmark = pytest.mark.gpu


def _ids(rng, T, k, E, zipf=None):
    if zipf is None:
        return rng.integers(0, E, size=(T, k)).astype(np.int32)
    p = (np.arange(E) + 1.0) ** -zipf
    return rng.choice(E, size=(T, k), p=p / p.sum()).astype(np.int32)


# up to 65536 pairs one CTA routes; beyond that, chunked histograms, a scan and ranks
CASES = [(1, 1, 1, None), (7, 1, 4, None), (1000, 2, 64, None), (8192, 1, 8, 1.1),
         (5000, 4, 256, None), (3000, 2, 16, 2.5), (2049, 3, 5, None), (16384, 4, 8, None),
         (40000, 2, 32, 1.1), (70001, 1, 256, None)]


@pytest.mark.parametrize("T,k,E,zipf", CASES)
def test_route_bit_exact(T, k, E, zipf):
    rng = np.random.default_rng(T * 31 + k * 7 + E)
    ids = _ids(rng, T, k, E, zipf)
    off, dest, src = nv.moe_route(torch.from_numpy(ids).cuda(), E)
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    ro, rd, rs = om.route(ids, E)
    assert np.array_equal(off.cpu().numpy(), ro)
    assert np.array_equal(dest.cpu().numpy(), rd)
    assert np.array_equal(src.cpu().numpy(), rs)


def test_route_empty_and_unused_experts():
    off, dest, src = nv.moe_route(torch.empty((0, 2), dtype=torch.int32, device="cuda"), 6)
    torch.cuda.synchronize()
    assert off.cpu().tolist() == [0] * 7 and dest.numel() == 0
    ids = np.array([[5, 5], [0, 5], [5, 0]], np.int32)      # experts 1-4 get nothing
    off, dest, src = nv.moe_route(torch.from_numpy(ids).cuda(), 6)
    ro, rd, rs = om.route(ids, 6)
    assert np.array_equal(off.cpu().numpy(), ro) and np.array_equal(dest.cpu().numpy(), rd)


@pytest.mark.parametrize("big", [False, True])
def test_route_bad_id_is_reported_and_left_out(big):
    ids = np.array([0, 3, 9, 1, -2, 3], np.int32)
    if big:   # past the one-CTA size
        ids = np.concatenate([np.random.default_rng(0).integers(0, 4, 70000).astype(np.int32), ids])
    off, dest, src = nv.moe_route(torch.from_numpy(ids).cuda(), 4)
    with pytest.raises(nv.NvFp4Error) as e:
        nv.nvfp4_check_device_error()
    assert e.value.status == nv.Status.INVALID_ARG
    nv.nvfp4_check_device_error()                            # the record was cleared
    ro, rd, rs = om.route(ids, 4)
    assert np.array_equal(off.cpu().numpy(), ro) and np.array_equal(dest.cpu().numpy(), rd)
    assert np.array_equal(src.cpu().numpy(), rs)


@pytest.mark.parametrize("T,k,E,row_bytes", [(300, 2, 8, 7168), (1000, 1, 64, 896),
                                             (17, 4, 3, 16), (4096, 2, 8, 2048)])
def test_permute_rows_bit_exact(T, k, E, row_bytes):
    rng = np.random.default_rng(T + row_bytes)
    ids = _ids(rng, T, k, E)
    x = rng.integers(0, 256, size=(T, row_bytes), dtype=np.uint8)
    off, dest, src = nv.moe_route(torch.from_numpy(ids).cuda(), E)
    g = nv.moe_permute_rows(torch.from_numpy(x).cuda(), src, k)
    torch.cuda.synchronize()
    ro, rd, rs = om.route(ids, E)
    assert np.array_equal(g.cpu().numpy(), om.permute_rows(x, rs, k))


@pytest.mark.parametrize("T,k,N,weighted", [(100, 1, 64, False), (257, 2, 5376, True),
                                            (33, 4, 14336, True), (1, 8, 8, True)])
def test_combine(T, k, N, weighted):
    rng = np.random.default_rng(T * k + N)
    E = 8
    ids = _ids(rng, T, k, E)
    off, dest, src = nv.moe_route(torch.from_numpy(ids).cuda(), E)
    Yg = torch.from_numpy(rng.standard_normal((T * k, N)).astype(np.float32)).to(torch.bfloat16).cuda()
    w = rng.random((T, k)).astype(np.float32) if weighted else None
    Y = nv.moe_combine(Yg, dest, None if w is None else torch.from_numpy(w).cuda(), T, k)
    torch.cuda.synchronize()
    ref = om.combine(bf16_to_f64(Yg), om.route(ids, E)[1], w, T, k)
    if not weighted and k == 1:
        assert np.array_equal(bf16_to_f64(Y), ref)           # a copy: exact
    else:
        check(bf16_to_f64(Y), ref, f"combine T{T} k{k} N{N}")


def test_whole_moe_layer_against_the_oracle():
    """BF16 tokens -> GPU quantiser -> route -> permute codes and scales -> grouped
    packing -> grouped W4A4 -> weighted combine, against the oracle's grouped product
    of the same permuted bytes and its combine."""
    rng = np.random.default_rng(7)
    T, k, E, N, K = 600, 2, 8, 512, 1024
    x = rng.standard_normal((T, K)).astype(np.float32)
    ids = _ids(rng, T, k, E, zipf=1.1)
    w = rng.random((T, k)).astype(np.float32)
    experts = [wl.quantize_nvfp4(rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02))
               for _ in range(E)]
    xd = torch.from_numpy(x).to(torch.bfloat16).cuda()
    codes, scales, _, g = nv.nvfp4_quantize_bf16(xd, plain=True, packed=False)
    off, dest, src = nv.moe_route(torch.from_numpy(ids).cuda(), E)
    gc = nv.moe_permute_rows(codes, src, k)
    gs = nv.moe_permute_rows(scales, src, k)
    offsets = off.cpu().tolist()                            # the grouped GEMM plans on the host
    sa_p = nv.nvfp4_pack_scales_grouped(gs, offsets, K)
    Wc = torch.from_numpy(np.stack([e.codes for e in experts])).cuda()
    Ws = torch.from_numpy(np.stack([e.scales for e in experts])).cuda()
    sw_p = nv.nvfp4_pack_scales_grouped(Ws.view(E * N, K // 16), [i * N for i in range(E + 1)], K)
    gA = float(g.cpu()[0])
    Yg = nv.gemm_nvfp4_w4a4_grouped_packed(gc, sa_p, gA, Wc, sw_p, [e.g for e in experts], offsets)
    Y = nv.moe_combine(Yg, dest, torch.from_numpy(w).cuda(), T, k)
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    # oracle: the same permuted bytes through the grouped definition, then its combine
    ro, rd, rs = om.route(ids, E)
    assert np.array_equal(gc.cpu().numpy(), om.permute_rows(codes.cpu().numpy(), rs, k))
    Yg_ref = oracle.gemm_grouped_w4a4(gc.cpu().numpy(), gs.cpu().numpy(), gA, Wc.cpu().numpy(),
                                      Ws.cpu().numpy(), np.array([e.g for e in experts]), ro, N, K)
    check(bf16_to_f64(Yg), Yg_ref, "moe grouped product")
    # the combine step alone: one BF16 rounding of the weighted sum of the GPU's Yg
    check(bf16_to_f64(Y), om.combine(bf16_to_f64(Yg), rd, w, T, k), "moe combine")
    # end to end against FP64 throughout: the layer rounds to BF16 twice (the grouped
    # product's output, then the combine), each worth ~1.5e-3 relative Frobenius, so
    # the bar is the single-rounding 2e-3 scaled by sqrt(2)
    ref = om.combine(Yg_ref, rd, w, T, k)
    rel = np.linalg.norm(bf16_to_f64(Y) - ref) / np.linalg.norm(ref)
    assert rel <= 2e-3 * np.sqrt(2), f"moe layer: relative Frobenius error {rel:.3e}"
    assert np.max(np.abs(bf16_to_f64(Y) - ref)) <= 1e-2 * np.max(np.abs(ref))


def test_expert_parallel_path_on_one_rank_equals_the_direct_layer():
    """ep.dispatch / ep.combine with the CUDA kernels and no process group (one rank
    owning every expert) give the direct layer's output bit for bit."""
    from block_scaled_precision_nvfp4_b200 import ep
    rng = np.random.default_rng(11)
    T, k, E, N, K = 300, 2, 4, 256, 512
    ids = _ids(rng, T, k, E)
    w = torch.from_numpy(rng.random((T, k)).astype(np.float32)).cuda()
    A = wl.quantize_nvfp4(rng.standard_normal((T, K), dtype=np.float32))
    experts = [wl.quantize_nvfp4(rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02))
               for _ in range(E)]
    Wc = torch.from_numpy(np.stack([e.codes for e in experts])).cuda()
    Ws = torch.from_numpy(np.stack([e.scales for e in experts])).cuda()
    gws = [e.g for e in experts]

    def grouped(codes, scales, offsets):
        return nv.gemm_nvfp4_w4a4_grouped(codes, scales, A.g, Wc, Ws, gws, offsets)

    codes, scales = torch.from_numpy(A.codes).cuda(), torch.from_numpy(A.scales).cuda()
    idd = torch.from_numpy(ids).cuda()
    st = ep.dispatch(codes, scales, idd, E)
    Y1 = ep.combine(grouped(st.codes, st.scales, st.local_offsets), st, w)
    off, dest, src = nv.moe_route(idd, E)
    gc, gs = nv.moe_permute_rows(codes, src, k), nv.moe_permute_rows(scales, src, k)
    Y2 = nv.moe_combine(grouped(gc, gs, off.cpu().tolist()), dest, w, T, k)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
