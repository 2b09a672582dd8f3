"""The grouped product planned on the device from device-resident expert offsets:
the same bytes as the host-planned entry (same tiles, same alphas), parity with the
oracle, bad offsets reported, and a whole MoE layer captured in one CUDA graph; and
the same product with the top-1 combine fused into its epilogue."""
import numpy as np
import pytest
import torch

import oracle
from oracle import moe as om
import block_scaled_precision_nvfp4_b200 as nv
from block_scaled_precision_nvfp4_b200 import workloads as wl

from parity import bf16_to_f64, check

pytestmark = pytest.mark.gpu


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _random_grouped(counts, N, K, seed):
    rng = np.random.default_rng(seed)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    A = wl.uniform_operand(rng, int(off[-1]), K)
    Ws = [wl.uniform_operand(rng, N, K) for _ in counts]
    Wc = np.stack([w.codes for w in Ws]); Wsc = np.stack([w.scales for w in Ws])
    gW = rng.choice([0.25, 0.5, 1.0, 2.0], len(counts))
    return A, Wc, Wsc, gW, off


COUNTS = [([1, 8, 17, 64, 127, 128], 520, 512), ([0, 130, 0, 1, 256, 300], 264, 256),
          ([127, 128, 129, 383, 384, 385], 136, 768), ([16], 1000, 1024), ([40] * 20, 384, 256),
          ([5, 300, 129, 64], 100, 256), ([0, 0, 0], 256, 256)]


@pytest.mark.parametrize("counts,N,K", COUNTS)
def test_device_schedule_equals_host_plan(counts, N, K):
    A, Wc, Ws, gW, off = _random_grouped(counts, N, K, sum(counts) * 3 + N + K)
    E, M = len(counts), int(off[-1])
    sw = nv.nvfp4_pack_scales_grouped(_dev(Ws.reshape(E * N, K // 16)),
                                      [e * N for e in range(E + 1)], K)
    sched = nv.GroupedSchedule(_dev(off.astype(np.int32)), E, M, N, K, gW, gA=1.5)
    sa_d = sched.pack(_dev(A.scales))
    y_d = sched.gemm(_dev(A.codes), sa_d, _dev(Wc), sw)
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    if M == 0:
        assert y_d.numel() == 0
        return
    sa_h = nv.nvfp4_pack_scales_grouped(_dev(A.scales), list(off), K)
    y_h = nv.gemm_nvfp4_w4a4_grouped_packed(_dev(A.codes), sa_h, 1.5, _dev(Wc), sw, list(gW),
                                            list(off))
    torch.cuda.synchronize()
    n = nv.nvfp4_grouped_scale_layout_bytes(list(off), K)
    assert torch.equal(sa_d[:n], sa_h[:n])
    assert torch.equal(y_d.view(torch.int16), y_h.view(torch.int16))
    ref = oracle.gemm_grouped_w4a4(A.codes, A.scales, 1.5, Wc, Ws, gW, off, N, K)
    check(bf16_to_f64(y_d), ref, f"grouped sched {counts}")


def test_device_gA_equals_host_gA():
    A, Wc, Ws, gW, off = _random_grouped([100, 0, 257], 256, 512, 5)
    E, N, K, M = 3, 256, 512, int(off[-1])
    sw = nv.nvfp4_pack_scales_grouped(_dev(Ws.reshape(E * N, K // 16)),
                                      [e * N for e in range(E + 1)], K)
    ga = torch.tensor([0.375], dtype=torch.float32, device="cuda")
    ys = []
    for g in (ga, 0.375):
        s = nv.GroupedSchedule(_dev(off.astype(np.int32)), E, M, N, K, gW, gA=g)
        ys.append(s.gemm(_dev(A.codes), s.pack(_dev(A.scales)), _dev(Wc), sw))
    torch.cuda.synchronize()
    assert torch.equal(ys[0].view(torch.int16), ys[1].view(torch.int16))


def test_product_right_after_replanning_reads_the_new_schedule():
    """The product is launched programmatically (it may start while the kernel before
    it still runs); when that kernel is the schedule itself, the product must still
    read the schedule only once it is complete.  Re-planning one buffer with new
    offsets and launching the product straight after must give the new plan's result,
    equal to the host-planned product's, every time."""
    E, N, K = 3, 384, 512
    plans = [[300, 5, 200], [10, 480, 15], [0, 0, 505], [256, 1, 248]]
    M = sum(plans[0])
    rng = np.random.default_rng(31)
    A = wl.uniform_operand(rng, M, K)
    Ws = [wl.uniform_operand(rng, N, K) for _ in range(E)]
    Wc = _dev(np.stack([w.codes for w in Ws]))
    gW = [0.5, 1.0, 2.0]
    sw = nv.nvfp4_pack_scales_grouped(_dev(np.stack([w.scales for w in Ws]).reshape(E * N, -1)),
                                      [e * N for e in range(E + 1)], K)
    a_d, s_d = _dev(A.codes), _dev(A.scales)
    offs, packed, expect = [], [], []
    for counts in plans:
        assert sum(counts) == M
        off = [0] + list(np.cumsum(counts))
        offs.append(torch.tensor(off, dtype=torch.int32, device="cuda"))
        sa = nv.nvfp4_pack_scales_grouped(s_d, off, K)
        pad = torch.zeros(nv.load_library().nvfp4_grouped_scale_layout_bytes_bound(M, E, K),
                          dtype=torch.uint8, device="cuda")
        pad[:sa.numel()] = sa
        packed.append(pad)
        expect.append(nv.gemm_nvfp4_w4a4_grouped_packed(a_d, sa, 1.25, Wc, sw, gW, off))
    sched = nv.GroupedSchedule(offs[0], E, M, N, K, gW, gA=1.25)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    for rep in range(6):
        for i in range(len(plans)):
            sched.plan(offs[i], gW, gA=1.25)
            sched.gemm(a_d, packed[i], Wc, sw, out=y)
            torch.cuda.synchronize()
            assert torch.equal(y.view(torch.int16), expect[i].view(torch.int16)), (rep, plans[i])
    nv.nvfp4_check_device_error()


def test_bad_device_offsets_are_reported_and_write_nothing():
    A, Wc, Ws, gW, off = _random_grouped([64, 64], 256, 256, 9)
    E, N, K, M = 2, 256, 256, 128
    sw = nv.nvfp4_pack_scales_grouped(_dev(Ws.reshape(E * N, K // 16)), [0, N, 2 * N], K)
    bad = torch.tensor([0, 100, 90], dtype=torch.int32, device="cuda")   # decreasing, wrong end
    s = nv.GroupedSchedule(bad, E, M, N, K, gW)
    y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    s.gemm(_dev(A.codes), s.pack(_dev(A.scales)), _dev(Wc), sw, out=y)
    with pytest.raises(nv.NvFp4Error) as e:
        nv.nvfp4_check_device_error()
    assert e.value.status == nv.Status.INVALID_ARG
    assert bool((y.float() == 7.0).all())


@pytest.mark.parametrize("fused", [False, True])
def test_whole_moe_layer_in_one_cuda_graph(fused):
    """quantise -> route -> permute -> schedule -> pack -> grouped W4A4 -> combine (a
    separate kernel, or fused into the product's epilogue), captured once and
    replayed, equals the eager layer bit for bit."""
    rng = np.random.default_rng(21)
    T, E, N, K = 700, 4, 384, 512
    x = torch.from_numpy(rng.standard_normal((T, K)).astype(np.float32)).to(torch.bfloat16).cuda()
    ids = torch.from_numpy(rng.integers(0, E, size=(T, 1)).astype(np.int32)).cuda()
    w = torch.ones((T, 1), dtype=torch.float32, device="cuda")
    experts = [wl.quantize_nvfp4(rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02))
               for _ in range(E)]
    Wc = _dev(np.stack([e.codes for e in experts]))
    sw = nv.nvfp4_pack_scales_grouped(_dev(np.stack([e.scales for e in experts]).reshape(E * N, -1)),
                                      [e * N for e in range(E + 1)], K)
    gws = [e.g for e in experts]
    lib = nv.load_library()
    route_ws = torch.empty(lib.nvfp4_moe_route_workspace_bytes(T, E), dtype=torch.uint8, device="cuda")
    q_ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    bufs = dict(codes=torch.empty((T, K // 2), dtype=torch.uint8, device="cuda"),
                scales=torch.empty((T, K // 16), dtype=torch.uint8, device="cuda"),
                g=torch.empty(4, dtype=torch.float32, device="cuda"),
                gc=torch.empty((T, K // 2), dtype=torch.uint8, device="cuda"),
                gs=torch.empty((T, K // 16), dtype=torch.uint8, device="cuda"),
                sa=torch.empty(lib.nvfp4_grouped_scale_layout_bytes_bound(T, E, K), dtype=torch.uint8,
                               device="cuda"),
                yg=torch.empty((T, N), dtype=torch.bfloat16, device="cuda"),
                y=torch.empty((T, N), dtype=torch.bfloat16, device="cuda"))

    def layer(s):
        b = bufs
        nv.nvfp4_quantize_bf16(x, plain=True, packed=False, workspace=q_ws, stream=s,
                               out=(b["codes"], b["scales"], None, b["g"]))
        off, dest, src = nv.moe_route(ids, E, workspace=route_ws, stream=s)
        nv.moe_permute_rows(b["codes"], src, 1, out=b["gc"], stream=s)
        nv.moe_permute_rows(b["scales"], src, 1, out=b["gs"], stream=s)
        sched = nv.GroupedSchedule(off, E, T, N, K, gws, gA=b["g"][:1], stream=s)
        sched.pack(b["gs"], out=b["sa"], stream=s)
        if fused:
            sched.gemm_combine(b["gc"], b["sa"], Wc, sw, src, T, weights=w, out=b["y"], stream=s)
        else:
            sched.gemm(b["gc"], b["sa"], Wc, sw, out=b["yg"], stream=s)
            nv.moe_combine(b["yg"], dest, w, T, 1, out=b["y"], stream=s)
        return sched, off, dest, src

    cur = torch.cuda.current_stream()
    keep = layer(cur)
    torch.cuda.synchronize()
    eager = bufs["y"].clone()
    bufs["y"].zero_()
    s = torch.cuda.Stream()
    s.wait_stream(cur)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        keep2 = layer(s)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    assert torch.equal(bufs["y"].view(torch.int16), eager.view(torch.int16))
    del g


def _top1_layer(counts, N, K, seed):
    """Tokens routed top-1 to experts with the given token counts, in a shuffled token
    order; returns the inputs and the routed, permuted, packed state of the layer."""
    rng = np.random.default_rng(seed)
    E, T = len(counts), int(sum(counts))
    ids = rng.permutation(np.repeat(np.arange(E, dtype=np.int32), counts)).reshape(T, 1)
    A = wl.uniform_operand(rng, T, K)
    Ws = [wl.uniform_operand(rng, N, K) for _ in counts]
    Wc = np.stack([w.codes for w in Ws]); Wsc = np.stack([w.scales for w in Ws])
    gW = rng.choice([0.25, 0.5, 1.0, 2.0], E)
    w = rng.random(T).astype(np.float32) + np.float32(0.5)
    off, dest, src = nv.moe_route(_dev(ids), E)
    gc = nv.moe_permute_rows(_dev(A.codes), src, 1)
    gs = nv.moe_permute_rows(_dev(A.scales), src, 1)
    sw = nv.nvfp4_pack_scales_grouped(_dev(Wsc.reshape(E * N, K // 16)),
                                      [e * N for e in range(E + 1)], K)
    sched = nv.GroupedSchedule(off, E, T, N, K, gW, gA=1.5)
    sa = sched.pack(gs)
    return dict(E=E, T=T, ids=ids, A=A, Wc=Wc, Wsc=Wsc, gW=gW, w=w, off=off, dest=dest, src=src,
                gc=gc, gs=gs, sw=sw, sched=sched, sa=sa, Wc_d=_dev(Wc))


FUSED = [([300, 129, 0, 1, 256, 14], 264, 512), ([700], 512, 256), ([5, 60, 127, 128, 3], 256, 768),
         ([40] * 9, 136, 256)]


@pytest.mark.parametrize("counts,N,K", FUSED)
def test_fused_top1_combine_against_the_oracle(counts, N, K):
    """Y[t] = BF16(w[t] * alpha_e * sum_k ...) for each token t routed to expert e, rounded
    once, against the oracle's grouped product and combine in FP64."""
    L = _top1_layer(counts, N, K, sum(counts) + N)
    y = L["sched"].gemm_combine(L["gc"], L["sa"], L["Wc_d"], L["sw"], L["src"], L["T"],
                                weights=_dev(L["w"]))
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    ro, rd, rs = om.route(L["ids"], L["E"])
    g = om.permute_rows(L["A"].codes, rs, 1), om.permute_rows(L["A"].scales, rs, 1)
    Yg = oracle.gemm_grouped_w4a4(g[0], g[1], 1.5, L["Wc"], L["Wsc"], L["gW"], ro, N, K)
    ref = om.combine(Yg, rd, L["w"].reshape(-1, 1), L["T"], 1)
    check(bf16_to_f64(y), ref, f"fused combine {counts}")


@pytest.mark.parametrize("counts,N,K", FUSED[:2])
def test_fused_top1_combine_against_the_unfused_layer(counts, N, K):
    L = _top1_layer(counts, N, K, 3 * sum(counts) + K)
    s = L["sched"]
    yg = s.gemm(L["gc"], L["sa"], L["Wc_d"], L["sw"])
    # without weights the fused epilogue writes the unfused rows, permuted: same bits
    y1 = s.gemm_combine(L["gc"], L["sa"], L["Wc_d"], L["sw"], L["src"], L["T"])
    y0 = nv.moe_combine(yg, L["dest"], None, L["T"], 1)
    # with weights the unfused path rounds twice, the fused one once
    wd = _dev(L["w"])
    y2 = s.gemm_combine(L["gc"], L["sa"], L["Wc_d"], L["sw"], L["src"], L["T"], weights=wd)
    y3 = nv.moe_combine(yg, L["dest"], wd.reshape(-1, 1), L["T"], 1)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y0.view(torch.int16))
    a, b = bf16_to_f64(y2), bf16_to_f64(y3)
    assert np.all(np.abs(a - b) <= 2.0 ** -7 * np.maximum(np.abs(a), np.abs(b)))


def test_fused_combine_reports_a_bad_destination_and_skips_it():
    L = _top1_layer([100, 28], 256, 256, 77)
    T = L["T"]
    src = L["src"].clone()
    victim = int(src[5].item())
    src[5] = T                                                    # outside [0, T)
    y = torch.full((T, 256), 3.0, dtype=torch.bfloat16, device="cuda")
    L["sched"].gemm_combine(L["gc"], L["sa"], L["Wc_d"], L["sw"], src, T, out=y)
    with pytest.raises(nv.NvFp4Error) as e:
        nv.nvfp4_check_device_error()
    assert e.value.status == nv.Status.INVALID_ARG
    assert bool((y[victim].float() == 3.0).all())                 # that token's row is not written
    others = [int(t) for t in L["src"].tolist() if int(t) != victim]
    assert not bool((y[others].float() == 3.0).all())


@pytest.mark.parametrize("counts,N,K", COUNTS[:5])
def test_plain_scale_entry_with_device_offsets(counts, N, K):
    """gemm_nvfp4_w4a4_grouped: plain scales, device offsets and one caller workspace
    (its size from nvfp4_workspace_size); equal to the host-planned packed product
    bit for bit, and within tolerance of the oracle."""
    A, Wc, Ws, gW, off = _random_grouped(counts, N, K, sum(counts) * 7 + N)
    E, M = len(counts), int(off[-1])
    need = nv.nvfp4_workspace_size(nv.Op.W4A4_GROUPED, M, N, K, E)
    ws = torch.full((need,), 0xAB, dtype=torch.uint8, device="cuda")   # needs no zeroing
    off_d = _dev(off.astype(np.int32))
    y = nv.gemm_nvfp4_w4a4_grouped(_dev(A.codes), _dev(A.scales), 0.75, _dev(Wc), _dev(Ws), gW,
                                   off_d, workspace=ws)
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    if M == 0:
        return
    sw = nv.nvfp4_pack_scales_grouped(_dev(Ws.reshape(E * N, K // 16)),
                                      [e * N for e in range(E + 1)], K)
    sa = nv.nvfp4_pack_scales_grouped(_dev(A.scales), list(off), K)
    y_h = nv.gemm_nvfp4_w4a4_grouped_packed(_dev(A.codes), sa, 0.75, _dev(Wc), sw, list(gW),
                                            list(off))
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_h.view(torch.int16))
    ref = oracle.gemm_grouped_w4a4(A.codes, A.scales, 0.75, Wc, Ws, gW, off, N, K)
    check(bf16_to_f64(y), ref, f"grouped device offsets {counts}")
