"""The C-ABI library: loads, exports every declared symbol, plans and rejects (CPU only)."""
import ctypes
import os
import re

import pytest

import block_scaled_precision_nvfp4_b200 as nv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"^NVFP4_API\s+[\w\s\*]+?\b(\w+)\(", src, flags=re.M)
    return names


def test_library_exports_every_declared_symbol():
    lib = nv.load_library()
    names = declared_functions()
    assert len(names) >= 16
    for name in names:
        assert hasattr(lib, name), name
        assert name in nv.C_FUNCTIONS, f"{name} has no binding"
    assert set(nv.C_FUNCTIONS) == set(names)


def test_library_is_sm100a_only_and_has_no_cpu_symbols():
    # the product library carries no oracle code
    lib = nv.load_library()
    for bad in ("oracle_gemm_w4a4", "oracle_e2m1_value"):
        with pytest.raises(AttributeError):
            getattr(lib, bad)


def test_kind_of():
    assert nv.nvfp4_kind_of(nv.Fmt.BF16) == nv.Kind.BF16_MMA
    assert nv.nvfp4_kind_of(nv.Fmt.FP8_E4M3) == nv.Kind.FP8_MMA
    assert nv.nvfp4_kind_of(nv.Fmt.NVFP4) == nv.Kind.FP4_BLOCK_SCALED
    assert nv.load_library().nvfp4_kind_of(7) == -1


def test_pair_name():
    F = nv.Fmt
    assert nv.nvfp4_pair_name(F.NVFP4, F.NVFP4) == "W4A4"
    assert nv.nvfp4_pair_name(F.NVFP4, F.BF16) == "W4A16"
    assert nv.nvfp4_pair_name(F.NVFP4, F.FP8_E4M3) == "W4A8"
    assert nv.nvfp4_pair_name(F.BF16, F.BF16) == "W16A16"
    assert nv.load_library().nvfp4_pair_name(9, 0) == b"?"


@pytest.mark.parametrize("arch,expect", [
    (100, "FP4_MMA"), (103, "NO_FP4_KERNEL"), (120, "NO_FP4_KERNEL"), (90, "NO_PATH"),
    (89, "NO_PATH"), (80, "NO_PATH")])
def test_exec_of_w4a4_by_class(arch, expect):
    assert nv.nvfp4_exec_of_arch(arch, nv.Fmt.NVFP4, nv.Fmt.NVFP4).name == expect


def test_exec_of_other_pairs():
    F, E = nv.Fmt, nv.Exec
    assert nv.nvfp4_exec_of_arch(100, F.NVFP4, F.BF16) == E.BF16_WIDEN
    assert nv.nvfp4_exec_of_arch(90, F.NVFP4, F.BF16) == E.NO_PATH
    # W4A8: no single-instruction MMA; the exact E4M3 path where its kernel is compiled
    # (sm_100), no path elsewhere, never widened to BF16
    assert nv.nvfp4_exec_of_arch(100, F.NVFP4, F.FP8_E4M3) == E.FP8_EXACT
    for arch in (89, 90, 103, 120, 80):
        assert nv.nvfp4_exec_of_arch(arch, F.NVFP4, F.FP8_E4M3) == E.NO_PATH
    # the FP4-kernel switch concerns the FP4 MMA only
    assert nv.nvfp4_exec_of_arch(100, F.NVFP4, F.FP8_E4M3, fp4_kernel_disabled=True) == E.FP8_EXACT
    for w in (F.BF16, F.FP8_E4M3):
        for a in F:
            assert nv.nvfp4_exec_of_arch(100, w, a) == E.NO_PATH


def test_kernel_missing_flag_is_no_fp4_kernel_not_an_upcast():
    E, F = nv.Exec, nv.Fmt
    assert nv.nvfp4_exec_of_arch(100, F.NVFP4, F.NVFP4, fp4_kernel_disabled=True) \
        == E.NO_FP4_KERNEL
    # the activation format is never re-planned at a wider format
    assert nv.nvfp4_exec_of_arch(90, F.NVFP4, F.NVFP4) != E.BF16_WIDEN


def test_exec_of_without_device_is_no_path():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    assert nv.nvfp4_exec_of(0, nv.Fmt.NVFP4, nv.Fmt.NVFP4) == nv.Exec.NO_PATH


def _call_w4a4(lib, A=16, sA=16, W=16, sW=16, Y=16, M=4, N=4, K=64, name="gemm_nvfp4_w4a4"):
    return getattr(lib, name)(A, sA, 1.0, W, sW, 1.0, Y, M, N, K, None)


@pytest.mark.parametrize("name", ["gemm_nvfp4_w4a4", "gemm_nvfp4_via_fp8"])
def test_argument_errors_need_no_device(name):
    lib = nv.load_library()
    assert _call_w4a4(lib, M=-1, name=name) == nv.Status.INVALID_ARG
    assert _call_w4a4(lib, K=48, name=name) == nv.Status.INVALID_ARG
    assert _call_w4a4(lib, K=0, name=name) == nv.Status.INVALID_ARG
    assert _call_w4a4(lib, A=0, name=name) == nv.Status.INVALID_ARG
    assert _call_w4a4(lib, A=17, name=name) == nv.Status.MISALIGNED
    assert _call_w4a4(lib, Y=24, name=name) == nv.Status.MISALIGNED
    assert b"16-byte" in lib.nvfp4_last_error()


def test_grouped_argument_errors_need_no_device():
    lib = nv.load_library()
    gws = (ctypes.c_float * 3)(1.0, 1.0, 1.0)
    def call(offs, E=2, K=256, N=64, A=16):
        o = (ctypes.c_int32 * len(offs))(*offs)
        return lib.gemm_nvfp4_w4a4_grouped_host(A, 16, 1.0, 16, 16,
                                                ctypes.cast(gws, ctypes.c_void_p),
                                                ctypes.cast(o, ctypes.c_void_p), E, 16, N, K, None)
    assert call([0, 6, 5]) == nv.Status.INVALID_ARG          # decreasing
    assert call([1, 6, 8]) == nv.Status.INVALID_ARG          # offsets[0] != 0
    assert call([0, 0], E=0) == nv.Status.INVALID_ARG        # no experts
    assert call([0] * 3, E=300) == nv.Status.INVALID_ARG     # too many experts
    assert call([0, 4, 8], K=96) == nv.Status.INVALID_ARG    # K % 32
    assert call([0, 4, 8], A=24) == nv.Status.MISALIGNED


def test_grouped_packed_argument_errors_need_no_device():
    lib = nv.load_library()
    gws = (ctypes.c_float * 3)(1.0, 1.0, 1.0)
    def call(offs, E=2, K=256, N=64, A=16):
        o = (ctypes.c_int32 * len(offs))(*offs)
        return lib.gemm_nvfp4_w4a4_grouped_packed(A, 16, 1.0, 16, 16,
                                                  ctypes.cast(gws, ctypes.c_void_p),
                                                  ctypes.cast(o, ctypes.c_void_p), E, 16, N, K, None)
    assert call([0, 6, 5]) == nv.Status.INVALID_ARG          # decreasing
    assert call([1, 6, 8]) == nv.Status.INVALID_ARG          # offsets[0] != 0
    assert call([0, 0], E=0) == nv.Status.INVALID_ARG        # no experts
    assert call([0] * 3, E=300) == nv.Status.INVALID_ARG     # too many experts
    assert call([0, 4, 8], K=96) == nv.Status.INVALID_ARG    # K % 32
    assert call([0, 4, 8], A=24) == nv.Status.MISALIGNED


def test_grouped_scale_layout_bytes_is_per_group_blocks():
    # every group starts on a 128-row block: sum of ceil(rows/128) blocks of 128 * K/16 bytes
    assert nv.nvfp4_grouped_scale_layout_bytes([0, 1], 64) == 128 * 4
    assert nv.nvfp4_grouped_scale_layout_bytes([0, 1, 1, 129, 385], 256) == (1 + 0 + 1 + 2) * 128 * 16
    assert nv.nvfp4_grouped_scale_layout_bytes([0, 3278, 4751], 4096) == (26 + 12) * 128 * 256
    E, N = 8, 14336
    assert (nv.nvfp4_grouped_scale_layout_bytes([e * N for e in range(E + 1)], 4096)
            == E * nv.nvfp4_scale_layout_bytes(N, 4096))
    assert nv.nvfp4_grouped_scale_layout_bytes([0, 5], 96) == 0      # K % 64
    assert nv.nvfp4_grouped_scale_layout_bytes([0, 5, 4], 64) == 0   # decreasing
    assert nv.nvfp4_grouped_scale_layout_bytes([2, 5], 64) == 0      # offsets[0] != 0


def test_grouped_pack_argument_errors_need_no_device():
    lib = nv.load_library()
    def call(offs, E, K=256, s=16):
        o = (ctypes.c_int32 * len(offs))(*offs)
        return lib.nvfp4_pack_scales_grouped(s, ctypes.cast(o, ctypes.c_void_p), E, K, 16, None)
    assert call([0, 4, 2], 2) == nv.Status.INVALID_ARG
    assert call([0, 4], 1, K=96) == nv.Status.INVALID_ARG
    assert call([0, 4], 1, s=8) == nv.Status.MISALIGNED
    assert call([0, 0, 0], 2) == nv.Status.OK                 # nothing to pack


def test_w4a8_argument_errors_need_no_device():
    lib = nv.load_library()
    def call(A=16, W=16, sW=16, Y=16, M=4, N=4, K=256):
        return lib.gemm_nvfp4_w4a8(A, 1.0, W, sW, 1.0, Y, M, N, K, None)
    assert call(M=-1) == nv.Status.INVALID_ARG
    assert call(K=128) == nv.Status.INVALID_ARG      # K % 256
    assert call(K=384) == nv.Status.INVALID_ARG
    assert call(K=0) == nv.Status.INVALID_ARG
    assert call(A=0) == nv.Status.INVALID_ARG
    assert call(sW=40) == nv.Status.MISALIGNED
    assert call(Y=8) == nv.Status.MISALIGNED


@pytest.mark.parametrize("arch,expect", [
    (100, "NO_FP4_KERNEL"), (103, "NO_FP4_KERNEL"), (120, "NO_FP4_KERNEL"), (90, "NO_PATH"),
    (89, "NO_PATH"), (80, "NO_PATH")])
def test_fp4_fallback_by_class(arch, expect):
    # a class with the FP4 MMA lacks only the kernel; other classes would need this
    # library's exact-path kernel, which is compiled for sm_100 only
    assert nv.nvfp4_fp4_fallback(arch).name == expect


ALL_PAIRS = [(w, a) for w in nv.Fmt for a in nv.Fmt]


@pytest.mark.parametrize("arch", [100, 103, 120, 90, 89, 80])
@pytest.mark.parametrize("disabled", [False, True])
def test_node_exec_is_exec_of_per_node(arch, disabled):
    nodes = ALL_PAIRS * 2
    got = nv.nvfp4_node_exec(arch, nodes, fp4_kernel_disabled=disabled)
    assert got == [nv.nvfp4_exec_of_arch(arch, w, a, disabled) for w, a in nodes]


def test_node_exec_without_fp4_kernel_takes_fp4_fallback():
    F, E = nv.Fmt, nv.Exec
    nodes = [(F.NVFP4, F.NVFP4), (F.NVFP4, F.FP8_E4M3), (F.NVFP4, F.BF16), (F.FP8_E4M3, F.FP8_E4M3)]
    assert nv.nvfp4_node_exec(100, nodes) == [E.FP4_MMA, E.FP8_EXACT, E.BF16_WIDEN, E.NO_PATH]
    assert nv.nvfp4_node_exec(100, nodes, fp4_kernel_disabled=True) == [
        nv.nvfp4_fp4_fallback(100), E.FP8_EXACT, E.BF16_WIDEN, E.NO_PATH]


def test_node_exec_never_plans_a_wider_format():
    F, E = nv.Fmt, nv.Exec
    for arch in (100, 101, 103, 110, 120, 121, 90, 89, 80, 75):
        for disabled in (False, True):
            for (w, a), e in zip(ALL_PAIRS, nv.nvfp4_node_exec(arch, ALL_PAIRS, disabled)):
                if e == E.FP4_MMA:
                    assert a == F.NVFP4 and w == F.NVFP4
                if e == E.FP8_EXACT:
                    assert w == F.NVFP4 and a in (F.NVFP4, F.FP8_E4M3)
                if e == E.BF16_WIDEN:
                    assert a == F.BF16


def test_node_exec_bad_formats_and_arguments():
    lib = nv.load_library()
    w = (ctypes.c_int32 * 3)(2, 7, -1)
    a = (ctypes.c_int32 * 3)(2, 2, 2)
    out = (ctypes.c_int32 * 3)(-9, -9, -9)
    assert lib.nvfp4_node_exec(100, 0, w, a, 3, out) == nv.Status.OK
    assert list(out) == [nv.Exec.FP4_MMA, nv.Exec.NO_PATH, nv.Exec.NO_PATH]
    assert lib.nvfp4_node_exec(100, 0, w, a, -1, out) == nv.Status.INVALID_ARG
    assert lib.nvfp4_node_exec(100, 0, None, a, 3, out) == nv.Status.INVALID_ARG
    assert lib.nvfp4_node_exec(100, 0, None, None, 0, None) == nv.Status.OK
    assert nv.nvfp4_node_exec(100, []) == []


def test_stream_k_workspace_plan_needs_no_device():
    """The pair kernel's tile balance plan (pure host arithmetic): a workspace only
    when the last wave of 256 x 256 tiles would be at most 60 % full, 512 KB per pair
    boundary plus 64 bytes of tickets each (rounded up to 256)."""
    lib = nv.load_library()
    f = lib.nvfp4_w4a4_packed_workspace_bytes_for

    def need(pairs):
        slots = pairs - 1
        return (slots * 64 + 255) // 256 * 256 + slots * 2 * 2 * 8 * 32 * 128 * 4

    # FFN down on 148 SMs: 336 tiles on 74 pairs, last wave 40/74 = 54 % full -> cut
    assert f(4096, 5376, 14336, 0, 148) == need(74) == 38277888
    # 6144 x 5376: 504 tiles, last wave 60/74 = 81 % full -> whole tiles
    assert f(6144, 5376, 14336, 0, 148) == 0
    # whole waves: 296 tiles on 74 pairs
    assert f(2048, 9472, 14336, 0, 148) == 0
    # fewer tiles than pairs: no full wave to balance against
    assert f(1024, 1024, 14336, 0, 148) == 0
    # a single K-block cannot be cut
    assert f(4096, 5376, 256, 0, 148) == 0
    # max_pairs caps the pairs: 12 tiles on 5 pairs (last wave 40 %), on 7 (71 %)
    assert f(768, 1024, 1024, 5, 148) == need(5)
    assert f(768, 1024, 1024, 7, 148) == 0
    # the threshold is inclusive: 8 tiles on 5 pairs leave a 60 % full last wave
    assert f(512, 1024, 1024, 5, 148) == need(5)
    # fewer SMs, fewer pairs
    assert f(4096, 5376, 14336, 0, 132) == need(66)     # 336 on 66: 6/66 full
    # degenerate arguments
    for args in [(0, 5376, 14336, 0, 148), (4096, 0, 14336, 0, 148), (4096, 5376, 0, 0, 148),
                 (4096, 5376, 14336, -1, 148), (4096, 5376, 14336, 0, 1)]:
        assert f(*args) == 0
    # without a device the device query gives 0
    assert lib.nvfp4_w4a4_packed_workspace_bytes(4096, 5376, 14336, 0) == 0 or \
        __import__("torch").cuda.is_available()


def test_balanced_w4a4_argument_errors_need_no_device():
    lib = nv.load_library()

    def call(A=16, M=512, N=512, K=1024, max_pairs=0, ws=None, nws=0):
        return lib.gemm_nvfp4_w4a4_packed_ws(A, 16, 1.0, 16, 16, 1.0, 16, M, N, K, max_pairs, ws,
                                             nws, None)
    assert call(max_pairs=-1) == nv.Status.INVALID_ARG
    assert call(M=-1) == nv.Status.INVALID_ARG
    assert call(K=320) == nv.Status.INVALID_ARG              # the pair kernel needs K % 256
    assert call(A=0) == nv.Status.INVALID_ARG
    assert call(A=24) == nv.Status.MISALIGNED


def test_fused_combine_argument_errors_need_no_device():
    lib = nv.load_library()

    def call(E=2, M=64, src=16, T=64, N=256, K=256):
        return lib.gemm_nvfp4_w4a4_grouped_packed_sched_combine(16, 16, 16, 16, 16, E, M, src, None,
                                                                16, T, N, K, None)
    assert call(src=None) == nv.Status.INVALID_ARG           # rows but no destinations
    assert call(M=65) == nv.Status.INVALID_ARG               # top-1: at most one row per token
    assert call(T=-1) == nv.Status.INVALID_ARG
    assert call(N=255) == nv.Status.INVALID_ARG              # rows leave as 4-byte pairs
    assert call(E=0) == nv.Status.INVALID_ARG
    assert call(K=320) == nv.Status.INVALID_ARG


# The boundary's generic names: every call the hot-path scope lists exists under its
# own name, with its own argument order.
BOUNDARY_NAMES = ["nvfp4_exec_of", "nvfp4_pair_name", "gemm_nvfp4_w4a4", "gemm_nvfp4_via_fp8",
                  "gemm_w4a16", "gemm_nvfp4_w4a4_grouped", "nvfp4_workspace_size",
                  "nvfp4_prepare_scales", "nvfp4_last_error", "nvfp4_check_device_error"]


def test_boundary_names_are_exported():
    lib = nv.load_library()
    declared = set(declared_functions())
    for name in BOUNDARY_NAMES:
        assert name in declared, name
        assert hasattr(lib, name), name


def test_workspace_size_per_op():
    lib = nv.load_library()
    Op = nv.Op
    for op in (Op.W4A4, Op.VIA_FP8, Op.W4A16, Op.W4A8):
        assert lib.nvfp4_workspace_size(int(op), 4096, 5376, 14336, 1) == 0
    assert lib.nvfp4_workspace_size(int(Op.QUANTIZE), 4096, 0, 14336, 1) == \
        lib.nvfp4_quantize_workspace_bytes()
    assert lib.nvfp4_workspace_size(int(Op.MOE_ROUTE), 8192, 0, 0, 8) == \
        lib.nvfp4_moe_route_workspace_bytes(8192, 8)
    # grouped: the schedule, the packed activation scales (their bound) and the
    # experts' packed weight scales, each rounded up to 256 bytes
    M, N, K, E = 8192, 14336, 4096, 8
    r = lambda b: (b + 255) // 256 * 256
    expect = (r(lib.nvfp4_grouped_sched_bytes()) + r(lib.nvfp4_grouped_scale_layout_bytes_bound(M, E, K))
              + r(E * ((N + 127) // 128) * 128 * (K // 16)))
    assert lib.nvfp4_workspace_size(int(Op.W4A4_GROUPED), M, N, K, E) == expect
    assert lib.nvfp4_workspace_size(int(Op.W4A4_GROUPED), M, N, 4000, E) == 0   # K % 256
    assert lib.nvfp4_workspace_size(int(Op.W4A4_GROUPED), M, N, K, 0) == 0      # no experts
    assert lib.nvfp4_workspace_size(99, 1, 1, 64, 1) == 2 ** 64 - 1             # unknown op
    import torch
    if not torch.cuda.is_available():
        assert lib.nvfp4_workspace_size(int(Op.W4A4_PACKED), 4096, 5376, 14336, 1) == 0


def test_device_offset_grouped_argument_errors_need_no_device():
    lib = nv.load_library()
    gws = (ctypes.c_float * 2)(1.0, 1.0)
    need = lib.nvfp4_workspace_size(int(nv.Op.W4A4_GROUPED), 64, 256, 256, 2)
    assert need > 0

    def call(E=2, M=64, N=256, K=256, A=16, off=16, ws=4096, ws_bytes=None):
        return lib.gemm_nvfp4_w4a4_grouped(A, 16, 1.0, 16, 16, ctypes.cast(gws, ctypes.c_void_p),
                                           off, E, M, 16, N, K, ws,
                                           need if ws_bytes is None else ws_bytes, None)
    assert call(E=0) == nv.Status.INVALID_ARG
    assert call(E=300) == nv.Status.INVALID_ARG
    assert call(K=96) == nv.Status.INVALID_ARG              # K % 32
    assert call(K=320) == nv.Status.INVALID_ARG             # K % 256
    assert call(off=0) == nv.Status.INVALID_ARG             # null offsets
    assert call(ws=0) == nv.Status.INVALID_ARG              # no workspace
    assert call(ws_bytes=need - 1) == nv.Status.INVALID_ARG  # too small
    assert b"nvfp4_workspace_size" in lib.nvfp4_last_error()
    assert call(A=24) == nv.Status.MISALIGNED
    assert call(ws=4104) == nv.Status.MISALIGNED
    assert call(M=0) == nv.Status.OK                        # nothing to do


def test_prepare_scales_argument_errors_need_no_device():
    lib = nv.load_library()
    assert lib.nvfp4_prepare_scales(16, 16, 128, 96, None) == nv.Status.INVALID_ARG   # K % 64
    assert lib.nvfp4_prepare_scales(0, 16, 128, 128, None) == nv.Status.INVALID_ARG
    assert lib.nvfp4_prepare_scales(24, 16, 128, 128, None) == nv.Status.MISALIGNED
    assert lib.nvfp4_prepare_scales(16, 16, 0, 128, None) == nv.Status.OK
