// nvfp4_api.cu -- the C ABI of include/nvfp4.h: argument checks, the exec_of
// planner (metrale_circuit `hardware::exec`: Exec, exec_of, fp4_fallback,
// kind_of, pair_name), tensor-map encoding and kernel launches.
//
// This is the only translation unit of the library; every kernel header is
// included here.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/nvfp4.h"
#include "ptx.cuh"
#include "w4a4_kernel.cuh"
#include "w4a4_pair_kernel.cuh"
#include "pack_scales_kernel.cuh"
#include "w4a16_kernel.cuh"
#include "via_fp8_kernel.cuh"
#include "w4a8_kernel.cuh"
#include "grouped_kernel.cuh"
#include "grouped_pair_kernel.cuh"
#include "quantize_kernel.cuh"
#include "moe_kernel.cuh"

namespace {

thread_local char t_last_error[512] = "";
std::atomic<int> g_fp4_kernel_disabled{0};

nvfp4_status fail(nvfp4_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
    va_end(ap);
    return st;
}

nvfp4_status ok() {
    t_last_error[0] = '\0';
    return NVFP4_OK;
}

nvfp4_status cuda_fail(cudaError_t e, const char* what) {
    return fail(NVFP4_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------- device info
struct DevInfo {
    bool valid = false;
    int sm_arch = 0;     // 10*major + minor
    int num_sms = 0;
    size_t smem_optin = 0;
};

std::mutex g_dev_mu;
DevInfo g_dev[64];

bool device_info(int dev, DevInfo& out) {
    if (dev < 0 || dev >= 64) return false;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!g_dev[dev].valid) {
        int major = 0, minor = 0, sms = 0, smem = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
                cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        g_dev[dev].sm_arch = major * 10 + minor;
        g_dev[dev].num_sms = sms;
        g_dev[dev].smem_optin = (size_t)smem;
        g_dev[dev].valid = true;
    }
    out = g_dev[dev];
    return true;
}

bool current_device(int& dev, DevInfo& info) {
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return device_info(dev, info);
}

// ---------------------------------------------------------------- planner
// Device classes that carry the block-scaled FP4 MMA instruction.
bool class_has_fp4_mma(int arch) {
    return arch == 100 || arch == 101 || arch == 103 || arch == 110 || arch == 120 || arch == 121;
}
// ... and the FP8 MMA.
bool class_has_fp8_mma(int arch) { return arch >= 89; }
// Classes this library compiles its kernels for (sm_100a code runs on CC 10.0 only).
bool class_compiles_fp4_kernel(int arch) { return arch == 100; }
bool class_compiles_fp8_exact_kernel(int arch) { return arch == 100; }
bool class_compiles_bf16_widen_kernel(int arch) { return arch == 100; }

// fp4_fallback: an NVFP4 activation on a class without an FP4 block-scale
// kernel.  NoFp4Kernel where the class's tensor cores do FP4 but this library
// compiles no kernel for it; else the exact FP8 path where the class has the FP8
// MMA (and this library's exact-path kernel); else no path.
nvfp4_exec fp4_fallback(int arch) {
    if (class_has_fp4_mma(arch)) return NVFP4_EXEC_NO_FP4_KERNEL;
    if (class_has_fp8_mma(arch) && class_compiles_fp8_exact_kernel(arch)) return NVFP4_EXEC_FP8_EXACT;
    return NVFP4_EXEC_NO_PATH;
}

bool valid_fmt(nvfp4_fmt f) {
    return f == NVFP4_FMT_BF16 || f == NVFP4_FMT_FP8_E4M3 || f == NVFP4_FMT_NVFP4;
}

// Launch-time check shared by the W4A4 entry points.
nvfp4_status check_fp4_path(int& dev, DevInfo& info) {
    if (!current_device(dev, info)) return fail(NVFP4_ERR_CUDA, "cannot query the current CUDA device");
    nvfp4_exec e = nvfp4_exec_of_arch(info.sm_arch, NVFP4_FMT_NVFP4, NVFP4_FMT_NVFP4,
                                      g_fp4_kernel_disabled.load());
    if (e == NVFP4_EXEC_FP4_MMA) return NVFP4_OK;
    if (e == NVFP4_EXEC_NO_FP4_KERNEL)
        return fail(NVFP4_ERR_NO_FP4_KERNEL,
                    "sm_%d has the FP4 MMA but no FP4 block-scale kernel is compiled for it",
                    info.sm_arch);
    return fail(NVFP4_ERR_NOPATH, "W4A4 has no FP4 MMA path on sm_%d (plan: %s)", info.sm_arch,
                nvfp4_exec_name(e));
}

// ---------------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool get_encoder() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        cudaGetLastError();
    });
    return g_encode != nullptr;
}

// 2D uint8 map over a row-major [rows][row_bytes] buffer, box [box_rows][box_bytes],
// zero fill out of bounds; 128-byte swizzle (box_bytes == 128) or none.
nvfp4_status make_map_u8(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows,
                         uint32_t box_bytes, uint32_t box_rows,
                         CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
    if (!get_encoder()) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t dims[2] = {row_bytes, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_bytes, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return NVFP4_OK;
}

// 3D uint8 map over packed scales viewed as [blocks][ksteps*4][128 B]
// (one 128-row block's packed scales are ksteps 512-byte atoms), box
// (128, 16, box_blocks): one K-block (four K = 64 steps) of box_blocks blocks.
nvfp4_status make_map_packed_sf(CUtensorMap* map, const void* base, uint64_t blocks,
                                uint64_t ksteps, uint32_t box_blocks) {
    if (!get_encoder()) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t dims[3] = {128, ksteps * 4, blocks};
    cuuint64_t strides[2] = {128, ksteps * 512};
    cuuint32_t box[3] = {128, 16, box_blocks};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return NVFP4_OK;
}

// Output map of the pair kernels' TMA-store epilogue: Y bf16 [rows][N], box
// 64 columns (128 bytes) x 32 rows, 128-byte swizzle.  Needs N % 8 == 0 (the
// row pitch must be a multiple of 16 bytes); otherwise `valid` is 0 and the
// kernels use plain stores (the map is then zero and never read).
nvfp4_status make_map_out(CUtensorMap* map, const void* Y, uint64_t rows, uint64_t N, int& valid) {
    memset(map, 0, sizeof(*map));
    valid = 0;
    if (N % 8 != 0) return NVFP4_OK;
    if (!get_encoder()) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t dims[2] = {N, rows};
    cuuint64_t strides[1] = {N * 2};
    cuuint32_t box[2] = {64, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(Y), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    valid = 1;
    return NVFP4_OK;
}

// ---------------------------------------------------------------- argument checks
nvfp4_status check_w4a4_args(const void* A, const void* sA, const void* W, const void* sW,
                             const void* Y, int M, int N, int K) {
    if (M < 0 || N < 0) return fail(NVFP4_ERR_INVALID_ARG, "M and N must be >= 0 (got %d, %d)", M, N);
    if (K < 32 || K % 32 != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "K must be a positive multiple of 32 (got %d)", K);
    if (M == 0 || N == 0) return NVFP4_OK;
    if (!A || !sA || !W || !sW || !Y) return fail(NVFP4_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned16(A) || !aligned16(sA) || !aligned16(W) || !aligned16(sW) || !aligned16(Y))
        return fail(NVFP4_ERR_MISALIGNED, "every buffer must be 16-byte aligned");
    return NVFP4_OK;
}

// offsets (int32 [E+1], host): offsets[0] == 0, non-decreasing; total rows in M.
nvfp4_status check_offsets(const int32_t* offsets_host, int E, int max_groups, int& M) {
    if (E < 1 || E > max_groups)
        return fail(NVFP4_ERR_INVALID_ARG, "E must be in [1, %d] (got %d)", max_groups, E);
    if (!offsets_host) return fail(NVFP4_ERR_INVALID_ARG, "null offsets");
    if (offsets_host[0] != 0) return fail(NVFP4_ERR_INVALID_ARG, "offsets[0] must be 0");
    for (int e = 0; e < E; ++e)
        if (offsets_host[e + 1] < offsets_host[e])
            return fail(NVFP4_ERR_INVALID_ARG, "offsets must be non-decreasing");
    M = offsets_host[E];
    return NVFP4_OK;
}

// sum over groups of ceil(rows/128): the grouped packed layout's block count
int64_t grouped_blocks(const int32_t* offsets_host, int E) {
    int64_t b = 0;
    for (int e = 0; e < E; ++e) b += (offsets_host[e + 1] - offsets_host[e] + 127) / 128;
    return b;
}

template <typename Kern>
nvfp4_status set_smem(Kern k, size_t bytes, const DevInfo& info, const char* name) {
    if (bytes > info.smem_optin)
        return fail(NVFP4_ERR_CUDA, "%s needs %zu B of shared memory, device allows %zu", name,
                    bytes, info.smem_optin);
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return cuda_fail(e, name);
    return NVFP4_OK;
}

using W4a16LdgKern = void (*)(const uint16_t*, const uint8_t*, const uint8_t*, __nv_bfloat16*, int,
                              int, int, float, int);
// the register-load instantiation for `nb` row blocks per CTA (1..LDG_MAX_NB)
W4a16LdgKern w4a16_ldg_kernel_for(int nb) {
    namespace k16 = nvfp4::w4a16;
    static_assert(k16::LDG_MAX_NB == 6, "one instantiation per row-block count");
    switch (nb) {
        case 1: return k16::w4a16_ldg_kernel<1>;
        case 2: return k16::w4a16_ldg_kernel<2>;
        case 3: return k16::w4a16_ldg_kernel<3>;
        case 4: return k16::w4a16_ldg_kernel<4>;
        case 5: return k16::w4a16_ldg_kernel<5>;
        default: return k16::w4a16_ldg_kernel<6>;
    }
}

}  // namespace

// =====================================================================================
extern "C" {

const char* nvfp4_version(void) { return "nvfp4-b200 0.1 (sm_100a)"; }

const char* nvfp4_last_error(void) { return t_last_error; }

nvfp4_kind nvfp4_kind_of(nvfp4_fmt activation) {
    switch (activation) {
    case NVFP4_FMT_BF16: return NVFP4_KIND_BF16_MMA;
    case NVFP4_FMT_FP8_E4M3: return NVFP4_KIND_FP8_MMA;
    case NVFP4_FMT_NVFP4: return NVFP4_KIND_FP4_BLOCK_SCALED;
    }
    return NVFP4_KIND_INVALID;
}

const char* nvfp4_pair_name(nvfp4_fmt weight, nvfp4_fmt activation) {
    static const char* names[3][3] = {
        {"W16A16", "W16A8", "W16A4"}, {"W8A16", "W8A8", "W8A4"}, {"W4A16", "W4A8", "W4A4"}};
    if (!valid_fmt(weight) || !valid_fmt(activation)) return "?";
    return names[weight][activation];
}

const char* nvfp4_exec_name(nvfp4_exec e) {
    switch (e) {
    case NVFP4_EXEC_FP4_MMA: return "FP4_MMA";
    case NVFP4_EXEC_FP8_EXACT: return "FP8_EXACT";
    case NVFP4_EXEC_BF16_WIDEN: return "BF16_WIDEN";
    case NVFP4_EXEC_NO_FP4_KERNEL: return "NO_FP4_KERNEL";
    case NVFP4_EXEC_NO_PATH: return "NO_PATH";
    }
    return "?";
}

nvfp4_exec nvfp4_exec_of_arch(int arch, nvfp4_fmt weight, nvfp4_fmt activation,
                              int fp4_kernel_disabled) {
    if (!valid_fmt(weight) || !valid_fmt(activation)) return NVFP4_EXEC_NO_PATH;
    if (weight != NVFP4_FMT_NVFP4) return NVFP4_EXEC_NO_PATH;  // NVFP4-weight paths only
    switch (nvfp4_kind_of(activation)) {
    case NVFP4_KIND_FP4_BLOCK_SCALED:
        if (class_has_fp4_mma(arch) && class_compiles_fp4_kernel(arch) && !fp4_kernel_disabled)
            return NVFP4_EXEC_FP4_MMA;
        return fp4_fallback(arch);
    case NVFP4_KIND_BF16_MMA:
        return class_compiles_bf16_widen_kernel(arch) ? NVFP4_EXEC_BF16_WIDEN : NVFP4_EXEC_NO_PATH;
    case NVFP4_KIND_FP8_MMA:
        // W4A8 has no single-instruction MMA (no FP4 x FP8 MMA takes E4M3 group-16
        // scales); it takes the exact E4M3 path where that kernel is compiled.
        if (class_has_fp8_mma(arch) && class_compiles_fp8_exact_kernel(arch)) return NVFP4_EXEC_FP8_EXACT;
        return NVFP4_EXEC_NO_PATH;
    default:
        return NVFP4_EXEC_NO_PATH;
    }
}

nvfp4_exec nvfp4_fp4_fallback(int sm_arch) { return fp4_fallback(sm_arch); }

nvfp4_status nvfp4_node_exec(int sm_arch, int fp4_kernel_disabled, const int32_t* weight_fmt,
                             const int32_t* activation_fmt, int n, int32_t* exec_out) {
    if (n < 0) return fail(NVFP4_ERR_INVALID_ARG, "node count must be >= 0 (got %d)", n);
    if (n > 0 && (!weight_fmt || !activation_fmt || !exec_out))
        return fail(NVFP4_ERR_INVALID_ARG, "null node array");
    for (int i = 0; i < n; ++i)
        exec_out[i] = (int32_t)nvfp4_exec_of_arch(sm_arch, (nvfp4_fmt)weight_fmt[i],
                                                  (nvfp4_fmt)activation_fmt[i], fp4_kernel_disabled);
    return ok();
}

nvfp4_exec nvfp4_exec_of(int device, nvfp4_fmt weight, nvfp4_fmt activation) {
    DevInfo info;
    if (!device_info(device, info)) return NVFP4_EXEC_NO_PATH;
    return nvfp4_exec_of_arch(info.sm_arch, weight, activation, g_fp4_kernel_disabled.load());
}

void nvfp4_set_fp4_kernel_disabled(int disabled) { g_fp4_kernel_disabled.store(disabled ? 1 : 0); }

nvfp4_status nvfp4_check_device_error(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int v = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&v, nvfp4::g_device_error, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    if (v == 0) return ok();
    e = cudaMemcpyToSymbol(nvfp4::g_device_error, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
    if (v & 0xFF)
        return fail(NVFP4_ERR_DEVICE_TIMEOUT, "a kernel wait expired (role %d)", (v >> 8) & 0xFF);
    if (v & nvfp4::grouped_pair::BAD_OFFSETS)
        return fail(NVFP4_ERR_INVALID_ARG,
                    "device expert offsets were not a non-decreasing run from 0 to M");
    if (v & nvfp4::grouped_pair::BAD_DEST)
        return fail(NVFP4_ERR_INVALID_ARG, "a grouped row's output row (src) was outside [0, T)");
    return fail(NVFP4_ERR_INVALID_ARG, "a routed expert id was outside [0, E)");
}

// ------------------------------------------------------------------------- W4A4
nvfp4_status gemm_nvfp4_w4a4(const uint8_t* A, const uint8_t* sA, float gA, const uint8_t* W,
                             const uint8_t* sW, float gW, void* Y, int M, int N, int K,
                             void* stream) {
    nvfp4_status st = check_w4a4_args(A, sA, W, sW, Y, M, N, K);
    if (st != NVFP4_OK) return st;
    int dev;
    DevInfo info;
    if ((st = check_fp4_path(dev, info)) != NVFP4_OK) return st;
    if (M == 0 || N == 0) return ok();

    const bool sf_tma = (K % nvfp4::w4a4::BK) == 0;  // scale row pitch K/16 is 16-byte aligned
    constexpr int BN = 256, STAGES = 4;
    using C = nvfp4::w4a4::Cfg<BN, STAGES>;
    auto kern = sf_tma ? nvfp4::w4a4::w4a4_kernel<BN, STAGES, true>
                       : nvfp4::w4a4::w4a4_kernel<BN, STAGES, false>;
    CUtensorMap tmA, tmB, tmSA, tmSB;
    if ((st = make_map_u8(&tmA, A, (uint64_t)K / 2, (uint64_t)M, nvfp4::w4a4::BKB,
                          nvfp4::w4a4::BM)) != NVFP4_OK)
        return st;
    if ((st = make_map_u8(&tmB, W, (uint64_t)K / 2, (uint64_t)N, nvfp4::w4a4::BKB, BN)) != NVFP4_OK)
        return st;
    if (sf_tma) {
        if ((st = make_map_u8(&tmSA, sA, (uint64_t)K / 16, (uint64_t)M, 16, nvfp4::w4a4::BM,
                              CU_TENSOR_MAP_SWIZZLE_NONE)) != NVFP4_OK)
            return st;
        if ((st = make_map_u8(&tmSB, sW, (uint64_t)K / 16, (uint64_t)N, 16, BN,
                              CU_TENSOR_MAP_SWIZZLE_NONE)) != NVFP4_OK)
            return st;
    } else {
        tmSA = tmA;  // unused
        tmSB = tmB;
    }
    if ((st = set_smem(kern, C::SMEM_BYTES, info, "w4a4_kernel")) != NVFP4_OK) return st;

    const int tiles = ((M + nvfp4::w4a4::BM - 1) / nvfp4::w4a4::BM) * ((N + BN - 1) / BN);
    const int grid = tiles < info.num_sms ? tiles : info.num_sms;
    kern<<<grid, nvfp4::w4a4::NUM_THREADS, C::SMEM_BYTES, static_cast<cudaStream_t>(stream)>>>(
        tmA, tmB, tmSA, tmSB, sA, sW, reinterpret_cast<__nv_bfloat16*>(Y), M, N, K, gA * gW);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launching w4a4_kernel");
    return ok();
}

// ------------------------------------------------------------------------- packed scales
size_t nvfp4_scale_layout_bytes(int rows, int K) {
    if (rows < 0 || K < 64 || K % 64 != 0) return 0;
    return (size_t)((rows + 127) / 128) * 128 * (size_t)(K / 16);
}

nvfp4_status nvfp4_pack_scales(const uint8_t* s_plain, int rows, int K, uint8_t* s_packed,
                               void* stream) {
    if (rows < 0) return fail(NVFP4_ERR_INVALID_ARG, "rows must be >= 0 (got %d)", rows);
    if (K < 64 || K % 64 != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "packing needs K %% 64 == 0 (got %d)", K);
    if (rows == 0) return ok();
    if (!s_plain || !s_packed) return fail(NVFP4_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned16(s_plain) || !aligned16(s_packed))
        return fail(NVFP4_ERR_MISALIGNED, "s_plain and s_packed must be 16-byte aligned");
    const int ksteps = K / 64;
    const dim3 grid((unsigned)((rows + 127) / 128),
                    (unsigned)((ksteps + nvfp4::pack::KCHUNK - 1) / nvfp4::pack::KCHUNK));
    if (grid.y > 65535) return fail(NVFP4_ERR_INVALID_ARG, "K too large for packing");
    nvfp4::pack::pack_scales_kernel<<<grid, nvfp4::pack::ROWS, 0, static_cast<cudaStream_t>(stream)>>>(
        s_plain, s_packed, rows, K / 16, ksteps);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launching pack_scales_kernel");
    return ok();
}

// ------------------------------------------------------------------------- quantiser
size_t nvfp4_quantize_workspace_bytes(void) { return NVFP4_QUANTIZE_WORKSPACE_BYTES; }

namespace {
// The quantiser's checks and launches; dest == nullptr writes row r to row r,
// otherwise to rows dest[r k + j].
nvfp4_status quantize_bf16_impl(const void* X, int rows, int K, uint8_t* codes, uint8_t* scales,
                                uint8_t* scales_packed, float* g_out, void* workspace,
                                size_t workspace_bytes, void* stream, const int32_t* dest, int k) {
    namespace q = nvfp4::quant;
    if (rows < 0) return fail(NVFP4_ERR_INVALID_ARG, "rows must be >= 0 (got %d)", rows);
    if (K < 16 || K % 16 != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "K must be a positive multiple of 16 (got %d)", K);
    if (!g_out || !workspace || (rows > 0 && (!X || !codes)))
        return fail(NVFP4_ERR_INVALID_ARG, "null pointer argument");
    if (!scales && !scales_packed)
        return fail(NVFP4_ERR_INVALID_ARG, "at least one of scales and scales_packed is needed");
    if (scales_packed && K % 64 != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "packed scales need K %% 64 == 0 (got %d)", K);
    if (workspace_bytes < NVFP4_QUANTIZE_WORKSPACE_BYTES)
        return fail(NVFP4_ERR_INVALID_ARG, "the workspace needs %d bytes (got %zu)",
                    NVFP4_QUANTIZE_WORKSPACE_BYTES, workspace_bytes);
    if ((X && !aligned16(X)) || (codes && !aligned16(codes)) || (scales && !aligned16(scales)) ||
        (scales_packed && !aligned16(scales_packed)) || !aligned16(workspace) ||
        reinterpret_cast<uintptr_t>(g_out) % 4 != 0)
        return fail(NVFP4_ERR_MISALIGNED, "buffers must be 16-byte aligned (g_out 4-byte)");
    if ((long long)rows * K > (1ll << 40)) return fail(NVFP4_ERR_INVALID_ARG, "tensor too large");
    int dev;
    DevInfo info;
    if (!current_device(dev, info)) return fail(NVFP4_ERR_CUDA, "cannot query the current CUDA device");
    if (info.sm_arch != 100)
        return fail(NVFP4_ERR_NOPATH, "the quantiser is compiled for sm_100 only (device sm_%d)",
                    info.sm_arch);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned* amax = static_cast<unsigned*>(workspace);
    cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(unsigned), st);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the quantiser workspace");
    const size_t total = (size_t)rows * K;
    const size_t n16 = total / 8;
    if (total > 0) {
        size_t blocks = (n16 + q::AMAX_THREADS - 1) / q::AMAX_THREADS;
        const size_t cap = (size_t)info.num_sms * 4;
        if (blocks > cap) blocks = cap;
        if (blocks == 0) blocks = 1;
        const uint16_t* x16 = static_cast<const uint16_t*>(X);
        q::amax_bf16_kernel<<<(unsigned)blocks, q::AMAX_THREADS, 0, st>>>(
            reinterpret_cast<const uint4*>(X), n16, x16 + n16 * 8, (int)(total - n16 * 8), amax);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "launching amax_bf16_kernel");
    }
    // at least one CTA, so that g_out is written for an empty tensor too
    const dim3 grid((unsigned)(rows > 0 ? (rows + q::TILE_ROWS - 1) / q::TILE_ROWS : 1),
                    (unsigned)((K + q::TILE_COLS - 1) / q::TILE_COLS));
    if (grid.y > 65535) return fail(NVFP4_ERR_INVALID_ARG, "K too large (got %d)", K);
    // launched programmatically: its CTAs may start (and read X) while the amax kernel
    // finishes; they read the maximum only after griddepcontrol.wait
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(q::THREADS);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // 256-bit loads when X starts on a 32-byte boundary (rows then do too: K % 16 == 0)
    const bool v8 = reinterpret_cast<uintptr_t>(X) % 32 == 0;
    auto kern = dest ? (v8 ? q::quantize_bf16_kernel<true, true> : q::quantize_bf16_kernel<false, true>)
                     : (v8 ? q::quantize_bf16_kernel<true, false> : q::quantize_bf16_kernel<false, false>);
    e = cudaLaunchKernelEx(&cfg, kern, static_cast<const __nv_bfloat16*>(X), rows, K,
                           static_cast<const unsigned*>(amax), codes, scales, scales_packed, g_out,
                           dest, k);
    if (e != cudaSuccess) return cuda_fail(e, "launching quantize_bf16_kernel");
    return ok();
}
}  // namespace

nvfp4_status nvfp4_quantize_bf16(const void* X, int rows, int K, uint8_t* codes, uint8_t* scales,
                                 uint8_t* scales_packed, float* g_out, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    return quantize_bf16_impl(X, rows, K, codes, scales, scales_packed, g_out, workspace,
                              workspace_bytes, stream, nullptr, 1);
}

nvfp4_status nvfp4_quantize_bf16_routed(const void* X, int rows, int K, const int32_t* dest, int k,
                                        uint8_t* codes, uint8_t* scales, float* g_out,
                                        void* workspace, size_t workspace_bytes, void* stream) {
    if (k < 1 || k > 8) return fail(NVFP4_ERR_INVALID_ARG, "k must be in [1, 8] (got %d)", k);
    if (!scales) return fail(NVFP4_ERR_INVALID_ARG, "the routed quantiser writes plain scales: null scales");
    if (rows > 0 && !dest) return fail(NVFP4_ERR_INVALID_ARG, "null dest");
    if (dest && reinterpret_cast<uintptr_t>(dest) % 4 != 0)
        return fail(NVFP4_ERR_MISALIGNED, "dest must be 4-byte aligned");
    if ((long long)rows * k > INT32_MAX) return fail(NVFP4_ERR_INVALID_ARG, "rows * k too large");
    return quantize_bf16_impl(X, rows, K, codes, scales, nullptr, g_out, workspace, workspace_bytes,
                              stream, rows > 0 ? dest : nullptr, k);
}

// ------------------------------------------------------------------------- quantiser without
// a caller workspace
//
// nvfp4_quantize_bf16 keeps its running amax in a few bytes of caller-owned
// device scratch.  This variant keeps them in a static device array instead, so
// a caller that cannot allocate device memory (or cannot keep a scratch buffer
// between calls) can still quantise.  The array lives in every GPU that loads
// the library until the process exits.
namespace {
constexpr size_t kNoAllocScratchBytes = 256;  // the stated maximum; the quantiser needs 16
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
static_assert(NVFP4_QUANTIZE_WORKSPACE_BYTES <= kNoAllocScratchBytes,
              "the static scratch must hold the quantiser's workspace");

// The device address of g_noalloc_scratch in the current context (the host-side
// name is only a stand-in for it).  Looked up on every call: the address belongs
// to a context, not to a device ordinal, so a cached one could outlive its context
// (after cudaDeviceReset, or under a caller's own driver context).  The lookup
// allocates nothing; the first one in a context loads the library's device code
// there, which is why the first call should come before any stream capture.
nvfp4_status noalloc_scratch(void** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "looking up the static quantiser scratch");
    *out = p;
    return NVFP4_OK;
}
}  // namespace

nvfp4_status nvfp4_quantize_bf16_noalloc(const void* X, int rows, int K, uint8_t* codes,
                                         uint8_t* scales, uint8_t* scales_packed, float* g_out,
                                         void* stream) {
    const size_t need = nvfp4_quantize_workspace_bytes();  // does not grow with the tensor
    if (need > kNoAllocScratchBytes)
        return fail(NVFP4_ERR_INVALID_ARG,
                    "this call needs %zu bytes of scratch, more than the %zu of the static array",
                    need, kNoAllocScratchBytes);
    void* scratch = nullptr;
    nvfp4_status st = noalloc_scratch(&scratch);
    if (st != NVFP4_OK) return st;
    return nvfp4_quantize_bf16(X, rows, K, codes, scales, scales_packed, g_out, scratch,
                               kNoAllocScratchBytes, stream);
}

namespace {
// How the pair kernel hands out its tiles: `pairs` clusters; tiles below dp_tiles
// whole and in turn, the rest as K-block ranges (stream-K) with `slots` cut tiles.
struct PairPlan {
    int pairs = 0, tiles = 0, dp_tiles = 0, slots = 0;
};

PairPlan pair_plan(int M, int N, int K, int num_sms, int max_pairs, bool split) {
    namespace wp = nvfp4::w4a4_pair;
    PairPlan p;
    p.tiles = ((M + wp::TILE_M - 1) / wp::TILE_M) * ((N + wp::BN - 1) / wp::BN);
    p.pairs = p.tiles < num_sms / 2 ? p.tiles : num_sms / 2;
    if (max_pairs > 0 && p.pairs > max_pairs) p.pairs = max_pairs;
    p.dp_tiles = p.tiles;
    if (p.pairs < 1) return p;
    const int full = p.tiles / p.pairs, rem = p.tiles % p.pairs;
    // A last wave of whole tiles keeps (pairs - rem) pairs idle for one tile's
    // time; balanced, that wave costs rem/pairs of a tile instead.  The balancing
    // itself costs about 0.4 of a tile's time on a B200 (the partial-sum exchange,
    // one more segment per pair, and no power headroom from idle SMs), so it is
    // used when the last wave is at most 60 % full.  A cut needs K / 256 >= 2.
    if (split && full >= 1 && rem != 0 && rem * 5 <= p.pairs * 3 && K / wp::BK >= 2) {
        p.dp_tiles = (full - 1) * p.pairs;  // leaves rem + pairs tiles: every range >= 1 tile
        p.slots = p.pairs - 1;
    }
    return p;
}

nvfp4_status launch_w4a4_pair(const uint8_t* A, const uint8_t* sA_packed, float gA,
                              const uint8_t* W, const uint8_t* sW_packed, float gW, void* Y,
                              int M, int N, int K, int max_pairs, void* workspace,
                              size_t workspace_bytes, void* stream) {
    namespace wp = nvfp4::w4a4_pair;
    if (max_pairs < 0) return fail(NVFP4_ERR_INVALID_ARG, "max_pairs must be >= 0 (got %d)", max_pairs);
    nvfp4_status st = check_w4a4_args(A, sA_packed, W, sW_packed, Y, M, N, K);
    if (st != NVFP4_OK) return st;
    if (K % wp::BK != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "the packed-scale path needs K %% 256 == 0 (got %d)", K);
    int dev;
    DevInfo info;
    if ((st = check_fp4_path(dev, info)) != NVFP4_OK) return st;
    if (M == 0 || N == 0) return ok();
    if (info.num_sms < 2) return fail(NVFP4_ERR_CUDA, "the pair kernel needs at least two SMs");

    CUtensorMap tmA, tmB, tmSA, tmSB;
    const uint64_t ks = (uint64_t)K / 64;
    if ((st = make_map_u8(&tmA, A, (uint64_t)K / 2, (uint64_t)M, wp::BKB, wp::BM)) != NVFP4_OK) return st;
    if ((st = make_map_u8(&tmB, W, (uint64_t)K / 2, (uint64_t)N, wp::BKB, wp::BNH)) != NVFP4_OK) return st;
    if ((st = make_map_packed_sf(&tmSA, sA_packed, (uint64_t)(M + 127) / 128, ks, 1)) != NVFP4_OK)
        return st;
    if ((st = make_map_packed_sf(&tmSB, sW_packed, (uint64_t)(N + 127) / 128, ks, wp::NRB)) != NVFP4_OK)
        return st;
    CUtensorMap tmY;
    int tma_out = 0;
    if ((st = make_map_out(&tmY, Y, (uint64_t)M, (uint64_t)N, tma_out)) != NVFP4_OK) return st;
    if ((st = set_smem(wp::w4a4_pair_kernel, wp::SMEM_BYTES, info, "w4a4_pair_kernel")) != NVFP4_OK)
        return st;
    const PairPlan plan = pair_plan(M, N, K, info.num_sms, max_pairs, workspace != nullptr);
    float* partials = nullptr;
    unsigned* tickets = nullptr;
    if (plan.slots > 0) {
        const size_t need = wp::split_workspace_bytes(plan.slots);
        if (workspace_bytes < need)
            return fail(NVFP4_ERR_INVALID_ARG, "the workspace holds %zu bytes; this shape needs %zu",
                        workspace_bytes, need);
        if (!aligned16(workspace)) return fail(NVFP4_ERR_MISALIGNED, "the workspace must be 16-byte aligned");
        tickets = static_cast<unsigned*>(workspace);
        partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + wp::ticket_bytes(plan.slots));
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * plan.pairs);
    cfg.blockDim = dim3(wp::NUM_THREADS);
    cfg.dynamicSmemBytes = wp::SMEM_BYTES;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // may start while the stream's previous kernel (the scale packing) finishes; the
    // kernel waits for it before reading anything it wrote
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, wp::w4a4_pair_kernel, tmA, tmB, tmSA, tmSB, tmY,
                                       tma_out, reinterpret_cast<__nv_bfloat16*>(Y), M, N, K,
                                       gA * gW, plan.dp_tiles, partials, tickets);
    if (e != cudaSuccess) return cuda_fail(e, "launching w4a4_pair_kernel");
    return ok();
}
}  // namespace

nvfp4_status gemm_nvfp4_w4a4_packed(const uint8_t* A, const uint8_t* sA_packed, float gA,
                                    const uint8_t* W, const uint8_t* sW_packed, float gW,
                                    void* Y, int M, int N, int K, void* stream) {
    return launch_w4a4_pair(A, sA_packed, gA, W, sW_packed, gW, Y, M, N, K, 0, nullptr, 0, stream);
}

size_t nvfp4_w4a4_packed_workspace_bytes_for(int M, int N, int K, int max_pairs, int num_sms) {
    if (M <= 0 || N <= 0 || K <= 0 || max_pairs < 0 || num_sms < 2) return 0;
    const PairPlan plan = pair_plan(M, N, K, num_sms, max_pairs, true);
    return plan.slots > 0 ? nvfp4::w4a4_pair::split_workspace_bytes(plan.slots) : 0;
}

size_t nvfp4_w4a4_packed_workspace_bytes(int M, int N, int K, int max_pairs) {
    int dev;
    DevInfo info;
    if (!current_device(dev, info)) return 0;
    return nvfp4_w4a4_packed_workspace_bytes_for(M, N, K, max_pairs, info.num_sms);
}

nvfp4_status gemm_nvfp4_w4a4_packed_ws(const uint8_t* A, const uint8_t* sA_packed, float gA,
                                       const uint8_t* W, const uint8_t* sW_packed, float gW,
                                       void* Y, int M, int N, int K, int max_pairs,
                                       void* workspace, size_t workspace_bytes, void* stream) {
    return launch_w4a4_pair(A, sA_packed, gA, W, sW_packed, gW, Y, M, N, K, max_pairs, workspace,
                            workspace_bytes, stream);
}

// ------------------------------------------------------------------------- via FP8
nvfp4_status gemm_nvfp4_via_fp8(const uint8_t* A, const uint8_t* sA, float gA, const uint8_t* W,
                                const uint8_t* sW, float gW, void* Y, int M, int N, int K,
                                void* stream) {
    namespace v8 = nvfp4::via_fp8;
    nvfp4_status st = check_w4a4_args(A, sA, W, sW, Y, M, N, K);
    if (st != NVFP4_OK) return st;
    if (K % v8::BK != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "the exact FP8 path needs K %% 256 == 0 (got %d)", K);
    int dev;
    DevInfo info;
    if (!current_device(dev, info)) return fail(NVFP4_ERR_CUDA, "cannot query the current CUDA device");
    if (!class_has_fp8_mma(info.sm_arch) || !class_compiles_fp8_exact_kernel(info.sm_arch))
        return fail(NVFP4_ERR_NOPATH, "no exact FP8-path kernel is compiled for sm_%d", info.sm_arch);
    if (M == 0 || N == 0) return ok();

    CUtensorMap tmA, tmB, tmSA, tmSB;
    if ((st = make_map_u8(&tmA, A, (uint64_t)K / 2, (uint64_t)M, 128, v8::BM)) != NVFP4_OK) return st;
    if ((st = make_map_u8(&tmB, W, (uint64_t)K / 2, (uint64_t)N, 128, v8::BN)) != NVFP4_OK) return st;
    if ((st = make_map_u8(&tmSA, sA, (uint64_t)K / 16, (uint64_t)M, 16, v8::BM,
                          CU_TENSOR_MAP_SWIZZLE_NONE)) != NVFP4_OK)
        return st;
    if ((st = make_map_u8(&tmSB, sW, (uint64_t)K / 16, (uint64_t)N, 16, v8::BN,
                          CU_TENSOR_MAP_SWIZZLE_NONE)) != NVFP4_OK)
        return st;
    if ((st = set_smem(v8::via_fp8_kernel, v8::SMEM_BYTES, info, "via_fp8_kernel")) != NVFP4_OK)
        return st;
    const int tiles = ((M + v8::BM - 1) / v8::BM) * ((N + v8::BN - 1) / v8::BN);
    const int grid = tiles < info.num_sms ? tiles : info.num_sms;
    v8::via_fp8_kernel<<<grid, v8::NUM_THREADS, v8::SMEM_BYTES, static_cast<cudaStream_t>(stream)>>>(
        tmA, tmB, tmSA, tmSB, reinterpret_cast<__nv_bfloat16*>(Y), M, N, K, gA * gW);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launching via_fp8_kernel");
    return ok();
}

// ------------------------------------------------------------------------- W4A8
nvfp4_status gemm_nvfp4_w4a8(const uint8_t* A_fp8, float gA, const uint8_t* W, const uint8_t* sW,
                             float gW, void* Y, int M, int N, int K, void* stream) {
    namespace k8 = nvfp4::w4a8;
    if (M < 0 || N < 0) return fail(NVFP4_ERR_INVALID_ARG, "M and N must be >= 0 (got %d, %d)", M, N);
    if (K < k8::BK || K % k8::BK != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "W4A8 needs K a positive multiple of 256 (got %d)", K);
    if (M > 0 && N > 0) {
        if (!A_fp8 || !W || !sW || !Y) return fail(NVFP4_ERR_INVALID_ARG, "null pointer argument");
        if (!aligned16(A_fp8) || !aligned16(W) || !aligned16(sW) || !aligned16(Y))
            return fail(NVFP4_ERR_MISALIGNED, "every buffer must be 16-byte aligned");
    }
    int dev;
    DevInfo info;
    if (!current_device(dev, info)) return fail(NVFP4_ERR_CUDA, "cannot query the current CUDA device");
    if (nvfp4_exec_of_arch(info.sm_arch, NVFP4_FMT_NVFP4, NVFP4_FMT_FP8_E4M3, 0) != NVFP4_EXEC_FP8_EXACT)
        return fail(NVFP4_ERR_NOPATH, "no exact E4M3-path kernel for W4A8 is compiled for sm_%d",
                    info.sm_arch);
    if (M == 0 || N == 0) return ok();

    nvfp4_status st;
    CUtensorMap tmA, tmB, tmSB;
    // activations: 128-byte-wide boxes of the tile's 256 token rows (the MMA's B side);
    // weights: 128-byte boxes of the tile's 128 weight rows (converted into TMEM)
    if ((st = make_map_u8(&tmA, A_fp8, (uint64_t)K, (uint64_t)M, 128, k8::BT)) != NVFP4_OK) return st;
    if ((st = make_map_u8(&tmB, W, (uint64_t)K / 2, (uint64_t)N, 128, k8::BW)) != NVFP4_OK) return st;
    if ((st = make_map_u8(&tmSB, sW, (uint64_t)K / 16, (uint64_t)N, 16, k8::BW,
                          CU_TENSOR_MAP_SWIZZLE_NONE)) != NVFP4_OK)
        return st;
    if ((st = set_smem(k8::w4a8_kernel, k8::SMEM_BYTES, info, "w4a8_kernel")) != NVFP4_OK) return st;
    const int tiles = ((M + k8::BT - 1) / k8::BT) * ((N + k8::BW - 1) / k8::BW);
    const int grid = tiles < info.num_sms ? tiles : info.num_sms;
    k8::w4a8_kernel<<<grid, k8::NUM_THREADS, k8::SMEM_BYTES, static_cast<cudaStream_t>(stream)>>>(
        tmA, tmB, tmSB, reinterpret_cast<__nv_bfloat16*>(Y), M, N, K, gA * gW);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launching w4a8_kernel");
    return ok();
}

// ------------------------------------------------------------------------- MoE
namespace {
int route_chunks(int P) {
    const int c = (P + nvfp4::moe::ROUTE_THREADS - 1) / nvfp4::moe::ROUTE_THREADS;
    return c < nvfp4::moe::MAX_CHUNKS ? c : nvfp4::moe::MAX_CHUNKS;
}
}  // namespace

size_t nvfp4_moe_route_workspace_bytes(int num_pairs, int E) {
    if (num_pairs < 0 || E < 1 || E > nvfp4::moe::MAX_EXPERTS) return 0;
    return (size_t)2 * route_chunks(num_pairs) * E * sizeof(int32_t) + 16;
}

nvfp4_status nvfp4_moe_route(const int32_t* expert_ids, int num_pairs, int E, int32_t* offsets,
                             int32_t* dest, int32_t* src, void* workspace, size_t workspace_bytes,
                             void* stream) {
    namespace mo = nvfp4::moe;
    if (num_pairs < 0) return fail(NVFP4_ERR_INVALID_ARG, "num_pairs must be >= 0 (got %d)", num_pairs);
    if (E < 1 || E > mo::MAX_EXPERTS)
        return fail(NVFP4_ERR_INVALID_ARG, "E must be in [1, %d] (got %d)", mo::MAX_EXPERTS, E);
    if (!offsets || (num_pairs > 0 && (!expert_ids || !dest || !src || !workspace)))
        return fail(NVFP4_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned16(workspace) && num_pairs > 0)
        return fail(NVFP4_ERR_MISALIGNED, "the workspace must be 16-byte aligned");
    const size_t need = nvfp4_moe_route_workspace_bytes(num_pairs, E);
    if (num_pairs > 0 && workspace_bytes < need)
        return fail(NVFP4_ERR_INVALID_ARG, "route workspace of %zu bytes is too small (need %zu)",
                    workspace_bytes, need);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (num_pairs == 0) {
        e = cudaMemsetAsync(offsets, 0, (size_t)(E + 1) * sizeof(int32_t), s);
        return e == cudaSuccess ? ok() : cuda_fail(e, "clearing the expert offsets");
    }
    if (num_pairs <= mo::SMALL_PAIRS) {  // one CTA does all three passes
        mo::route_small_kernel<<<1, mo::ROUTE_THREADS, 0, s>>>(expert_ids, num_pairs, E, offsets, dest,
                                                               src);
        e = cudaGetLastError();
        return e == cudaSuccess ? ok() : cuda_fail(e, "launching route_small_kernel");
    }
    // pairs with an out-of-range id are placed nowhere: their dest stays -1, and rows
    // no pair lands on keep src = -1
    if ((e = cudaMemsetAsync(dest, 0xFF, (size_t)num_pairs * sizeof(int32_t), s)) != cudaSuccess ||
        (e = cudaMemsetAsync(src, 0xFF, (size_t)num_pairs * sizeof(int32_t), s)) != cudaSuccess)
        return cuda_fail(e, "clearing the route maps");
    const int C = route_chunks(num_pairs);
    const int chunk = (num_pairs + C - 1) / C;
    int32_t* counts = static_cast<int32_t*>(workspace);
    int32_t* base = counts + (size_t)C * E;
    mo::route_count_kernel<<<C, mo::ROUTE_THREADS, 0, s>>>(expert_ids, num_pairs, E, chunk, counts);
    mo::route_scan_kernel<<<1, mo::MAX_EXPERTS, 0, s>>>(counts, C, E, base, offsets);
    mo::route_rank_kernel<<<C, mo::ROUTE_THREADS, 0, s>>>(expert_ids, num_pairs, E, chunk, base, dest,
                                                          src);
    e = cudaGetLastError();
    return e == cudaSuccess ? ok() : cuda_fail(e, "launching the route kernels");
}

nvfp4_status nvfp4_moe_permute_rows(const void* in, size_t row_bytes, int in_rows, int num_pairs,
                                    int k, const int32_t* src, void* out, void* stream) {
    if (in_rows < 0 || num_pairs < 0 || k < 1)
        return fail(NVFP4_ERR_INVALID_ARG, "in_rows, num_pairs >= 0 and k >= 1 required");
    if (row_bytes == 0 || row_bytes % 16 != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "row_bytes must be a positive multiple of 16 (got %zu)",
                    row_bytes);
    if (num_pairs == 0) return ok();
    if (!in || !src || !out) return fail(NVFP4_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned16(in) || !aligned16(out))
        return fail(NVFP4_ERR_MISALIGNED, "in and out must be 16-byte aligned");
    nvfp4::moe::permute_rows_kernel<<<(num_pairs + 7) / 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint8_t*>(in), row_bytes, in_rows, num_pairs, k, src,
        static_cast<uint8_t*>(out));
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ok() : cuda_fail(e, "launching permute_rows_kernel");
}

nvfp4_status nvfp4_moe_combine(const void* Yg, int num_pairs, const int32_t* dest,
                               const float* weights, int T, int k, int N, void* Y, void* stream) {
    if (T < 0 || num_pairs < 0 || k < 1 || N < 0)
        return fail(NVFP4_ERR_INVALID_ARG, "T, num_pairs, N >= 0 and k >= 1 required");
    if (N % 8 != 0) return fail(NVFP4_ERR_INVALID_ARG, "N must be a multiple of 8 (got %d)", N);
    if (T == 0 || N == 0) return ok();
    if (!dest || !Y || (num_pairs > 0 && !Yg)) return fail(NVFP4_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned16(Y) || (Yg && !aligned16(Yg)))
        return fail(NVFP4_ERR_MISALIGNED, "Yg and Y must be 16-byte aligned");
    const int cols = (N / 8 + 255) / 256;
    const dim3 grid(cols, T < 65535 ? T : 65535);
    nvfp4::moe::combine_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16*>(Yg), num_pairs, dest, weights, T, k, N,
        static_cast<__nv_bfloat16*>(Y));
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ok() : cuda_fail(e, "launching combine_kernel");
}

// ------------------------------------------------------------------------- W4A16
nvfp4_status gemm_w4a16(const void* A, const uint8_t* W, const uint8_t* sW, float gW, void* Y,
                        int M, int N, int K, void* stream) {
    namespace k16 = nvfp4::w4a16;
    if (M < 0 || N < 0) return fail(NVFP4_ERR_INVALID_ARG, "M and N must be >= 0 (got %d, %d)", M, N);
    if (K < 32 || K % 32 != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "K must be a positive multiple of 32 (got %d)", K);
    if (M > 0 && N > 0) {
        if (!A || !W || !sW || !Y) return fail(NVFP4_ERR_INVALID_ARG, "null pointer argument");
        if (!aligned16(A) || !aligned16(W) || !aligned16(sW) || !aligned16(Y))
            return fail(NVFP4_ERR_MISALIGNED, "every buffer must be 16-byte aligned");
    }
    int dev;
    DevInfo info;
    if (!current_device(dev, info)) return fail(NVFP4_ERR_CUDA, "cannot query the current CUDA device");
    if (nvfp4_exec_of_arch(info.sm_arch, NVFP4_FMT_NVFP4, NVFP4_FMT_BF16, 0) != NVFP4_EXEC_BF16_WIDEN)
        return fail(NVFP4_ERR_NOPATH, "W4A16 has no BF16-widen kernel for sm_%d", info.sm_arch);
    if (M == 0 || N == 0) return ok();

    // one wave: blocks of 8 weight rows spread evenly over the SMs, at most
    // LDG_MAX_NB per CTA (more CTAs than SMs only for very tall W)
    const int nrb = (N + k16::ROWS - 1) / k16::ROWS;
    int grid = nrb < info.num_sms ? nrb : info.num_sms;
    int nb = (nrb + grid - 1) / grid;
    if (nb > k16::LDG_MAX_NB) {
        nb = k16::LDG_MAX_NB;
        grid = (nrb + nb - 1) / nb;
    }
    W4a16LdgKern kern = w4a16_ldg_kernel_for(nb);
    const float out_scale = 128.0f * gW;  // undoes the 2^-7 carried by the widened weights
    for (int m0 = 0; m0 < M; m0 += k16::TOK) {
        const int mc = M - m0 < k16::TOK ? M - m0 : k16::TOK;
        const uint16_t* a = static_cast<const uint16_t*>(A) + (size_t)m0 * K;
        __nv_bfloat16* y = static_cast<__nv_bfloat16*>(Y) + (size_t)m0 * N;
        kern<<<grid, k16::LDG_THREADS, 0, static_cast<cudaStream_t>(stream)>>>(
            a, W, sW, y, mc, N, K, out_scale, nrb);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "launching w4a16_ldg_kernel");
    }
    return ok();
}

// ------------------------------------------------------------------------- grouped W4A4
nvfp4_status gemm_nvfp4_w4a4_grouped_host(const uint8_t* A, const uint8_t* sA, float gA,
                                          const uint8_t* W, const uint8_t* sW,
                                          const float* gW_host, const int32_t* offsets_host, int E,
                                          void* Y, int N, int K, void* stream) {
    namespace gk = nvfp4::grouped;
    if (E < 1 || E > gk::MAX_EXPERTS)
        return fail(NVFP4_ERR_INVALID_ARG, "E must be in [1, %d] (got %d)", gk::MAX_EXPERTS, E);
    if (!offsets_host || !gW_host) return fail(NVFP4_ERR_INVALID_ARG, "null offsets or gW");
    if (offsets_host[0] != 0) return fail(NVFP4_ERR_INVALID_ARG, "offsets[0] must be 0");
    for (int e = 0; e < E; ++e)
        if (offsets_host[e + 1] < offsets_host[e])
            return fail(NVFP4_ERR_INVALID_ARG, "offsets must be non-decreasing");
    const int M = offsets_host[E];
    nvfp4_status st = check_w4a4_args(A, sA, W, sW, Y, M, N, K);
    if (st != NVFP4_OK) return st;
    if (K % gk::BK != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "the grouped path needs K %% 256 == 0 (got %d)", K);
    if ((int64_t)E * N > INT32_MAX) return fail(NVFP4_ERR_INVALID_ARG, "E*N too large");
    int dev;
    DevInfo info;
    if ((st = check_fp4_path(dev, info)) != NVFP4_OK) return st;
    if (M == 0 || N == 0) return ok();

    gk::Params prm;
    memset(&prm, 0, sizeof(prm));
    prm.E = E;
    prm.N = N;
    prm.K = K;
    int64_t total = 0;
    for (int e = 0; e < E; ++e) {
        prm.tile_start[e] = (int)total;
        prm.row_start[e] = offsets_host[e];
        prm.alpha[e] = gA * gW_host[e];
        total += gk::tiles_of_expert(offsets_host[e + 1] - offsets_host[e], N);
    }
    if (total > INT32_MAX) return fail(NVFP4_ERR_INVALID_ARG, "too many tiles");
    prm.tile_start[E] = (int)total;
    prm.row_start[E] = M;

    CUtensorMap tmA, tmW256, tmW128, tmSA, tmSW256, tmSW128;
    const uint64_t wrows = (uint64_t)E * N;
    if ((st = make_map_u8(&tmA, A, (uint64_t)K / 2, (uint64_t)M, gk::BKB, gk::BM)) != NVFP4_OK) return st;
    if ((st = make_map_u8(&tmW256, W, (uint64_t)K / 2, wrows, gk::BKB, gk::BN)) != NVFP4_OK) return st;
    if ((st = make_map_u8(&tmW128, W, (uint64_t)K / 2, wrows, gk::BKB, gk::SBN)) != NVFP4_OK) return st;
    if ((st = make_map_u8(&tmSA, sA, (uint64_t)K / 16, (uint64_t)M, 16, gk::BM,
                          CU_TENSOR_MAP_SWIZZLE_NONE)) != NVFP4_OK)
        return st;
    if ((st = make_map_u8(&tmSW256, sW, (uint64_t)K / 16, wrows, 16, gk::BN,
                          CU_TENSOR_MAP_SWIZZLE_NONE)) != NVFP4_OK)
        return st;
    if ((st = make_map_u8(&tmSW128, sW, (uint64_t)K / 16, wrows, 16, gk::SBN,
                          CU_TENSOR_MAP_SWIZZLE_NONE)) != NVFP4_OK)
        return st;
    if ((st = set_smem(gk::grouped_kernel, gk::C::SMEM_BYTES, info, "grouped_kernel")) != NVFP4_OK)
        return st;
    const int grid = total < info.num_sms ? (int)total : info.num_sms;
    gk::grouped_kernel<<<grid, gk::NUM_THREADS, gk::C::SMEM_BYTES, static_cast<cudaStream_t>(stream)>>>(
        tmA, tmW256, tmW128, tmSA, tmSW256, tmSW128, prm, reinterpret_cast<__nv_bfloat16*>(Y));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launching grouped_kernel");
    return ok();
}

// ------------------------------------------------------------------------- grouped, packed scales
size_t nvfp4_grouped_scale_layout_bytes(const int32_t* offsets_host, int E, int K) {
    if (K < 64 || K % 64 != 0 || !offsets_host || E < 1 || E > nvfp4::pack::MAX_GROUPS) return 0;
    if (offsets_host[0] != 0) return 0;
    for (int e = 0; e < E; ++e)
        if (offsets_host[e + 1] < offsets_host[e]) return 0;
    return (size_t)grouped_blocks(offsets_host, E) * 128 * (size_t)(K / 16);
}

nvfp4_status nvfp4_pack_scales_grouped(const uint8_t* s_plain, const int32_t* offsets_host, int E,
                                       int K, uint8_t* s_packed, void* stream) {
    namespace pk = nvfp4::pack;
    int M = 0;
    nvfp4_status st = check_offsets(offsets_host, E, pk::MAX_GROUPS, M);
    if (st != NVFP4_OK) return st;
    if (K < 64 || K % 64 != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "packing needs K %% 64 == 0 (got %d)", K);
    if (M == 0) return ok();
    if (!s_plain || !s_packed) return fail(NVFP4_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned16(s_plain) || !aligned16(s_packed))
        return fail(NVFP4_ERR_MISALIGNED, "s_plain and s_packed must be 16-byte aligned");
    pk::GroupedPack gp;
    memset(&gp, 0, sizeof(gp));
    gp.groups_n = E;
    int64_t blocks = 0;
    for (int e = 0; e <= E; ++e) {
        gp.row_start[e] = offsets_host[e];
        gp.block_start[e] = (int)blocks;
        if (e < E) blocks += (offsets_host[e + 1] - offsets_host[e] + 127) / 128;
    }
    const int ksteps = K / 64;
    const dim3 grid((unsigned)blocks, (unsigned)((ksteps + pk::KCHUNK - 1) / pk::KCHUNK));
    if (grid.y > 65535) return fail(NVFP4_ERR_INVALID_ARG, "K too large for packing");
    pk::pack_scales_grouped_kernel<<<grid, pk::ROWS, 0, static_cast<cudaStream_t>(stream)>>>(
        s_plain, s_packed, gp, nullptr, K / 16, ksteps);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launching pack_scales_grouped_kernel");
    return ok();
}

nvfp4_status gemm_nvfp4_w4a4_grouped_packed(const uint8_t* A, const uint8_t* sA_packed, float gA,
                                            const uint8_t* W, const uint8_t* sW_packed,
                                            const float* gW_host, const int32_t* offsets_host,
                                            int E, void* Y, int N, int K, void* stream) {
    namespace gp = nvfp4::grouped_pair;
    int M = 0;
    nvfp4_status st = check_offsets(offsets_host, E, gp::MAX_EXPERTS, M);
    if (st != NVFP4_OK) return st;
    if (!gW_host) return fail(NVFP4_ERR_INVALID_ARG, "null gW");
    if ((st = check_w4a4_args(A, sA_packed, W, sW_packed, Y, M, N, K)) != NVFP4_OK) return st;
    if (K % gp::BK != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "the grouped path needs K %% 256 == 0 (got %d)", K);
    if ((int64_t)E * N > INT32_MAX) return fail(NVFP4_ERR_INVALID_ARG, "E*N too large");
    int dev;
    DevInfo info;
    if ((st = check_fp4_path(dev, info)) != NVFP4_OK) return st;
    if (M == 0 || N == 0) return ok();
    if (info.num_sms < 2) return fail(NVFP4_ERR_CUDA, "the pair kernel needs at least two SMs");

    gp::Params prm;
    memset(&prm, 0, sizeof(prm));
    prm.E = E;
    prm.N = N;
    prm.K = K;
    int64_t total = 0, blocks = 0;
    for (int e = 0; e < E; ++e) {
        const int Me = offsets_host[e + 1] - offsets_host[e];
        prm.tile_start[e] = (int)total;
        prm.row_start[e] = offsets_host[e];
        prm.block_start[e] = (int)blocks;
        prm.alpha[e] = gA * gW_host[e];
        total += gp::tiles_of_expert(Me, N);
        blocks += (Me + 127) / 128;
    }
    if (total > INT32_MAX) return fail(NVFP4_ERR_INVALID_ARG, "too many tiles");
    prm.tile_start[E] = (int)total;
    prm.row_start[E] = M;
    prm.block_start[E] = (int)blocks;

    CUtensorMap tmA, tmA64, tmW, tmSA, tmSW2, tmSW1;
    const uint64_t ks = (uint64_t)K / 64;
    const uint64_t wblocks = (uint64_t)E * ((N + 127) / 128);
    if ((st = make_map_u8(&tmA, A, (uint64_t)K / 2, (uint64_t)M, gp::BKB, gp::BM)) != NVFP4_OK) return st;
    if ((st = make_map_u8(&tmA64, A, (uint64_t)K / 2, (uint64_t)M, gp::BKB, gp::SWAP_HALF)) != NVFP4_OK)
        return st;
    if ((st = make_map_u8(&tmW, W, (uint64_t)K / 2, (uint64_t)E * N, gp::BKB, gp::BNH)) != NVFP4_OK)
        return st;
    if ((st = make_map_packed_sf(&tmSA, sA_packed, (uint64_t)blocks, ks, 1)) != NVFP4_OK) return st;
    if ((st = make_map_packed_sf(&tmSW2, sW_packed, wblocks, ks, gp::NRB)) != NVFP4_OK) return st;
    if ((st = make_map_packed_sf(&tmSW1, sW_packed, wblocks, ks, 1)) != NVFP4_OK) return st;
    CUtensorMap tmY;
    int tma_out = 0;
    if ((st = make_map_out(&tmY, Y, (uint64_t)M, (uint64_t)N, tma_out)) != NVFP4_OK) return st;
    if ((st = set_smem(gp::grouped_pair_kernel, gp::SMEM_BYTES, info, "grouped_pair_kernel")) != NVFP4_OK)
        return st;
    const int pairs = total < info.num_sms / 2 ? (int)total : info.num_sms / 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(gp::NUM_THREADS);
    cfg.dynamicSmemBytes = gp::SMEM_BYTES;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // may start while the stream's previous kernel (the scale packing) finishes; the
    // kernel waits for it before reading anything it wrote
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, gp::grouped_pair_kernel, tmA, tmA64, tmW, tmSA, tmSW2,
                                       tmSW1, tmY, tma_out, prm, (const gp::Params*)nullptr,
                                       reinterpret_cast<__nv_bfloat16*>(Y), (const int32_t*)nullptr,
                                       (const float*)nullptr, 0);
    if (e != cudaSuccess) return cuda_fail(e, "launching grouped_pair_kernel");
    return ok();
}

// ------------------------------------------------------------------------- grouped, device offsets
size_t nvfp4_grouped_sched_bytes(void) {
    return ((sizeof(nvfp4::grouped_pair::Params) + 255) / 256) * 256 +
           ((sizeof(nvfp4::pack::GroupedPack) + 255) / 256) * 256;
}

size_t nvfp4_grouped_scale_layout_bytes_bound(int M, int E, int K) {
    if (M < 0 || E < 1 || K < 64 || K % 64 != 0) return 0;
    return ((size_t)(M + 127) / 128 + (size_t)E) * 128 * (size_t)(K / 16);
}

namespace {
nvfp4::grouped_pair::Params* sched_params(void* sched) {
    return static_cast<nvfp4::grouped_pair::Params*>(sched);
}
nvfp4::pack::GroupedPack* sched_pack(void* sched) {
    return reinterpret_cast<nvfp4::pack::GroupedPack*>(
        static_cast<uint8_t*>(sched) + ((sizeof(nvfp4::grouped_pair::Params) + 255) / 256) * 256);
}
}  // namespace

nvfp4_status nvfp4_grouped_schedule(const int32_t* offsets_dev, int E, int M, int N, int K,
                                    const float* gA_dev, float gA, const float* gW_host,
                                    void* sched, void* stream) {
    namespace gp = nvfp4::grouped_pair;
    if (E < 1 || E > gp::MAX_EXPERTS)
        return fail(NVFP4_ERR_INVALID_ARG, "E must be in [1, %d] (got %d)", gp::MAX_EXPERTS, E);
    if (M < 0 || N < 1 || K < gp::BK || K % gp::BK != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "M >= 0, N >= 1 and K %% 256 == 0 required");
    if (!offsets_dev || !gW_host || !sched) return fail(NVFP4_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned16(sched)) return fail(NVFP4_ERR_MISALIGNED, "the schedule buffer must be 16-byte aligned");
    gp::GwArray gw;
    memset(&gw, 0, sizeof(gw));
    for (int e = 0; e < E; ++e) gw.v[e] = gW_host[e];
    gp::grouped_schedule_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        offsets_dev, E, M, N, K, gA_dev, gA, gw, sched_params(sched), sched_pack(sched));
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ok() : cuda_fail(e, "launching grouped_schedule_kernel");
}

nvfp4_status nvfp4_pack_scales_grouped_sched(const uint8_t* s_plain, int M, int E, int K,
                                             const void* sched, uint8_t* s_packed, void* stream) {
    namespace pk = nvfp4::pack;
    if (M < 0 || E < 1 || E > pk::MAX_GROUPS)
        return fail(NVFP4_ERR_INVALID_ARG, "M >= 0 and E in [1, %d] required", pk::MAX_GROUPS);
    if (K < 64 || K % 64 != 0) return fail(NVFP4_ERR_INVALID_ARG, "packing needs K %% 64 == 0 (got %d)", K);
    if (M == 0) return ok();
    if (!s_plain || !s_packed || !sched) return fail(NVFP4_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned16(s_plain) || !aligned16(s_packed))
        return fail(NVFP4_ERR_MISALIGNED, "s_plain and s_packed must be 16-byte aligned");
    pk::GroupedPack none;
    memset(&none, 0, sizeof(none));
    const int ksteps = K / 64;
    const dim3 grid((unsigned)((M + 127) / 128 + E), (unsigned)((ksteps + pk::KCHUNK - 1) / pk::KCHUNK));
    if (grid.y > 65535) return fail(NVFP4_ERR_INVALID_ARG, "K too large for packing");
    pk::pack_scales_grouped_kernel<<<grid, pk::ROWS, 0, static_cast<cudaStream_t>(stream)>>>(
        s_plain, s_packed, none, sched_pack(const_cast<void*>(sched)), K / 16, ksteps);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ok() : cuda_fail(e, "launching pack_scales_grouped_kernel");
}

namespace {
// The device-scheduled grouped product; with row_dest, grouped row r is written to
// Y row row_dest[r] (of dest_rows), times row_w[that row] if row_w is given.
nvfp4_status launch_grouped_sched(const uint8_t* A, const uint8_t* sA_packed, const uint8_t* W,
                                  const uint8_t* sW_packed, const void* sched, int E, int M, void* Y,
                                  int N, int K, const int32_t* row_dest, const float* row_w,
                                  int dest_rows, void* stream) {
    namespace gp = nvfp4::grouped_pair;
    if (E < 1 || E > gp::MAX_EXPERTS)
        return fail(NVFP4_ERR_INVALID_ARG, "E must be in [1, %d] (got %d)", gp::MAX_EXPERTS, E);
    nvfp4_status st = check_w4a4_args(A, sA_packed, W, sW_packed, Y, M, N, K);
    if (st != NVFP4_OK) return st;
    if (K % gp::BK != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "the grouped path needs K %% 256 == 0 (got %d)", K);
    if ((int64_t)E * N > INT32_MAX) return fail(NVFP4_ERR_INVALID_ARG, "E*N too large");
    if (!sched) return fail(NVFP4_ERR_INVALID_ARG, "null schedule");
    int dev;
    DevInfo info;
    if ((st = check_fp4_path(dev, info)) != NVFP4_OK) return st;
    if (M == 0 || N == 0) return ok();
    if (info.num_sms < 2) return fail(NVFP4_ERR_CUDA, "the pair kernel needs at least two SMs");
    CUtensorMap tmA, tmA64, tmW, tmSA, tmSW2, tmSW1;
    const uint64_t ks = (uint64_t)K / 64;
    const uint64_t wblocks = (uint64_t)E * ((N + 127) / 128);
    const uint64_t ablocks = (uint64_t)(M + 127) / 128 + (uint64_t)E;  // the packed sA bound
    if ((st = make_map_u8(&tmA, A, (uint64_t)K / 2, (uint64_t)M, gp::BKB, gp::BM)) != NVFP4_OK) return st;
    if ((st = make_map_u8(&tmA64, A, (uint64_t)K / 2, (uint64_t)M, gp::BKB, gp::SWAP_HALF)) != NVFP4_OK)
        return st;
    if ((st = make_map_u8(&tmW, W, (uint64_t)K / 2, (uint64_t)E * N, gp::BKB, gp::BNH)) != NVFP4_OK)
        return st;
    if ((st = make_map_packed_sf(&tmSA, sA_packed, ablocks, ks, 1)) != NVFP4_OK) return st;
    if ((st = make_map_packed_sf(&tmSW2, sW_packed, wblocks, ks, gp::NRB)) != NVFP4_OK) return st;
    if ((st = make_map_packed_sf(&tmSW1, sW_packed, wblocks, ks, 1)) != NVFP4_OK) return st;
    CUtensorMap tmY;
    int tma_out = 0;
    if ((st = make_map_out(&tmY, Y, (uint64_t)(row_dest ? dest_rows : M), (uint64_t)N, tma_out)) !=
        NVFP4_OK)
        return st;
    if ((st = set_smem(gp::grouped_pair_kernel, gp::SMEM_BYTES, info, "grouped_pair_kernel")) != NVFP4_OK)
        return st;
    gp::Params none;
    memset(&none, 0, sizeof(none));
    // the tile count is on the device: one cluster per SM pair, idle clusters return
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (info.num_sms / 2));
    cfg.blockDim = dim3(gp::NUM_THREADS);
    cfg.dynamicSmemBytes = gp::SMEM_BYTES;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // may start while the stream's previous kernel (the scale packing) finishes; the
    // kernel waits for it before reading anything it wrote
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, gp::grouped_pair_kernel, tmA, tmA64, tmW, tmSA, tmSW2,
                                       tmSW1, tmY, tma_out, none,
                                       (const gp::Params*)sched_params(const_cast<void*>(sched)),
                                       reinterpret_cast<__nv_bfloat16*>(Y), row_dest, row_w,
                                       dest_rows);
    if (e != cudaSuccess) return cuda_fail(e, "launching grouped_pair_kernel");
    return ok();
}
}  // namespace

nvfp4_status gemm_nvfp4_w4a4_grouped_packed_sched(const uint8_t* A, const uint8_t* sA_packed,
                                                  const uint8_t* W, const uint8_t* sW_packed,
                                                  const void* sched, int E, int M, void* Y, int N,
                                                  int K, void* stream) {
    return launch_grouped_sched(A, sA_packed, W, sW_packed, sched, E, M, Y, N, K, nullptr, nullptr,
                                0, stream);
}

nvfp4_status gemm_nvfp4_w4a4_grouped_packed_sched_combine(const uint8_t* A,
                                                          const uint8_t* sA_packed, const uint8_t* W,
                                                          const uint8_t* sW_packed, const void* sched,
                                                          int E, int M, const int32_t* src,
                                                          const float* weights, void* Y, int T,
                                                          int N, int K, void* stream) {
    if (M > 0 && !src) return fail(NVFP4_ERR_INVALID_ARG, "null src");
    if (T < 0 || M > T) return fail(NVFP4_ERR_INVALID_ARG, "top-1 needs M <= T (got M %d, T %d)", M, T);
    if (N % 2 != 0) return fail(NVFP4_ERR_INVALID_ARG, "the fused combine needs an even N (got %d)", N);
    return launch_grouped_sched(A, sA_packed, W, sW_packed, sched, E, M, Y, N, K, src, weights, T,
                                stream);
}


// ------------------------------------------------------------------------- grouped W4A4 from plain
// scales and device offsets: schedule, pack both scale matrices, product
namespace {
size_t round256(size_t b) { return (b + 255) / 256 * 256; }
// Offsets of the three parts of the grouped entry's workspace.
struct GroupedWs {
    size_t sched = 0, sa = 0, sw = 0, total = 0;
};
bool grouped_ws_layout(int M, int N, int K, int E, GroupedWs& w) {
    if (M < 0 || N < 1 || E < 1 || E > nvfp4::grouped_pair::MAX_EXPERTS || K < 256 || K % 256 != 0)
        return false;
    w.sched = 0;
    w.sa = round256(nvfp4_grouped_sched_bytes());
    w.sw = w.sa + round256(nvfp4_grouped_scale_layout_bytes_bound(M, E, K));
    w.total = w.sw + round256((size_t)E * (size_t)((N + 127) / 128) * 128 * (size_t)(K / 16));
    return true;
}
}  // namespace

nvfp4_status gemm_nvfp4_w4a4_grouped(const uint8_t* A, const uint8_t* sA, float gA,
                                     const uint8_t* W, const uint8_t* sW, const float* gW_host,
                                     const int32_t* offsets_dev, int E, int total_M, void* Y,
                                     int N, int K, void* workspace, size_t ws_bytes,
                                     void* stream) {
    namespace gp = nvfp4::grouped_pair;
    if (E < 1 || E > gp::MAX_EXPERTS)
        return fail(NVFP4_ERR_INVALID_ARG, "E must be in [1, %d] (got %d)", gp::MAX_EXPERTS, E);
    nvfp4_status st = check_w4a4_args(A, sA, W, sW, Y, total_M, N, K);
    if (st != NVFP4_OK) return st;
    if (K % gp::BK != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "the grouped path needs K %% 256 == 0 (got %d)", K);
    if ((int64_t)E * N > INT32_MAX) return fail(NVFP4_ERR_INVALID_ARG, "E*N too large");
    if (!offsets_dev || !gW_host) return fail(NVFP4_ERR_INVALID_ARG, "null offsets or gW");
    GroupedWs w;
    if (!grouped_ws_layout(total_M, N, K, E, w)) return fail(NVFP4_ERR_INVALID_ARG, "bad sizes");
    if (total_M == 0 || N == 0) return ok();
    if (!workspace || ws_bytes < w.total)
        return fail(NVFP4_ERR_INVALID_ARG,
                    "the workspace must hold nvfp4_workspace_size(NVFP4_OP_W4A4_GROUPED, ...) = %zu "
                    "bytes (got %zu)", w.total, ws_bytes);
    if (!aligned16(workspace)) return fail(NVFP4_ERR_MISALIGNED, "the workspace must be 16-byte aligned");
    int dev;
    DevInfo info;
    if ((st = check_fp4_path(dev, info)) != NVFP4_OK) return st;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    void* sched = ws + w.sched;
    uint8_t* sa_packed = ws + w.sa;
    uint8_t* sw_packed = ws + w.sw;
    // the weights' groups: E experts of N rows each
    int32_t woff[nvfp4::grouped_pair::MAX_EXPERTS + 1];
    for (int e = 0; e <= E; ++e) woff[e] = e * N;
    if ((st = nvfp4_grouped_schedule(offsets_dev, E, total_M, N, K, nullptr, gA, gW_host, sched,
                                     stream)) != NVFP4_OK)
        return st;
    if ((st = nvfp4_pack_scales_grouped_sched(sA, total_M, E, K, sched, sa_packed, stream)) != NVFP4_OK)
        return st;
    if ((st = nvfp4_pack_scales_grouped(sW, woff, E, K, sw_packed, stream)) != NVFP4_OK) return st;
    return launch_grouped_sched(A, sa_packed, W, sw_packed, sched, E, total_M, Y, N, K, nullptr,
                                nullptr, 0, stream);
}

// ------------------------------------------------------------------------- generic queries
size_t nvfp4_workspace_size(int op, int M, int N, int K, int E) {
    switch (op) {
        case NVFP4_OP_W4A4:
        case NVFP4_OP_VIA_FP8:
        case NVFP4_OP_W4A16:
        case NVFP4_OP_W4A8:
            return 0;
        case NVFP4_OP_W4A4_GROUPED: {
            GroupedWs w;
            return grouped_ws_layout(M, N, K, E, w) ? w.total : 0;
        }
        case NVFP4_OP_W4A4_PACKED:
            return nvfp4_w4a4_packed_workspace_bytes(M, N, K, 0);
        case NVFP4_OP_QUANTIZE:
            return nvfp4_quantize_workspace_bytes();
        case NVFP4_OP_MOE_ROUTE:
            return nvfp4_moe_route_workspace_bytes(M, E);
        default:
            return SIZE_MAX;
    }
}

nvfp4_status nvfp4_prepare_scales(const uint8_t* s_plain, uint8_t* s_mma, int rows, int K,
                                  void* stream) {
    return nvfp4_pack_scales(s_plain, rows, K, s_mma, stream);
}

#ifdef NVFP4_WAIT_TEST
// Test-only build: sets the pipeline waits' time limit and the stall switch of
// the single-SM W4A4 kernel on the current device.  Not in the product library.
__attribute__((visibility("default"))) nvfp4_status nvfp4_test_set_wait(uint64_t limit_ns,
                                                                        int stall) {
    cudaError_t e = cudaMemcpyToSymbol(nvfp4::g_wait_limit_ns, &limit_ns, sizeof(limit_ns));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(nvfp4::g_wait_test_stall, &stall, sizeof(stall));
    return e == cudaSuccess ? ok() : cuda_fail(e, "setting the test wait variables");
}
#endif

}  // extern "C"
