/*
 * nvfp4.h -- C ABI of the B200 (sm_100a) block-scaled NVFP4 matmul library.
 *
 * The operation (metrale_circuit `hardware::exec` module doc, bullets 1-2; the
 * NVFP4 formats it names):
 *
 *     Y[m,n] = BF16( alpha * sum_g sA[m,g]*sW[n,g] * sum_{k in g} a[m,k]*w[n,k] )
 *
 * where a, w are E2M1 (FP4) values, g runs over groups of 16 consecutive k,
 * sA, sW are E4M3 group scales, alpha = gA*gW is the product of the two FP32
 * per-tensor scales, accumulation is FP32 and the output is BF16 (round to
 * nearest even).  The declared formats are never widened (module doc,
 * Invariants): a format pair that has neither a native kernel nor an exact
 * conversion here is reported as NVFP4_EXEC_NO_PATH, and every matmul entry
 * point refuses it.
 *
 * Layouts (all row-major, contiguous, no padding):
 *   A      uint8 [M][K/2]   E2M1 codes, two per byte, even k in the low nibble
 *   W      uint8 [N][K/2]   same; W is stored [N,K] so Y = A . W^T (TN)
 *   sA     uint8 [M][K/16]  E4M3 group scales, finite and non-negative (0x00..0x7E)
 *   sW     uint8 [N][K/16]  same
 *   Y      bf16  [M][N]
 * Every pointer is a DEVICE pointer, owned by the caller, and must be 16-byte
 * aligned.  The library allocates no device memory in any call; kernels
 * allocate and free their own tensor memory (TMEM) on chip.
 *
 * Calls are asynchronous on `stream` (a cudaStream_t; 0 = legacy default
 * stream).  NVFP4_OK means "enqueued".  Argument errors are detected on the
 * host before anything is enqueued.  A kernel whose internal wait exceeds its
 * time limit records a device error word and exits without hanging; it is
 * read (and cleared) by nvfp4_check_device_error().
 *
 * Thread safety: every entry point may be called from several host threads;
 * the only global state is a mutex-protected per-device capability cache and
 * the per-thread last-error string.
 */
#ifndef NVFP4_B200_H
#define NVFP4_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,     /* bad size, null pointer, bad enum, K % 32 != 0 ... */
    NVFP4_ERR_MISALIGNED = 2,      /* a pointer is not 16-byte aligned */
    NVFP4_ERR_NOPATH = 3,          /* the declared pair has no path on this device */
    NVFP4_ERR_NO_FP4_KERNEL = 4,   /* device has the FP4 MMA but no kernel is compiled for it */
    NVFP4_ERR_CUDA = 5,            /* a CUDA runtime/driver call failed (see nvfp4_last_error) */
    NVFP4_ERR_DEVICE_TIMEOUT = 6   /* a kernel's bounded wait expired (nvfp4_check_device_error) */
} nvfp4_status;

/* Declared operand formats (module doc, bullet 1: the activation format picks
 * the MMA kind). */
typedef enum {
    NVFP4_FMT_BF16 = 0,
    NVFP4_FMT_FP8_E4M3 = 1,
    NVFP4_FMT_NVFP4 = 2
} nvfp4_fmt;

/* The MMA kind an activation format needs (`kind_of`). */
typedef enum {
    NVFP4_KIND_BF16_MMA = 0,       /* BF16 activations; weights widened in registers */
    NVFP4_KIND_FP8_MMA = 1,
    NVFP4_KIND_FP4_BLOCK_SCALED = 2,
    NVFP4_KIND_INVALID = -1
} nvfp4_kind;

/* How a device executes a declared (weight, activation) pair (`enum Exec`). */
typedef enum {
    NVFP4_EXEC_FP4_MMA = 0,        /* block-scaled FP4 MMA: gemm_nvfp4_w4a4 */
    NVFP4_EXEC_FP8_EXACT = 1,      /* exact E2M1->E4M3 conversion on the FP8 MMA: gemm_nvfp4_via_fp8 (W4A4), gemm_nvfp4_w4a8 (W4A8) */
    NVFP4_EXEC_BF16_WIDEN = 2,     /* BF16 MMA, NVFP4 weights widened in registers: gemm_w4a16 */
    NVFP4_EXEC_NO_FP4_KERNEL = 3,  /* device has the FP4 MMA, but its class has no compiled kernel */
    NVFP4_EXEC_NO_PATH = 4         /* neither native nor exact: refused, never widened */
} nvfp4_exec;

/* ---- planning (host only, no device work) -------------------------------- */

/* kind_of: the MMA kind `activation` needs.  NVFP4_KIND_INVALID for a bad enum. */
NVFP4_API nvfp4_kind nvfp4_kind_of(nvfp4_fmt activation);

/* exec_of for a device CLASS given by its compute capability (e.g. 100 for
 * sm_100, 90 for sm_90, 120 for sm_120).  Pure function; usable without a GPU.
 * (NVFP4, NVFP4): FP4_MMA where this library compiles its block-scaled kernel
 * for the class (sm_100 only), NO_FP4_KERNEL on other classes that have the
 * FP4 MMA (sm_101/103/110/120/121), FP8_EXACT on a class without the FP4 MMA
 * but with the FP8 MMA for which this library compiles the exact-path kernel
 * (none besides sm_100, so NO_PATH on sm_89/sm_90), NO_PATH otherwise.
 * (NVFP4, BF16): BF16_WIDEN on sm_100, NO_PATH elsewhere.
 * (NVFP4, FP8) (W4A8): no single-instruction MMA takes FP8 activations under
 * NVFP4 weights with E4M3 group-16 scales, so the exact E4M3 path: FP8_EXACT on
 * sm_100 (gemm_nvfp4_w4a8), NO_PATH on every other class.
 * Pairs whose weights are not NVFP4: NO_PATH (this library carries NVFP4-weight
 * paths only).  `fp4_kernel_disabled` != 0 behaves as if the class compiled no
 * FP4 block-scale kernel (module doc, `fp4_fallback`, `avail::without_fp4_kernel`). */
NVFP4_API nvfp4_exec nvfp4_exec_of_arch(int sm_arch, nvfp4_fmt weight, nvfp4_fmt activation,
                              int fp4_kernel_disabled);

/* exec_of for CUDA device `device` (queries its compute capability; NO_PATH if
 * the device cannot be queried).  Honors nvfp4_set_fp4_kernel_disabled(). */
NVFP4_API nvfp4_exec nvfp4_exec_of(int device, nvfp4_fmt weight, nvfp4_fmt activation);

/* fp4_fallback (metrale_circuit `hardware::exec`, fp4_fallback): how an NVFP4
 * activation runs on class `sm_arch` when no FP4 block-scale kernel is
 * compiled for it.  NO_FP4_KERNEL where the class's tensor cores do FP4 but no
 * kernel for it is compiled (sm_100 with the switch below, sm_101/103/110/120/121);
 * FP8_EXACT on a class without the FP4 MMA that has the FP8 MMA and this
 * library's exact-path kernel (none besides sm_100, so in practice never);
 * NO_PATH otherwise.  Pure function; usable without a GPU. */
NVFP4_API nvfp4_exec nvfp4_fp4_fallback(int sm_arch);

/* node_exec over a list of weight-reading nodes (metrale_circuit
 * `hardware::exec`, node_exec): exec_out[i] is how node i, declared as
 * (weight_fmt[i], activation_fmt[i]), runs on class `sm_arch`.  That is
 * exec_of's answer, or fp4_fallback's where the class compiles no FP4
 * block-scale kernel (fp4_kernel_disabled != 0 mimics such a class).  Format
 * values outside nvfp4_fmt give NO_PATH for their node.  The arrays are host
 * memory of n int32 each, read or written during the call only.  Returns
 * NVFP4_ERR_INVALID_ARG for n < 0 or a null array with n > 0; n == 0 is OK.
 * A declared format is never planned at a wider one: a node's answer is
 * FP4_MMA only for NVFP4 activations, FP8_EXACT only for NVFP4 weights under
 * NVFP4 or FP8 activations, BF16_WIDEN only for BF16 activations. */
NVFP4_API nvfp4_status nvfp4_node_exec(int sm_arch, int fp4_kernel_disabled,
                                       const int32_t* weight_fmt, const int32_t* activation_fmt,
                                       int n, int32_t* exec_out);

/* Process-wide switch that mimics a device class without a compiled FP4
 * block-scale kernel (for planning tests): while set, exec_of reports
 * NO_FP4_KERNEL for (NVFP4, NVFP4) and gemm_nvfp4_w4a4 / the grouped entry
 * return NVFP4_ERR_NO_FP4_KERNEL without enqueueing anything. */
NVFP4_API void nvfp4_set_fp4_kernel_disabled(int disabled);

/* pair_name: the declared pair as "W4A16"-style text ("W4A4", "W4A8", "W16A16"
 * ...).  Static storage; "?" for a bad enum. */
NVFP4_API const char* nvfp4_pair_name(nvfp4_fmt weight, nvfp4_fmt activation);

/* Human-readable name of an nvfp4_exec value (static storage). */
NVFP4_API const char* nvfp4_exec_name(nvfp4_exec e);

/* ---- matmuls --------------------------------------------------------------- */

/* W4A4 on the block-scaled FP4 MMA (metrale_circuit `hardware::exec` module
 * doc, bullet 1, the NVFP4 row: NVFP4 activations take the block-scaled FP4
 * MMA; the product is the operation at the top of this file).  tcgen05.mma
 * kind::mxf4nvf4, scale_vec::4X, E4M3 scales, FP32 accumulation in tensor
 * memory, fused alpha and BF16 epilogue; plain [rows][K/16] scales, rearranged
 * on chip.  M, N >= 0 (0 returns OK and does nothing); K >= 32, K % 32 == 0.
 * Requires exec_of(device, NVFP4, NVFP4) == FP4_MMA, else NVFP4_ERR_NO_FP4_KERNEL
 * or NVFP4_ERR_NOPATH. */
NVFP4_API nvfp4_status gemm_nvfp4_w4a4(const uint8_t* A, const uint8_t* sA, float gA,
                             const uint8_t* W, const uint8_t* sW, float gW,
                             void* Y_bf16, int M, int N, int K, void* stream);

/* ---- scales in the MMA's layout ------------------------------------------- */

/* Bytes of a packed scale buffer for a [rows][K/16] scale matrix (0 if K is
 * not a positive multiple of 64): ceil(rows/128) * 128 * K/16. */
NVFP4_API size_t nvfp4_scale_layout_bytes(int rows, int K);

/* Rearranges plain E4M3 group scales s_plain [rows][K/16] (device, row-major)
 * (16-byte aligned) into the block-scaled MMA's scale layout in s_packed
 * (device, 16-byte aligned, nvfp4_scale_layout_bytes(rows, K) bytes,
 * caller-owned):
 *     s_packed[rb][ks][i][j][t] = s_plain[rb*128 + 32*j + i][4*ks + t]
 * for 128-row blocks rb, K = 64 steps ks, i < 32, j < 4, t < 4 (rows past
 * `rows` are zero).  One 512-byte [i][j][t] atom is exactly what one
 * tcgen05.cp 32x128b.warpx4 copies into TMEM for 128 rows and one K = 64 step.
 * Weights' scales are packed once; activations' scales once per product.
 * K % 64 == 0.  Asynchronous on `stream`. */
NVFP4_API nvfp4_status nvfp4_pack_scales(const uint8_t* s_plain, int rows, int K,
                                         uint8_t* s_packed, void* stream);

/* ---- activation quantiser (the step ahead of the W4A4 product) ----------- */

/* Bytes of device scratch nvfp4_quantize_bf16 needs (a constant). */
#define NVFP4_QUANTIZE_WORKSPACE_BYTES 16
NVFP4_API size_t nvfp4_quantize_workspace_bytes(void);

/* Two-level NVFP4 quantisation of a BF16 matrix, the encoding the W4A4 product
 * consumes (the FFN-down workload's: an E4M3 scale per 16 elements from their
 * largest magnitude over 6, taken relative to an FP32 per-tensor scale from the
 * tensor's largest magnitude over 6 x 448; metrale_circuit `hardware::exec`
 * module doc, bullet 1, the NVFP4 row, for the format).  Every step is an IEEE FP32 operation
 * rounded to nearest even, in this order:
 *     g    = amax|X| / 2688                (g = 1 when X is all zero)
 *     s_b  = E4M3(amax_b / (6 g))          per 16 consecutive k of a row,
 *                                          nearest even, saturating at 448
 *     code = sign(t) | E2M1(|t|),  t = x / (s_b g)   (t = +-0 when s_b = 0),
 *                                          nearest even, saturating at 6
 *   X_bf16         device, [rows][K] BF16 row-major, finite values
 *   codes          device, [rows][K/2] packed codes (even k in the low nibble)
 *   scales         device, [rows][K/16] E4M3 bytes, or NULL
 *   scales_packed  device, nvfp4_scale_layout_bytes(rows, K) bytes in the MMA
 *                  layout of nvfp4_pack_scales (rows past `rows` zero), or
 *                  NULL; needs K % 64 == 0
 *   g_out          device, one float: g (the per-tensor scale to pass as gA)
 *   workspace      device scratch of NVFP4_QUANTIZE_WORKSPACE_BYTES bytes,
 *                  caller-owned; the call clears it itself (so it needs no
 *                  initialisation), and calls that share one must not overlap
 * At least one of scales / scales_packed.  K % 16 == 0, rows >= 0 (rows == 0
 * writes g = 1 only).  All buffers 16-byte aligned, g_out 4-byte aligned.
 * Asynchronous on `stream` (one memset and two kernels); the result is
 * deterministic.  Errors as the other entry points. */
NVFP4_API nvfp4_status nvfp4_quantize_bf16(const void* X_bf16, int rows, int K, uint8_t* codes,
                                           uint8_t* scales, uint8_t* scales_packed, float* g_out,
                                           void* workspace, size_t workspace_bytes, void* stream);

/* nvfp4_quantize_bf16 for callers that cannot allocate device memory: the
 * same operation, arguments (minus the workspace), results and errors, with
 * the few bytes of scratch it needs kept in a static device array of 256 bytes
 * inside the library instead of a caller buffer.  It is meant for code that may
 * not call cudaMalloc at all -- for example code that runs after an inference
 * runtime has handed all device memory to its own pool, or a plugin whose
 * enqueue step must not allocate -- and for callers with nowhere to keep a
 * scratch buffer between calls.  This entry point has no counterpart on the
 * pages; it is a convenience of this library.
 *   - It allocates nothing and calls no allocating routine.  Every GPU that
 *     loads the library holds the 256-byte array until the process exits.
 *   - Every call looks up the array's address in the current context (a query
 *     that allocates nothing); make the first call on a device before any
 *     stream capture, since it may load the library's device code.
 *   - Every call uses the same array; the call clears the part it needs, but
 *     calls whose work overlaps on the GPU (other streams, other threads) race
 *     on it and must be ordered by the caller.
 *   - The scratch it needs does not grow with the tensor; a need beyond the
 *     array's 256 bytes is refused with NVFP4_ERR_INVALID_ARG. */
NVFP4_API nvfp4_status nvfp4_quantize_bf16_noalloc(const void* X_bf16, int rows, int K,
                                                   uint8_t* codes, uint8_t* scales,
                                                   uint8_t* scales_packed, float* g_out,
                                                   void* stream);

/* nvfp4_quantize_bf16 with the rows written in an MoE dispatch's order: the
 * quantisation of token row r (the same codes, scale bytes and g as the plain
 * call) is written to output rows dest[r*k + j] for j < k, so that an MoE layer
 * needs no separate permutation of the quantised rows before its grouped
 * product (page 2, the FlashInfer swapab_cutedsl_megakernel skill doc, Layout:
 * each expert's tokens as one contiguous block of rows).
 *   dest    device, [rows*k] int32, the destination row of each (token, slot),
 *           as nvfp4_moe_route writes it; a value outside [0, rows*k) (the
 *           route's -1 for a pair with an out-of-range expert id) writes
 *           nothing, and output rows no pair lands on are left untouched
 *   k       slots per token, 1..8
 *   codes   device, [rows*k][K/2];  scales  device, [rows*k][K/16] (required)
 * The packed scale layout is not written (an MoE layer packs per expert).
 * Other arguments, alignment, errors and determinism as nvfp4_quantize_bf16;
 * dest must be 4-byte aligned. */
NVFP4_API nvfp4_status nvfp4_quantize_bf16_routed(const void* X_bf16, int rows, int K,
                                                  const int32_t* dest, int k, uint8_t* codes,
                                                  uint8_t* scales, float* g_out, void* workspace,
                                                  size_t workspace_bytes, void* stream);

/* gemm_nvfp4_w4a4 with both scale matrices already packed
 * (nvfp4_pack_scales / nvfp4_prepare_scales); the same product, module doc
 * bullet 1, the NVFP4 row.  Runs on pairs of SMs (tcgen05 cta_group::2, 256 x 256
 * tiles) and moves the packed scales with plain TMA tile loads, so no scale
 * rewrite happens inside the product.  Same operation, operands and errors as
 * gemm_nvfp4_w4a4, with K % 256 == 0. */
NVFP4_API nvfp4_status gemm_nvfp4_w4a4_packed(const uint8_t* A, const uint8_t* sA_packed, float gA,
                                              const uint8_t* W, const uint8_t* sW_packed, float gW,
                                              void* Y_bf16, int M, int N, int K, void* stream);

/* Device bytes of the workspace that gemm_nvfp4_w4a4_packed_ws needs for this
 * shape on the current device with at most `max_pairs` SM pairs (0: one pair per
 * two SMs).  0 when the tiles divide evenly among the pairs, or when no split
 * pays: fewer tiles than pairs, a last wave of whole tiles that would be more
 * than 60 % full, or a single K-block. The call then needs none.
 * The need grows with the number of pairs, not with the tensors: 512 KB per pair,
 * about 38 MB on a 148-SM part.  0 also when the device cannot be queried. */
NVFP4_API size_t nvfp4_w4a4_packed_workspace_bytes(int M, int N, int K, int max_pairs);

/* The same for a device with `num_sms` SMs (148 on a B200), without querying any
 * device: a pure function, usable with no GPU (for instance to size a workspace
 * before a device is opened).  0 for num_sms < 2 or a non-positive size. */
NVFP4_API size_t nvfp4_w4a4_packed_workspace_bytes_for(int M, int N, int K, int max_pairs,
                                                       int num_sms);

/* gemm_nvfp4_w4a4_packed with the last waves of tiles balanced over the pairs
 * (stream-K).  This is a design of this library, not of the pages; the product
 * is the page-1 module doc's NVFP4 row, as for gemm_nvfp4_w4a4_packed.
 *   - Whole 256 x 256 tiles go to the pairs in turn until about one and a half
 *     waves of tiles are left. The K-blocks of those are laid end to end and
 *     cut into one contiguous range per pair, so that no pair idles through a
 *     part-empty last wave.
 *   - A tile cut between two pairs is summed in FP32 from the two partial
 *     products (the first K-blocks and the rest). That changes only where the
 *     FP32 accumulation is split. Each output element is still the FP32 sum
 *     over all of K, times gA*gW, rounded once to BF16. The sum of the two
 *     FP32 terms does not depend on which pair finishes first, so the output
 *     is the same on every run.
 *   - max_pairs: 0 = one pair per two SMs; otherwise at most that many pairs
 *     (for instance to leave SMs to concurrent work).
 *   - workspace: device memory, 16-byte aligned, of workspace_bytes >=
 *     nvfp4_w4a4_packed_workspace_bytes(M, N, K, max_pairs) (NULL when that is
 *     0; a smaller buffer is NVFP4_ERR_INVALID_ARG). The caller owns it. It
 *     must be all zero before its first use. Each call leaves it ready for the
 *     next (its tickets back at zero). Zero it again after a call that
 *     reported NVFP4_ERR_DEVICE_TIMEOUT. Calls whose work overlaps on the GPU
 *     need one workspace each.
 *   - Everything else (operands, errors) as gemm_nvfp4_w4a4_packed. */
NVFP4_API nvfp4_status gemm_nvfp4_w4a4_packed_ws(const uint8_t* A, const uint8_t* sA_packed,
                                                 float gA, const uint8_t* W,
                                                 const uint8_t* sW_packed, float gW, void* Y_bf16,
                                                 int M, int N, int K, int max_pairs,
                                                 void* workspace, size_t workspace_bytes,
                                                 void* stream);

/* The same product through the exact E2M1->E4M3 conversion on the FP8 MMA
 * (module doc, bullet 2): each packed code byte is split into its two nibbles,
 * each placed in the high nibble of a byte and converted by
 * (q & 0x80808080) | ((q & 0x70707070) >> 2) to an E4M3 value equal to the
 * code's value times 2^-6; each 16-group's FP8 partial sum is scaled in FP32 by
 * (sA*2^6)*(sW*2^6) and accumulated.  Same arguments and preconditions as
 * gemm_nvfp4_w4a4; needs a device class for which the FP8 kernel is compiled
 * (sm_100), else NVFP4_ERR_NOPATH. */
NVFP4_API nvfp4_status gemm_nvfp4_via_fp8(const uint8_t* A, const uint8_t* sA, float gA,
                                const uint8_t* W, const uint8_t* sW, float gW,
                                void* Y_bf16, int M, int N, int K, void* stream);

/* W4A8: FP8 (E4M3) activations under NVFP4 weights (metrale_circuit
 * `hardware::exec`, exec_of: W4A8 with group-16 E4M3 scales takes the exact
 * E4M3 path):
 *     Y[m,n] = BF16( gA*gW * sum_g sW[n,g] * sum_{k in g} a[m,k]*w[n,k] )
 * with a[m,k] the E4M3 value of byte A_fp8[m][k] (row-major [M][K], one byte per
 * element, any finite E4M3 byte; gA is its FP32 per-tensor scale) and W, sW, gW
 * as for gemm_nvfp4_w4a4 (the activations carry no group scales).  Each weight
 * times its group scale is written exactly as three E5M2 planes (the scale's
 * signed binary digits times the E2M1 value); three E4M3 x E5M2 FP8 MMAs per
 * K step accumulate every product exactly into one FP32 accumulator, as the
 * declared W4A4 product would.
 * M, N >= 0 (0 returns OK and does nothing); K >= 256, K % 256 == 0; every
 * pointer a 16-byte aligned device pointer.  Needs exec_of(device, NVFP4, FP8)
 * == FP8_EXACT (sm_100), else NVFP4_ERR_NOPATH. */
NVFP4_API nvfp4_status gemm_nvfp4_w4a8(const uint8_t* A_fp8, float gA, const uint8_t* W,
                                       const uint8_t* sW, float gW, void* Y_bf16, int M, int N,
                                       int K, void* stream);

/* ---- MoE dispatch and combine around the grouped product ------------------
 * (page 2, the MegaMoE swap-AB kernel: tokens are dispatched to their experts,
 * run through one grouped GEMM, and combined back with their routing weights.)
 * A "pair" is one (token t, slot j) of a top-k routing, numbered p = t*k + j. */

/* Workspace bytes of nvfp4_moe_route for num_pairs pairs and E experts (0 for
 * num_pairs < 0 or E outside [1, 256]). */
NVFP4_API size_t nvfp4_moe_route_workspace_bytes(int num_pairs, int E);

/* Route: expert_ids [num_pairs] (device int32, pair p's expert) ->
 *   offsets [E+1]       rows of expert e are offsets[e] .. offsets[e+1]-1 of the
 *                       expert-grouped order (the `offsets` of the grouped GEMM);
 *   dest [num_pairs]    pair p's row in that order;
 *   src  [num_pairs]    the pair on grouped row r (src[dest[p]] = p).
 * Inside an expert, pairs keep their order p (stable, hence deterministic).
 * All arrays are device memory owned by the caller; workspace is device memory
 * of nvfp4_moe_route_workspace_bytes bytes, 16-byte aligned, overwritten.  An id
 * outside [0, E) is placed nowhere (its dest stays -1, and offsets[E] counts only
 * placed pairs) and makes the next nvfp4_check_device_error return
 * NVFP4_ERR_INVALID_ARG.  E in [1, 256]; num_pairs == 0 writes zero offsets. */
NVFP4_API nvfp4_status nvfp4_moe_route(const int32_t* expert_ids, int num_pairs, int E,
                                       int32_t* offsets, int32_t* dest, int32_t* src,
                                       void* workspace, size_t workspace_bytes, void* stream);

/* Permute (dispatch on one GPU): out[r] = in[src[r] / k] for r < num_pairs, whole
 * rows of row_bytes bytes (a positive multiple of 16): the rows of a token's
 * codes (K/2 bytes) or plain scales (K/16 bytes), in token order in `in`
 * [in_rows][row_bytes], land in the expert-grouped order in `out`
 * [num_pairs][row_bytes], one copy per pair.  A row whose src is outside
 * [0, in_rows*k) is left untouched.  Device pointers, 16-byte aligned. */
NVFP4_API nvfp4_status nvfp4_moe_permute_rows(const void* in, size_t row_bytes, int in_rows,
                                              int num_pairs, int k, const int32_t* src,
                                              void* out, void* stream);

/* Combine: Y[t][n] = BF16( sum_{j<k} w[t][j] * Yg[dest[t*k+j]][n] ), the FP32
 * products added in the order j = 0..k-1 and rounded once to nearest even.
 * Yg is the grouped product's output, BF16 [num_pairs][N] in the expert-grouped
 * order; weights is device FP32 [T][k] or NULL for all ones; Y is BF16 [T][N].
 * A dest outside [0, num_pairs) contributes nothing.  N % 8 == 0; device
 * pointers, Yg and Y 16-byte aligned. */
NVFP4_API nvfp4_status nvfp4_moe_combine(const void* Yg_bf16, int num_pairs, const int32_t* dest,
                                         const float* weights, int T, int k, int N, void* Y_bf16,
                                         void* stream);

/* W4A16 (metrale_circuit `hardware::exec` module doc, bullet 1, the BF16 row:
 * BF16 activations take the BF16 MMA, with any weight format widened in
 * registers):
 *     Y[m,n] = BF16( gW * sum_g sW[n,g] * sum_{k in g} a[m,k]*w[n,k] )
 * BF16 activations A_bf16 [M][K] (row-major) times NVFP4 weights, the
 * weights widened to BF16 in registers (exactly: an E2M1 value times an E4M3
 * scale has at most 6 significant bits), FP32 accumulation, gW applied in the
 * epilogue, BF16 output Y [M][N].  Built for the memory-bound decode shape:
 * one launch covers 16 tokens (larger M runs as consecutive 16-token launches,
 * each re-reading W).  One wave of CTAs, each owning a range of weight rows over
 * the whole of K; K is split across the CTA's warps and their partial sums are
 * added in shared memory in a fixed order, so the call needs no workspace and
 * is deterministic.  M, N >= 0; K >= 32, K % 32 == 0. */
NVFP4_API nvfp4_status gemm_w4a16(const void* A_bf16, const uint8_t* W, const uint8_t* sW, float gW,
                        void* Y_bf16, int M, int N, int K, void* stream);

/* Grouped (MoE) W4A4 with the expert offsets in device memory (page 2, the
 * FlashInfer swapab_cutedsl_megakernel skill doc, Layout: the MoE kernel with
 * swapped A/B operands for small per-expert M; each expert's product is the
 * NVFP4 row of page 1's module doc, bullet 1).  Expert e owns rows
 * offsets[e] .. offsets[e+1]-1 of A (tokens grouped by expert), its weights
 * W + e*N*K/2 ([N][K/2]), plain scales sW + e*N*K/16 ([N][K/16]) and FP32
 * scale gW_host[e]; Y is [total_M][N]:
 *     Y[r,n] = BF16( gA*gW[e] * sum_g sA[r,g]*sW_e[n,g] * sum_{k in g} a[r,k]*w_e[n,k] )
 *   offsets_dev  device int32 [E+1]: offsets[0] = 0, non-decreasing,
 *                offsets[E] = total_M (for example nvfp4_moe_route's output);
 *                never read on the host, so no round trip.  Offsets that break
 *                these rules make the product write nothing and the next
 *                nvfp4_check_device_error return NVFP4_ERR_INVALID_ARG.
 *   gW_host      host float [E], read during the call only.
 *   workspace    device memory, 16-byte aligned, caller-owned, of ws_bytes >=
 *                nvfp4_workspace_size(NVFP4_OP_W4A4_GROUPED, total_M, N, K, E)
 *                bytes (smaller is NVFP4_ERR_INVALID_ARG); needs no
 *                initialisation; calls that overlap on the GPU need one each.
 * The call plans the tiles on the device, packs both scale matrices into the
 * workspace and runs the SM-pair product of gemm_nvfp4_w4a4_grouped_packed_sched:
 * 256-token blocks of an expert as 256 x 256 tiles, an expert's last 1..128
 * tokens swapped (weight rows on the MMA's M side, tokens on its N side).
 * 1 <= E <= 256; N >= 1; K % 256 == 0; total_M == 0 returns OK and does
 * nothing.  Callers that keep the weights' scales packed should call the
 * _packed_sched entry points directly and skip the per-call weight packing. */
NVFP4_API nvfp4_status gemm_nvfp4_w4a4_grouped(const uint8_t* A, const uint8_t* sA, float gA,
                                     const uint8_t* W, const uint8_t* sW,
                                     const float* gW_host, const int32_t* offsets_dev,
                                     int E, int total_M, void* Y_bf16, int N, int K,
                                     void* workspace, size_t ws_bytes, void* stream);

/* The grouped product planned on the host from host offsets, on single SMs
 * from plain scales (the same passages as gemm_nvfp4_w4a4_grouped).  Expert e
 * owns rows offsets[e] .. offsets[e+1]-1 of A, W + e*N*K/2, sW + e*N*K/16 and
 * gW_host[e]; Y is [offsets[E]][N].  `offsets_host` (int32 [E+1], host memory,
 * offsets[0] == 0, non-decreasing) is read during the call only.  Blocks of
 * fewer than 128 rows run with the operands swapped (Y_e^T = W_e . A_e^T:
 * weight rows on the MMA's M side, tokens on its N side).  No workspace.
 * 1 <= E <= 256; K % 256 == 0. */
NVFP4_API nvfp4_status gemm_nvfp4_w4a4_grouped_host(const uint8_t* A, const uint8_t* sA, float gA,
                                          const uint8_t* W, const uint8_t* sW,
                                          const float* gW_host, const int32_t* offsets_host,
                                          int E, void* Y_bf16, int N, int K, void* stream);

/* Bytes of a grouped packed scale buffer: groups g = 0..E-1 own rows
 * offsets[g] .. offsets[g+1]-1 and each starts on a 128-row block, so the size
 * is sum_g ceil(rows_g/128) * 128 * K/16 (0 if an argument is invalid).
 * `offsets_host` is int32 [E+1] in host memory, read during the call only. */
NVFP4_API size_t nvfp4_grouped_scale_layout_bytes(const int32_t* offsets_host, int E, int K);

/* nvfp4_pack_scales per group: group g's rows of s_plain [offsets[E]][K/16]
 * are packed into the blocks starting at block b_g = sum_{h<g} ceil(rows_h/128)
 * of s_packed (device, 16-byte aligned, nvfp4_grouped_scale_layout_bytes
 * bytes, caller-owned); rows past a group's end are zero.  Activation scales
 * of tokens grouped by expert are packed this way per product; the weight
 * scales of E experts of N rows each are packed once with offsets
 * {0, N, 2N, ..., E*N}.  1 <= E <= 256, K % 64 == 0; the offsets rules of
 * gemm_nvfp4_w4a4_grouped_host.  Asynchronous on `stream`. */
NVFP4_API nvfp4_status nvfp4_pack_scales_grouped(const uint8_t* s_plain, const int32_t* offsets_host,
                                                 int E, int K, uint8_t* s_packed, void* stream);

/* gemm_nvfp4_w4a4_grouped_host with packed scales (page 2, swapab_cutedsl_megakernel,
 * Layout: swap-AB for small M; page 1 module doc bullet 1, the NVFP4 row, per
 * expert): sA_packed packed by nvfp4_pack_scales_grouped with these offsets,
 * sW_packed with offsets {0, N, ..., E*N}.  Runs on pairs of SMs (tcgen05
 * cta_group::2): 256-token blocks of an expert as M = 256, N = 256 tiles; an
 * expert's last 1..128 tokens (all of a small expert) swapped, 256 weight rows
 * on the MMA's M side and 128 token slots on its N side.  Same operation,
 * operands and errors as gemm_nvfp4_w4a4_grouped_host (K % 256 == 0). */
NVFP4_API nvfp4_status gemm_nvfp4_w4a4_grouped_packed(const uint8_t* A, const uint8_t* sA_packed,
                                                      float gA, const uint8_t* W,
                                                      const uint8_t* sW_packed,
                                                      const float* gW_host,
                                                      const int32_t* offsets_host, int E,
                                                      void* Y_bf16, int N, int K, void* stream);

/* ---- grouped product with device-resident expert offsets, packed scales ----
 * (page 2, swapab_cutedsl_megakernel, Layout; page 1 module doc bullet 1, the
 * NVFP4 row, per expert.)  The _host and _packed entry points above plan their
 * tiles on the host from host offsets.  These take offsets[E+1] in device memory (for example from
 * nvfp4_moe_route), so a whole MoE layer runs with no host round trip and can
 * be captured in a CUDA graph: nvfp4_grouped_schedule plans on the device into
 * a small caller buffer, which the packing and the product then read.  Same
 * operation, layouts and rounding as gemm_nvfp4_w4a4_grouped_packed. */

/* Bytes of the schedule buffer (device memory, 16-byte aligned, caller-owned). */
NVFP4_API size_t nvfp4_grouped_sched_bytes(void);

/* Upper bound of the grouped packed layout of M rows in E groups, whatever the
 * offsets: (ceil(M/128) + E) * 128 * K/16 bytes (0 for bad sizes).  The packed
 * activation scales of the scheduled path need a buffer of this size. */
NVFP4_API size_t nvfp4_grouped_scale_layout_bytes_bound(int M, int E, int K);

/* One thread on the device reads offsets_dev [E+1] (int32, offsets[0] = 0,
 * non-decreasing, offsets[E] = M) and writes the tile schedule, alpha_e =
 * gA*gW[e] (gA from *gA_dev when gA_dev is not null, else the host value gA;
 * gW_host [E] host floats read during the call) and the packing map into
 * `sched`.  Offsets that break those rules give an empty schedule (the
 * products below then write nothing) and make the next
 * nvfp4_check_device_error return NVFP4_ERR_INVALID_ARG.  E in [1, 256]; N >= 1;
 * K % 256 == 0. */
NVFP4_API nvfp4_status nvfp4_grouped_schedule(const int32_t* offsets_dev, int E, int M, int N, int K,
                                              const float* gA_dev, float gA, const float* gW_host,
                                              void* sched, void* stream);

/* nvfp4_pack_scales_grouped with the groups of a schedule: s_plain [M][K/16] ->
 * s_packed (nvfp4_grouped_scale_layout_bytes_bound(M, E, K) bytes). */
NVFP4_API nvfp4_status nvfp4_pack_scales_grouped_sched(const uint8_t* s_plain, int M, int E, int K,
                                                       const void* sched, uint8_t* s_packed,
                                                       void* stream);

/* gemm_nvfp4_w4a4_grouped_packed with the tiles and alphas of a schedule: A
 * [M][K/2] grouped by expert, sA_packed from nvfp4_pack_scales_grouped_sched, W
 * [E][N][K/2] and sW_packed as for the host-planned entry, Y [M][N]. */
NVFP4_API nvfp4_status gemm_nvfp4_w4a4_grouped_packed_sched(const uint8_t* A, const uint8_t* sA_packed,
                                                            const uint8_t* W, const uint8_t* sW_packed,
                                                            const void* sched, int E, int M, void* Y_bf16,
                                                            int N, int K, void* stream);

/* gemm_nvfp4_w4a4_grouped_packed_sched with the top-1 combine fused into its
 * epilogue. Page 2's MegaMoE does its combine inside the expert kernel; this is
 * the same idea for one expert per token.
 *   - Grouped row r (the row of token pair src[r] in expert order, as
 *     nvfp4_moe_route / nvfp4_moe_permute_rows produce it with k = 1) is written
 *     to Y_bf16 row src[r]: Y[src[r]][n] = BF16(gA*gW[e] * w * acc[r][n]).
 *   - w is weights[src[r]] (device float [T]); w = 1 when weights is NULL.
 *   - The result equals nvfp4_moe_combine over the unfused product's rows,
 *     except that it is rounded to BF16 once instead of twice. The grouped
 *     rows never reach memory.
 *   - src: device int32 [M], a permutation of [0, T) in top-1 routing. Every
 *     Y row named by src is written once; other rows of Y are left as they are.
 *   - Y_bf16: device [T][N], caller-owned.
 *   - M <= T; N even.
 *   - A src entry outside [0, T) is not written. It makes the next
 *     nvfp4_check_device_error return NVFP4_ERR_INVALID_ARG.
 *   - Everything else as gemm_nvfp4_w4a4_grouped_packed_sched. */
NVFP4_API nvfp4_status gemm_nvfp4_w4a4_grouped_packed_sched_combine(
    const uint8_t* A, const uint8_t* sA_packed, const uint8_t* W, const uint8_t* sW_packed,
    const void* sched, int E, int M, const int32_t* src, const float* weights, void* Y_bf16, int T,
    int N, int K, void* stream);

/* ---- generic workspace query and scale preparation ------------------------ */

/* The operations whose workspace nvfp4_workspace_size reports. */
typedef enum {
    NVFP4_OP_W4A4 = 0,          /* gemm_nvfp4_w4a4: none */
    NVFP4_OP_VIA_FP8 = 1,       /* gemm_nvfp4_via_fp8: none */
    NVFP4_OP_W4A16 = 2,         /* gemm_w4a16: none */
    NVFP4_OP_W4A4_GROUPED = 3,  /* gemm_nvfp4_w4a4_grouped (M = total_M) */
    NVFP4_OP_W4A8 = 4,          /* gemm_nvfp4_w4a8: none */
    NVFP4_OP_W4A4_PACKED = 5,   /* gemm_nvfp4_w4a4_packed_ws on the current device, all pairs */
    NVFP4_OP_QUANTIZE = 6,      /* nvfp4_quantize_bf16 (a constant) */
    NVFP4_OP_MOE_ROUTE = 7      /* nvfp4_moe_route with num_pairs = M */
} nvfp4_op;

/* Device bytes of caller workspace that operation `op` (an nvfp4_op) needs for
 * an M x N x K product over E experts (E is ignored by ungrouped ops).  0 when
 * the call needs none or a size is invalid; SIZE_MAX for an unknown op.  Every
 * workspace-taking entry point accepts a buffer of at least this size; none
 * allocates device memory itself.  Host only (NVFP4_OP_W4A4_PACKED queries the
 * current device's SM count and is 0 without a device). */
NVFP4_API size_t nvfp4_workspace_size(int op, int M, int N, int K, int E);

/* Plain E4M3 group scales s_plain [rows][K/16] -> the block-scaled MMA's scale
 * layout in s_mma (nvfp4_scale_layout_bytes(rows, K) bytes): the same
 * rearrangement as nvfp4_pack_scales (whose comment gives the layout), with the
 * argument order of a prepare step.  K % 64 == 0; device pointers, 16-byte
 * aligned, caller-owned; asynchronous on `stream`. */
NVFP4_API nvfp4_status nvfp4_prepare_scales(const uint8_t* s_plain, uint8_t* s_mma, int rows, int K,
                                            void* stream);

/* ---- diagnostics ----------------------------------------------------------- */

/* Thread-local text of the last error returned on this host thread ("" if none). */
NVFP4_API const char* nvfp4_last_error(void);

/* Synchronizes `stream`, then reads and clears the device error word that a
 * kernel sets when one of its bounded waits expires.  NVFP4_OK if clear,
 * NVFP4_ERR_DEVICE_TIMEOUT if a wait expired, NVFP4_ERR_INVALID_ARG if the only
 * records are bad data seen on the device (an out-of-range expert id in
 * nvfp4_moe_route, bad offsets in nvfp4_grouped_schedule), NVFP4_ERR_CUDA if
 * synchronization failed. */
NVFP4_API nvfp4_status nvfp4_check_device_error(void* stream);

/* Library version string (static storage). */
NVFP4_API const char* nvfp4_version(void);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4_B200_H */
