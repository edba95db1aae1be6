/*
 * libw4a8 -- block-quantized W4A8 matmul y = x . W^T on one NVIDIA B200 (sm_100a).
 *
 * Weights are stored as Q4_0 (4-bit codes in blocks of 32 along K with one fp16 scale
 * per block); activations are quantised on the fly to Q8_0 (int8 codes in blocks of 32
 * with one f32 scale per block). Each 32-wide block dot product is computed exactly in
 * integer arithmetic and then rescaled by the two block scales and accumulated in f32.
 * Sources: tract PR #2432 "W4A8 (Q4_0 int8-dot) path for block_quant", sections
 * "Pipeline" (4-bit N x K weight, activation to int8 per block) and "The kernel"
 * (per-32-block weight scales, per-block f32 rescale, no per-op allocation wanted);
 * and for the affine variant, MLX PR #4802 "mx.qqmm ... mode=affine" (int8 MMA on the
 * original 4-bit codes, per-group scales and biases applied in the kernel).
 *
 * Conventions shared by every entry point
 *  - Every pointer argument is DEVICE memory owned by the caller; the library never
 *    allocates, frees or keeps a pointer after the call returns. Pointers must be
 *    16-byte aligned (W4A8_ERR_MISALIGNED otherwise).
 *  - All work is enqueued asynchronously on `stream` (0 = the legacy default stream).
 *    The returned status covers argument checks and launch errors only; a fault inside
 *    a kernel surfaces at the caller's next synchronisation.
 *  - Matrices are dense row-major with no padding: x is M x K, W is N x K ("N x K" as
 *    on the tract page), y is M x N (f32).
 *  - The kernels never trap, assert or wait without bound. Every internal wait has a
 *    time limit; when one runs out the kernel records W4A8_ERR_DEVICE_TIMEOUT in a
 *    device status word (read it with w4a8_last_device_error) and exits cleanly.
 *  - Calls run on the calling thread's current device and may come from several host
 *    threads. The host state the library keeps (each kernel's raised shared-memory limit,
 *    the no-alloc scratch address) is recorded per CUDA context under a lock, so calls
 *    keep working in a context created after cudaDeviceReset.
 */
#ifndef W4A8_H_
#define W4A8_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    W4A8_OK = 0,
    W4A8_ERR_INVALID_ARG = 1,    /* null pointer, non-positive or too large size, K % 32 != 0 */
    W4A8_ERR_UNSUPPORTED = 2,    /* a mode the kernels do not implement (dtype, group size, path) */
    W4A8_ERR_WORKSPACE = 3,      /* workspace pointer null or smaller than w4a8_workspace_bytes() */
    W4A8_ERR_CUDA = 4,           /* a CUDA runtime call or kernel launch failed */
    W4A8_ERR_DEVICE_TIMEOUT = 5, /* a bounded wait inside a kernel ran out (see w4a8_last_device_error) */
    W4A8_ERR_MISALIGNED = 6,     /* a pointer is not 16-byte aligned */
    W4A8_ERR_RANGE = 7,          /* a weight scale outside the tensor-core path's exact range
                                    (see w4a8_gemm); reported by w4a8_last_device_error */
    W4A8_ERR_CHECK = 8           /* checked build only (libw4a8_checked.so, -DW4A8_CHECKED): a
                                    device-side check of a copy's alignment failed and the
                                    copy was skipped; reported by w4a8_last_device_error */
} w4a8_status;

/* Element type of the unquantised input (x or W). bf16 is widened exactly to f32. */
typedef enum { W4A8_F32 = 0, W4A8_BF16 = 1 } w4a8_dtype;

/* Which kernel path a matmul takes. AUTO chooses by M (small M streams the weights
 * once with a dp4a GEMV; larger M runs the tcgen05 tensor-core GEMM). */
typedef enum { W4A8_PATH_AUTO = 0, W4A8_PATH_GEMV = 1, W4A8_PATH_GEMM = 2 } w4a8_path;

/* Largest M, N or K any entry point accepts (keeps every byte offset inside int64 and
 * every per-row count inside int32). */
#define W4A8_MAX_DIM (1 << 20)

/*
 * Q4_0 weight pack (once per weight; not part of the per-call matmul).
 * w      : N x K row-major, f32 or bf16 (`dtype`).
 * qs     : out, N x K/2 bytes. Row n, block b occupies bytes [n*K/2 + 16b, +16); byte j of
 *          a block holds the code of element 32b+j in its low nibble and of element
 *          32b+j+16 in its high nibble.
 * d_fp16 : out, N x K/32 fp16 bit patterns, the scale of each block.
 * Per block: mx = the element of largest magnitude (first on ties), d = mx / -8 (f32),
 * q = min(15, trunc(x * (1/d) + 8.5)) (0 when d == 0), stored scale fp16(d) (round to
 * nearest even). Dequantised weight: fp16(d) * (q - 8).
 * Errors: INVALID_ARG (null, N or K <= 0 or > W4A8_MAX_DIM, K % 32 != 0), MISALIGNED,
 * UNSUPPORTED (dtype), CUDA.
 */
w4a8_status w4a8_pack_q4_0(const void* w, w4a8_dtype dtype, int N, int K,
                           uint8_t* qs, uint16_t* d_fp16, cudaStream_t stream);

/*
 * Q8_0 activation quantisation (the per-call step that w4a8_gemm runs internally).
 * x  : M x K row-major, f32 or bf16.
 * qx : out, M x K int8 codes (row-major, same element order as x).
 * dx : out, M x K/32 f32 block scales, d = amax/127 over the block.
 * sx : out (may be NULL), M x K/32 int32 block sums of the codes.
 * q = clamp(round_half_away_from_zero(x * (1/d)), -127, 127); all codes 0 when d == 0.
 * Errors: as w4a8_pack_q4_0.
 */
w4a8_status w4a8_quant_act_q8_0(const void* x, w4a8_dtype dtype, int M, int K,
                                int8_t* qx, float* dx, int32_t* sx, cudaStream_t stream);

/*
 * Size in bytes of the workspace w4a8_gemm / w4a8_gemm_affine use for this shape
 * (group = 0 for Q4_0, else the affine group size) on the current device. Covers every
 * path, so one allocation serves AUTO and both forced paths. It includes room for the
 * tensor-core path's split of K (partial sums, reduced in a fixed order): at least one
 * split per 128 quant blocks (K > 4096), which bounds each output's f32 accumulation
 * chain, and more when the output tiles do not fill the SMs. A smaller workspace is
 * accepted down to the minimum of the path the call takes (GEMV: the quantised
 * activation; tensor cores: the operand plus the partial sums of the bounding split); the
 * extra split then shrinks to what fits, which can change the last bits of the result.
 * Below that minimum the calls return W4A8_ERR_WORKSPACE. Returns 0 for invalid sizes.
 */
size_t w4a8_workspace_bytes(int M, int N, int K, int group);

/*
 * Which kernel family w4a8_gemm (group = 0) or w4a8_gemm_affine (group = 32, 64 or 128)
 * runs for a shape on `path` (host logic only: no device work). The choice is the
 * M-based dispatch between the memory-bound small-M path and the tensor-core path (tract
 * PR #2432, follow-up on the decode regime; MLX PR #4802, introduction: its int8 kernel
 * only from M = 32), with the crossover measured on B200. Returns W4A8_KERNEL_GEMV (dp4a GEMV), W4A8_KERNEL_TC_INT8
 * (tcgen05 kind::i8, tokens as the MMA's N), W4A8_KERNEL_TC_FP16 (tcgen05 kind::f16, one
 * CTA), W4A8_KERNEL_TC_PAIR (kind::f16 on CTA pairs), or 0 for sizes, groups or paths the
 * call would reject.
 */
enum {
    W4A8_KERNEL_GEMV = 1,
    W4A8_KERNEL_TC_INT8 = 2,
    W4A8_KERNEL_TC_FP16 = 3,
    W4A8_KERNEL_TC_PAIR = 4
};
int w4a8_gemm_path(int M, int N, int K, int group, w4a8_path path);

/*
 * y = x . W^T with W in Q4_0 (from w4a8_pack_q4_0) and x quantised to Q8_0 inside the
 * call: y[m][n] = sum_b f32(d_w[n][b]) * d_x[m][b] * D[m][n][b], with
 * D = sum_{j<32} (q_w - 8) * q_x computed exactly. The sum over blocks is taken in f32;
 * each output is within 1e-5 * sum_b |term_b| of the exact value at every K: the GEMV
 * paths add at most a few dozen terms in any chain, and the tensor-core path splits K so
 * that no chain is longer than 128 blocks (error <= 160 * 2^-24 * sum_b |term_b|).
 * x        : M x K, f32 or bf16.       qs, d_fp16 : as produced by w4a8_pack_q4_0.
 * y        : out, M x N f32.           ws, ws_bytes : scratch of w4a8_workspace_bytes(M, N,
 *            K, 0) bytes (or at least the path's minimum, see there), owned by the
 *            caller; contents on entry are ignored and are garbage afterwards. Calls
 *            that share a workspace must be ordered on one stream.
 * Paths (AUTO): the dp4a GEMV for M = 1, for M = 2 when K <= 8192, for M <= 4 when
 * N * K <= 2^25, and for M <= 8 when K is not a multiple of 256; otherwise tensor
 * cores: int8 MMAs on the
 * original codes for M <= 64 (K a multiple of 256), fp16 MMAs on CTA pairs above.
 * Scale range: the fp16 tensor-core kernels hold d_w * (q - 8) exactly as two fp16 values
 * formed by one fused multiply-add each, which requires |d_w| < 2728 (weights of magnitude
 * up to ~21800). A larger, infinite or NaN scale makes the kernel set W4A8_ERR_RANGE in
 * the device status word (w4a8_last_device_error) and the affected outputs are not
 * reliable. The GEMV and the int8 kernel have no such limit.
 * Errors: INVALID_ARG, MISALIGNED, UNSUPPORTED, WORKSPACE, CUDA.
 */
w4a8_status w4a8_gemm(int M, int N, int K, const void* x, w4a8_dtype dtype,
                      const uint8_t* qs, const uint16_t* d_fp16, float* y,
                      void* ws, size_t ws_bytes, cudaStream_t stream);

/* w4a8_gemm with the kernel path forced (for tests and measurements). */
w4a8_status w4a8_gemm_ex(int M, int N, int K, const void* x, w4a8_dtype dtype,
                         const uint8_t* qs, const uint16_t* d_fp16, float* y,
                         void* ws, size_t ws_bytes, w4a8_path path, cudaStream_t stream);

/*
 * Affine 4-bit weight pack. Per row n and group g of `group` (32, 64 or 128) elements:
 * s = bf16((max - min) / 15), b = bf16(min), q = clamp(round_half_away((w - b) / s), 0, 15)
 * (q = 0 when s == 0), using the stored bf16 s and b. Dequantised weight: s * q + b.
 * w          : N x K row-major, f32 or bf16.
 * q          : out, N x K/8 uint32 words; element k of row n sits at bits 4*(k%8) of
 *              word n*K/8 + k/8.
 * scale_bf16 : out, N x K/group bf16 bit patterns.   bias_bf16 : out, same shape.
 * Errors: INVALID_ARG (also K % group != 0), UNSUPPORTED (group not 32, 64 or 128), MISALIGNED, CUDA.
 */
w4a8_status w4a8_pack_affine(const void* w, w4a8_dtype dtype, int N, int K, int group,
                             uint32_t* q, uint16_t* scale_bf16, uint16_t* bias_bf16,
                             cudaStream_t stream);

/*
 * y = x . W^T with W affine 4-bit (from w4a8_pack_affine) and x quantised to Q8_0 in the
 * call. The contraction runs on the original codes: per activation block b inside
 * group g, y += d_x * (s_g * sum q*q_x + b_g * sum q_x). Tolerance as w4a8_gemm.
 * Scale range of the tensor-core path: s = 0 or 2^-17 <= |s| <= 2720 (s * (q - 8) is then
 * exact in fp16), and on its CTA-pair kernel (128-token tiles with K/group a multiple of
 * 8) also |b + 8s| <= 65504, the bias term's factor being an fp16 operand there; other
 * values set W4A8_ERR_RANGE as in w4a8_gemm.
 * Arguments and errors as w4a8_gemm, plus `group` (32, 64 or 128).
 */
w4a8_status w4a8_gemm_affine(int M, int N, int K, int group, const void* x, w4a8_dtype dtype,
                             const uint32_t* q, const uint16_t* scale_bf16,
                             const uint16_t* bias_bf16, float* y, void* ws, size_t ws_bytes,
                             cudaStream_t stream);

/* w4a8_gemm_affine with the kernel path forced. */
w4a8_status w4a8_gemm_affine_ex(int M, int N, int K, int group, const void* x, w4a8_dtype dtype,
                                const uint32_t* q, const uint16_t* scale_bf16,
                                const uint16_t* bias_bf16, float* y, void* ws, size_t ws_bytes,
                                w4a8_path path, cudaStream_t stream);

/*
 * Output epilogue of a linear layer: y[m][n] = P[m][n] + bias[n], stored as f32 or bf16,
 * where P is the product w4a8_gemm / w4a8_gemm_affine compute. The bias is added in f32
 * (one rounding) to every row, as the Q4_K GEMM wrapper of the C-Kernel-Engine page
 * (gemm_kernels_q4k.c, "Engine-compatible wrapper: GEMM_NT with Q4_K weights") adds its
 * optional bias after the product; a bf16 output is that f32 value rounded to the nearest
 * bf16 (ties to even; NaN stays NaN, overflow gives infinity).
 *  bias      : N values of bias_dtype (W4A8_F32 or W4A8_BF16), naturally aligned, or NULL
 *              (no bias: P is stored unchanged).
 *  out_dtype : element type of y: W4A8_F32 (float) or W4A8_BF16 (bf16 bit patterns).
 * The struct is read during the call only; the bias must stay valid until the work
 * enqueued on `stream` has run.
 */
typedef struct {
    const void* bias;
    w4a8_dtype bias_dtype;
    w4a8_dtype out_dtype;
} w4a8_epilogue;

/*
 * w4a8_gemm_ex / w4a8_gemm_affine_ex with an epilogue (NULL: as w4a8_gemm_ex). y is M x N
 * elements of epi->out_dtype, 16-byte aligned. Errors: as w4a8_gemm, plus UNSUPPORTED for
 * an unknown bias or output type and MISALIGNED for a bias not aligned to its element size.
 */
w4a8_status w4a8_gemm_epi(int M, int N, int K, const void* x, w4a8_dtype dtype,
                          const uint8_t* qs, const uint16_t* d_fp16, const w4a8_epilogue* epi, void* y,
                          void* ws, size_t ws_bytes, w4a8_path path, cudaStream_t stream);
w4a8_status w4a8_gemm_affine_epi(int M, int N, int K, int group, const void* x, w4a8_dtype dtype,
                                 const uint32_t* q, const uint16_t* scale_bf16, const uint16_t* bias_bf16,
                                 const w4a8_epilogue* epi, void* y, void* ws, size_t ws_bytes, w4a8_path path,
                                 cudaStream_t stream);

/*
 * Split form of w4a8_gemm / w4a8_gemm_affine for an activation that feeds several
 * weight matrices (e.g. projections sharing one input): the activation is quantised
 * once and the per-call re-quantisation the tract page identifies as per-op overhead
 * ("W4A8MatMul op" measurements) is paid once.
 *  w4a8_prepare_act   quantises x (M x K) into `ws` in the layout of the path that a
 *                     matmul of this M takes (`path` AUTO resolves without N: the GEMV
 *                     for M <= 3 where w4a8_gemm would take the int8 tensor kernel,
 *                     else for M <= 8; group = 0 for Q4_0 weights, else 32, 64 or 128).
 *  w4a8_gemm_prepared / w4a8_gemm_affine_prepared
 *                     run only the contraction, reading the quantised activation from
 *                     `ws`. They must be given the same M, K, group and path as the
 *                     w4a8_prepare_act call that filled `ws`, on the same stream (or
 *                     after it completed); `ws` is only read.
 * Errors: as w4a8_gemm.
 */
w4a8_status w4a8_prepare_act(int M, int K, int group, const void* x, w4a8_dtype dtype, void* ws,
                             size_t ws_bytes, w4a8_path path, cudaStream_t stream);
w4a8_status w4a8_gemm_prepared(int M, int N, int K, const uint8_t* qs, const uint16_t* d_fp16, float* y,
                               const void* ws, size_t ws_bytes, w4a8_path path, cudaStream_t stream);
w4a8_status w4a8_gemm_affine_prepared(int M, int N, int K, int group, const uint32_t* q,
                                      const uint16_t* scale_bf16, const uint16_t* bias_bf16, float* y,
                                      const void* ws, size_t ws_bytes, w4a8_path path,
                                      cudaStream_t stream);

/*
 * Affine weights with 4-, 6- or 8-bit codes (MLX PR #4802 "mx.qqmm ... mode=affine": its
 * int8 kernel takes 4-, 6- and 8-bit affine weights; "Accuracy" gives 6- and 8-bit rows).
 * Pack, per row n and group g of `group` (32, 64 or 128) elements, with qmax = 2^bits - 1:
 * s = bf16((max - min) / qmax), b = bf16(min), q = clamp(round_half_away((w - b) / s), 0,
 * qmax) (q = 0 when s == 0), using the stored bf16 s and b.
 * q : N x (K*bits/8) bytes; the codes of a row form a little-endian bit stream, element k
 *     at bits [bits*k, bits*k + bits) of the row's bytes (row n starts at byte
 *     n*K*bits/8). For bits = 4 this is exactly the layout of w4a8_pack_affine.
 * scale_bf16, bias_bf16 : out, N x K/group bf16 bit patterns.
 * w4a8_gemm_affine_nbit computes y = x . W^T exactly as w4a8_gemm_affine does (per
 * activation block b inside group g: y += d_x * (s_g * sum q*q_x + b_g * sum q_x)), with
 * the output epilogue of w4a8_gemm_epi (`epi` may be NULL). bits = 4 takes every path of
 * w4a8_gemm_affine. bits = 6 and 8: M > 64 with K/group a multiple of 8 and K*bits/8 a
 * multiple of 16 runs the CTA-pair tensor-core kernel (AUTO or PATH_GEMM), which holds
 * the weights exactly for s = 0 or 2^-17 <= |s| <= 32 and |b + c*s| <= 65504 (c =
 * 2^(bits-1)); other values set W4A8_ERR_RANGE in the device status word. Every other
 * shape runs the GEMV (no range limit); PATH_GEMM there returns UNSUPPORTED.
 * Errors: as w4a8_gemm_affine; UNSUPPORTED also for bits not 4, 6 or 8.
 */
w4a8_status w4a8_pack_affine_nbit(const void* w, w4a8_dtype dtype, int N, int K, int group, int bits,
                                  uint8_t* q, uint16_t* scale_bf16, uint16_t* bias_bf16, cudaStream_t stream);
w4a8_status w4a8_gemm_affine_nbit(int M, int N, int K, int group, int bits, const void* x, w4a8_dtype dtype,
                                  const uint8_t* q, const uint16_t* scale_bf16, const uint16_t* bias_bf16,
                                  const w4a8_epilogue* epi, void* y, void* ws, size_t ws_bytes,
                                  w4a8_path path, cudaStream_t stream);

/*
 * Q4_K weights with FP32 activations (C-Kernel-Engine gemm_kernels_q4k.c, "GEMV: y = W @ x"
 * and "Backward Pass: Gradient w.r.t. Input"; the page follows the llama.cpp Q4_K layout).
 * w_q4k : N rows, each K/256 super-blocks of 144 bytes: d (fp16), dmin (fp16), 12 bytes of
 *         packed 6-bit sub-block scales sc[8] and mins m[8] (j < 4: sc = s[j] & 63,
 *         m = s[j+4] & 63; j >= 4: sc = (s[j+4] & 15) | (s[j-4] >> 6) << 4,
 *         m = (s[j+4] >> 4) | (s[j] >> 6) << 4), 128 code bytes (byte 32i + l: element
 *         64i + l in the low nibble, sub-block 2i; element 64i + 32 + l in the high nibble,
 *         sub-block 2i + 1). Weight: w = d*sc*q - dmin*m. K must be a multiple of 256.
 * w4a8_gemv_q4_k          : y[m][n] = sum_k w[n][k] * x[m][k]; x M x K f32, y M x N f32.
 * w4a8_gemv_q4_k_backward : dx[m][k] = sum_n w[n][k] * dy[m][n] (the input gradient of
 *                           y = x W^T; the weights get none); dy M x N f32, dx M x K f32.
 *                           `ws` of w4a8_q4_k_backward_workspace_bytes(M, N, K) bytes holds
 *                           partial sums over row ranges, added in a fixed order (the
 *                           result does not depend on scheduling). The size depends on the
 *                           current device's SM count (query it with that device current);
 *                           it is 16 when the shape needs a single row range, and then
 *                           `ws` may also be NULL. Returns 0 for invalid sizes.
 * Each weight is dequantised as the page's d1 * q - m1 rounded once (d1 = d * sc, m1 = dmin
 * * m, both exact in f32); sums are taken in f32 in short chains (forward: 32 products,
 * then a row's super-blocks, then a warp; backward: at most 512 rows per range, ranges
 * added in groups of 16), so each output is within 1e-5 * sum |terms| of the exact value.
 * All pointers device memory, 16-byte aligned, caller-owned; async on `stream`.
 * Errors: INVALID_ARG (sizes, K % 256, null), MISALIGNED, WORKSPACE, CUDA.
 */
w4a8_status w4a8_gemv_q4_k(int M, int N, int K, const float* x, const uint8_t* w_q4k, float* y,
                           cudaStream_t stream);
size_t w4a8_q4_k_backward_workspace_bytes(int M, int N, int K);
w4a8_status w4a8_gemv_q4_k_backward(int M, int N, int K, const float* dy, const uint8_t* w_q4k, float* dx,
                                    void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * w4a8_gemm for callers that cannot allocate device memory. Some callers are not allowed
 * to call cudaMalloc at all: a host application that reserves every byte of device memory
 * up front and owns its allocator, or a plug-in interface whose call signature carries
 * only the inputs and the output, so there is nowhere to pass a workspace. This entry
 * point computes exactly what w4a8_gemm computes (same kernels, same results) but takes
 * its scratch from a buffer compiled into the library: a static device array of
 * W4A8_NOALLOC_SCRATCH_BYTES (every GPU that loads the library holds it until the process
 * exits). The library itself never calls cudaMalloc or cudaFree here.
 *  - The first call on each device looks up that array's device address (with that device
 *    current), so that first call should come before any stream capture. The address
 *    belongs to the device's CUDA context: after a context reset (cudaDeviceReset) the
 *    library's device code is loaded again and the array may move, so the first call in
 *    the new context looks it up again (same rule on stream capture). The looked-up
 *    address is cached under a lock; concurrent first calls from several host threads
 *    are safe.
 *  - Shapes whose minimum workspace (see w4a8_workspace_bytes) exceeds the array are
 *    rejected with W4A8_ERR_WORKSPACE; nothing is launched. Within the array the
 *    tensor-core path splits K only as far as its partial sums fit.
 *  - Every call on a device shares the one array and the array keeps whatever the last call
 *    left in it (the kernels overwrite what they read, nothing needs to start at zero).
 *    Calls whose work overlaps on the GPU (different streams, or several host threads
 *    without ordering) race on that array and corrupt each other's results: order them.
 * Arguments and the other errors as w4a8_gemm. This entry point has no counterpart on the
 * pages; it is a packaging of w4a8_gemm for allocation-free callers.
 */
#define W4A8_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
w4a8_status w4a8_gemm_noalloc(int M, int N, int K, const void* x, w4a8_dtype dtype,
                              const uint8_t* qs, const uint16_t* d_fp16, float* y,
                              cudaStream_t stream);

/*
 * Reads and clears the device status word that kernels set when a bounded wait runs
 * out or a weight scale is outside the tensor-core path's range. Synchronises the
 * current device. Returns W4A8_OK when no kernel has reported a problem since the last
 * call; else, in order of precedence: W4A8_ERR_CHECK (checked build only) if a device-side
 * check failed (the timeout that the skipped copy causes is then reported as this),
 * W4A8_ERR_DEVICE_TIMEOUT if a wait ran out, W4A8_ERR_RANGE if only a scale was out of
 * range; W4A8_ERR_CUDA if the read itself failed.
 */
w4a8_status w4a8_last_device_error(void);

/*
 * Self-test of the failure path (not an operation of the method): runs one test kernel
 * on `stream` in which a warp waits, through the library's own bounded-wait code, on an
 * mbarrier that nothing arrives at, with a limit of `limit_ns` (1 us .. 1 s), while a
 * second warp waits on another such barrier with the production limit and must stop
 * through the abort flag that the first raises. No copy or MMA is in flight. Synchronises
 * `stream`, then writes to the host word *outcome: bit 0 = the first wait ran out, bit 1 =
 * the second wait stopped, bit 2 = it stopped within 100 ms (7 = all as designed). The
 * kernel records W4A8_ERR_DEVICE_TIMEOUT in the device status word, as a real timeout
 * does; the context stays usable.
 * Errors: INVALID_ARG (outcome NULL, limit out of range), CUDA.
 */
w4a8_status w4a8_selftest_bounded_wait(unsigned long long limit_ns, unsigned int* outcome, cudaStream_t stream);

/* Description of the CUDA error behind the last W4A8_ERR_CUDA returned to this thread
 * ("no error" if there was none). Static string, never NULL. */
const char* w4a8_last_cuda_error_string(void);

/* Static, human-readable name of a status code. */
const char* w4a8_status_string(w4a8_status status);

#ifdef __cplusplus
}
#endif

#endif /* W4A8_H_ */
