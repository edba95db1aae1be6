// libw4a8: C-ABI entry points (argument checks, workspace layout, M-dispatch, launches).
// Declarations and the contract of each call: include/w4a8.h.
#include "w4a8.h"

#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "device_common.cuh"
#include "gemm_tc.cuh"
#include "gemm_pair.cuh"
#include "gemm_i8.cuh"
#include "q4k.cuh"
#include "gemv.cuh"
#include "gemv_resident.cuh"
#include "quant.cuh"

namespace {

using namespace w4a8;

// Largest M served by the dp4a GEMV when the path is AUTO and there is no int8
// tensor-core kernel for the shape (affine codes, K not a multiple of 256).
constexpr int kGemvMaxM = 8;

// Shared memory of one SM on sm_100 (228 KB; one CTA may use up to 227 KB).
constexpr int kSmemPerSm = 233472;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

inline bool dims_ok(int a, int b) { return a > 0 && b > 0 && a <= W4A8_MAX_DIM && b <= W4A8_MAX_DIM; }

// Unique ID of the calling thread's current CUDA context (false when there is none, or
// when the driver does not offer the query).
bool current_context_id(unsigned long long* id) {
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    });
    if (!get_current || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Raises a kernel's dynamic shared-memory limit to `bytes` in the calling thread's current
// context, once per kernel and context. The attribute belongs to the context's copy of the
// kernel: a context created after cudaDeviceReset starts without it, so each record keeps
// the ID of the context it was set in, and the attribute is set again whenever the current
// context has no record (or cannot be identified). The records are read and written under
// a lock, so first calls from several host threads do not race.
cudaError_t smem_limit_once(const void* func, int bytes) {
    struct Rec {
        const void* func;
        unsigned long long ctx;
        int bytes;
    };
    static std::mutex mu;
    static std::vector<Rec> recs;
    unsigned long long id = 0;
    const bool known = current_context_id(&id);
    std::lock_guard<std::mutex> lock(mu);
    if (known)
        for (const Rec& r : recs)
            if (r.func == func && r.ctx == id && r.bytes >= bytes) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess || !known) return e;
    for (Rec& r : recs)
        if (r.func == func && r.ctx == id) {
            r.bytes = bytes;
            return e;
        }
    recs.push_back({func, id, bytes});
    return e;
}

template <typename Kernel>
cudaError_t smem_limit_once(Kernel* kernel, int bytes) {
    return smem_limit_once(reinterpret_cast<const void*>(kernel), bytes);
}

// Last CUDA error a call of this thread turned into W4A8_ERR_CUDA.
thread_local cudaError_t t_last_cuda_error = cudaSuccess;

w4a8_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return W4A8_OK;
    t_last_cuda_error = e;
    return W4A8_ERR_CUDA;
}

w4a8_status launch_status() { return cuda_status(cudaGetLastError()); }

// ------------------------------------------------------------------ workspace layouts
struct GemvWs {  // row-major Q8_0 activations
    int8_t* qx;
    float* dx;
    int32_t* sx;
    size_t bytes;
};
GemvWs gemv_ws(void* ws, int M, int K) {
    const int64_t B = K / 32;
    GemvWs w{};
    size_t off = 0;
    char* base = static_cast<char*>(ws);
    w.qx = reinterpret_cast<int8_t*>(base + off); off = align256(off + size_t(M) * K);
    w.dx = reinterpret_cast<float*>(base + off); off = align256(off + size_t(M) * B * 4);
    w.sx = reinterpret_cast<int32_t*>(base + off); off = align256(off + size_t(M) * B * 4);
    w.bytes = off;
    return w;
}

// Token tile of the tensor-core GEMM for M rows of x. Up to 64 rows the tokens are the
// MMA's N (16, 32 or 64 per tile, little padding); above, tiles of 128 tokens sit on the
// TMEM lanes and the weight rows are the MMA's N.
inline int tc_token_tile(int M) { return M <= 16 ? 16 : (M <= 32 ? 32 : (M <= 64 ? 64 : 128)); }
// Token tiles: 128-token tiles are processed by CTA pairs, so their count is rounded up
// to even (the padding tile holds zero codes and scales).
inline int tc_token_tiles(int M) {
    const int tt = tc_token_tile(M);
    const int n = int(cdiv(M, tt));
    return (tt == 128) ? (n + 1) / 2 * 2 : n;
}

// Q4_0 with at most 64 tokens per tile takes the int8 tensor-core kernel (gemm_i8.cuh)
// when the scale rows can be fetched by TMA (K a multiple of 256). The decision depends on
// M, K and the format only, so the prepared form (quantise, then contract) agrees with it.
inline bool use_i8(int M, int K, int group) { return group == 0 && tc_token_tile(M) <= 64 && K % 256 == 0; }

struct TcWs {  // tensor-core operand layout (see quant_act_tc_kernel)
    __half* tok;
    float* dxs;
    float* z;
    uint4* sums;  // affine, 128-token tiles: per token and block the bias MMA's token column
    int tt;      // tokens per tile
    int tiles;
    size_t bytes;
};
TcWs tc_ws(void* ws, int M, int K, int group) {
    const int64_t B = K / 32;
    TcWs w{};
    w.tt = tc_token_tile(M);
    w.tiles = tc_token_tiles(M);
    const int64_t rows = int64_t(w.tiles) * w.tt;
    size_t off = 0;
    char* base = static_cast<char*>(ws);
    w.tok = reinterpret_cast<__half*>(base + off); off = align256(off + size_t(rows) * B * 64);
    w.dxs = reinterpret_cast<float*>(base + off); off = align256(off + size_t(rows) * B * 4);
    w.z = reinterpret_cast<float*>(base + off);
    if (group > 0) off = align256(off + size_t(rows) * (K / group) * 4);
    w.sums = reinterpret_cast<uint4*>(base + off);
    if (group > 0 && w.tt == 128) off = align256(off + size_t(rows) * B * 16);
    w.bytes = off;
    return w;
}

// ------------------------------------------------------------------ launch helpers
// Launch with programmatic dependent launch allowed (`pdl`): the kernel may start while
// the preceding kernel of the stream drains; it reads that kernel's output only after
// griddepcontrol.wait.
template <typename Kern, typename... Args>
cudaError_t launch_pdl_if(bool pdl, Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                          Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}
template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args... args) {
    return launch_pdl_if(true, kernel, grid, block, smem, stream, args...);
}

w4a8_status run_quant_rowmajor(const void* x, w4a8_dtype dt, int M, int K, int8_t* qx, float* dx, int32_t* sx,
                               cudaStream_t stream) {
    const int64_t nblocks = int64_t(M) * (K / 32);
    const dim3 grid(unsigned(cdiv(nblocks * 8, 256)));
    if (dt == W4A8_BF16)
        quant_act_rowmajor_kernel<true><<<grid, 256, 0, stream>>>(x, nblocks, qx, dx, sx);
    else
        quant_act_rowmajor_kernel<false><<<grid, 256, 0, stream>>>(x, nblocks, qx, dx, sx);
    return launch_status();
}

// `wide`: the token order of the 6- and 8-bit affine weight expansion (element order).
w4a8_status run_quant_tc(const void* x, w4a8_dtype dt, int M, int K, int group, const TcWs& w, cudaStream_t stream,
                         bool wide = false) {
    const int64_t nblocks = int64_t(w.tiles) * w.tt * (K / 32);
    const dim3 grid(unsigned(cdiv(nblocks * 8, 256)));
    if (!wide && use_i8(M, K, group)) {  // int8 token operand for gemm_i8_kernel
        int8_t* tok = reinterpret_cast<int8_t*>(w.tok);
        if (dt == W4A8_BF16)
            quant_act_i8_kernel<true><<<grid, 256, 0, stream>>>(x, M, K, w.tt, nblocks, tok, w.dxs);
        else
            quant_act_i8_kernel<false><<<grid, 256, 0, stream>>>(x, M, K, w.tt, nblocks, tok, w.dxs);
        return launch_status();
    }
    if (wide) {
        if (dt == W4A8_BF16)
            quant_act_tc_kernel<true, 2><<<grid, 256, 0, stream>>>(x, M, K, w.tt, nblocks, w.tok, w.dxs, w.z, group,
                                                                 w.sums);
        else
            quant_act_tc_kernel<false, 2><<<grid, 256, 0, stream>>>(x, M, K, w.tt, nblocks, w.tok, w.dxs, w.z, group,
                                                                  w.sums);
    } else if (group == 0) {
        const dim3 grid4(unsigned(cdiv(nblocks * 4, 256)));  // four lanes per block
        if (dt == W4A8_BF16)
            quant_act_tc4_kernel<true><<<grid4, 256, 0, stream>>>(x, M, K, w.tt, nblocks, w.tok, w.dxs);
        else
            quant_act_tc4_kernel<false><<<grid4, 256, 0, stream>>>(x, M, K, w.tt, nblocks, w.tok, w.dxs);
    } else {
        if (dt == W4A8_BF16)
            quant_act_tc_kernel<true, 1><<<grid, 256, 0, stream>>>(x, M, K, w.tt, nblocks, w.tok, w.dxs, w.z, group,
                                                                 w.tt == 128 ? w.sums : nullptr);
        else
            quant_act_tc_kernel<false, 1><<<grid, 256, 0, stream>>>(x, M, K, w.tt, nblocks, w.tok, w.dxs, w.z, group,
                                                                 w.tt == 128 ? w.sums : nullptr);
    }
    return launch_status();
}

// Largest activation (shared-memory footprint) the persistent GEMV stages, and the
// largest M*K for which each CTA quantises x itself instead of a separate kernel.
constexpr size_t kGemv2MaxSmem = 160 * 1024;
constexpr int64_t kFuseMaxElems = 16384;

int sm_count() {
    static std::atomic<int> cached[64];  // zero until filled; every filler stores the same value
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int v = cached[dev].load(std::memory_order_relaxed);
    if (v == 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        cached[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

inline int gemv_mt(int mc) { return mc == 1 ? 1 : mc == 2 ? 2 : mc <= 4 ? 4 : 8; }

// Launch one persistent-GEMV instantiation (sets its shared-memory limit once per context).
template <int MT, int FMT, int XMODE>
cudaError_t launch_gemv2(int M, int N, int K, int group, const void* x, const int8_t* qx, const float* dx,
                         const int32_t* sx, const uint8_t* wq, const uint16_t* ws, const uint16_t* wb, void* y,
                         const Epilogue& epi, cudaStream_t stream) {
    const size_t smem = gemv2_smem_bytes(MT, K);
    const cudaError_t ea = smem_limit_once(gemv2_kernel<MT, FMT, XMODE>, int(kGemv2MaxSmem));
    if (ea != cudaSuccess) return ea;
    const int64_t ctas = cdiv(N, kGemv2Warps);
    const dim3 grid(unsigned(ctas < sm_count() ? ctas : sm_count()));
    return launch_pdl(gemv2_kernel<MT, FMT, XMODE>, grid, dim3(kGemv2Threads), smem, stream, M, N, K, group, x, qx,
                      dx, sx, wq, ws, wb, y, epi);
}

template <int FMT, int XMODE>
cudaError_t launch_gemv2_mt(int mt, int M, int N, int K, int group, const void* x, const int8_t* qx, const float* dx,
                            const int32_t* sx, const uint8_t* wq, const uint16_t* ws, const uint16_t* wb, void* y,
                            const Epilogue& epi, cudaStream_t stream) {
    switch (mt) {
        case 1: return launch_gemv2<1, FMT, XMODE>(M, N, K, group, x, qx, dx, sx, wq, ws, wb, y, epi, stream);
        case 2: return launch_gemv2<2, FMT, XMODE>(M, N, K, group, x, qx, dx, sx, wq, ws, wb, y, epi, stream);
        case 4: return launch_gemv2<4, FMT, XMODE>(M, N, K, group, x, qx, dx, sx, wq, ws, wb, y, epi, stream);
        default: return launch_gemv2<8, FMT, XMODE>(M, N, K, group, x, qx, dx, sx, wq, ws, wb, y, epi, stream);
    }
}

// ------------------------------------------------------------------ resident GEMV
// Geometry of one gemv_resident_kernel launch (see gemv_resident.cuh); ok = false when the
// shape does not suit it: scale rows not a whole number of 16-byte pieces, K too long for
// the lanes' registers, or a CTA's weights (beside the activation) beyond its share of
// shared memory -- those shapes take gemv2_kernel.
struct GvPlan {
    bool ok = false;
    int xs = 1, lnsw = 0, grid = 1;
    size_t smem = 0;
};
// Shared memory per CTA such that two CTAs (of consecutive calls) fit on one SM.
constexpr size_t kGvSmemMax = 112 * 1024;

GvPlan gv_plan(int mt, int N, int K, int group, bool affine, bool quantise) {
    GvPlan p;
    const int B = K / 32;
    const int E = affine ? K / group : B;
    if (E % 8 != 0) return p;
    const int NS = (B + 31) / 32;
    const int G = N < sm_count() ? N : sm_count();
    const int rc = int(cdiv(N, G));  // rows of the largest CTA
    const size_t smem = gv::kHeaderBytes + gv::xregion_bytes(mt, K, quantise) +
                        gv::resident_weight_bytes(rc, K, E, affine);
    if (smem > kGvSmemMax) return p;
    // Blocks per lane and row (xs): registers hold 8 words of x per block and token. The
    // slice warps of a row group are the power of two covering the row's slices.
    int64_t best = -1;
    for (int c : {1, 2, 4}) {
        if (c * mt > 8) continue;
        int lnsw = 0;
        while ((1 << lnsw) * c < NS) ++lnsw;
        if (lnsw > 3) continue;
        const int H = gv::warps_for(mt) >> lnsw;
        const int64_t T = cdiv(rc, H);  // rows per group
        // issue-slot estimate per warp: row-block dots, one reduce-scatter per pass (and a
        // block barrier when a row's slices are on several warps), x codes per owned block
        const int64_t cost =
            T * c * (10 + 14 * mt) + cdiv(T, gv::rows_per_pass(mt, c)) * (40 + (lnsw ? 60 : 0)) + c * mt * 24;
        if (best < 0 || cost < best) {
            best = cost;
            p.xs = c;
            p.lnsw = lnsw;
        }
    }
    if (best < 0) return p;
    p.grid = G;
    p.smem = smem;
    p.ok = true;
    return p;
}

template <int MT, int FMT, bool QX, int XS>
cudaError_t launch_gv(const GvPlan& p, int M, int N, int K, int group, const void* x, int xbf16, const int8_t* qx,
                      const float* dx, const int32_t* sx, const uint8_t* wq, const uint16_t* ws, const uint16_t* wb,
                      void* y, const Epilogue& epi, cudaStream_t stream) {
    const cudaError_t ea = smem_limit_once(gv::gemv_resident_kernel<MT, FMT, QX, XS>, int(kGvSmemMax));
    if (ea != cudaSuccess) return ea;
    return launch_pdl(gv::gemv_resident_kernel<MT, FMT, QX, XS>, dim3(unsigned(p.grid)),
                      dim3(gv::warps_for(MT) * 32), p.smem, stream, M, N, K, group, x, xbf16, qx, dx, sx, wq, ws, wb,
                      y, epi, p.lnsw);
}

template <int FMT, bool QX>
cudaError_t launch_gv_mt(const GvPlan& p, int mt, int M, int N, int K, int group, const void* x, int xbf16,
                         const int8_t* qx, const float* dx, const int32_t* sx, const uint8_t* wq, const uint16_t* ws,
                         const uint16_t* wb, void* y, const Epilogue& epi, cudaStream_t stream) {
#define W4A8_GV(MT_, XS_) \
    launch_gv<MT_, FMT, QX, XS_>(p, M, N, K, group, x, xbf16, qx, dx, sx, wq, ws, wb, y, epi, stream)
    switch (mt * 8 + p.xs) {
        case 1 * 8 + 1: return W4A8_GV(1, 1);
        case 1 * 8 + 2: return W4A8_GV(1, 2);
        case 1 * 8 + 4: return W4A8_GV(1, 4);
        case 2 * 8 + 1: return W4A8_GV(2, 1);
        case 2 * 8 + 2: return W4A8_GV(2, 2);
        case 2 * 8 + 4: return W4A8_GV(2, 4);
        case 4 * 8 + 1: return W4A8_GV(4, 1);
        case 4 * 8 + 2: return W4A8_GV(4, 2);
        case 8 * 8 + 1: return W4A8_GV(8, 1);
        default: return cudaErrorInvalidConfiguration;
    }
#undef W4A8_GV
}

// True when one call can quantise x inside the GEMV (no separate act-quant launch).
inline bool gemv_fused(int M, int K) {
    return int64_t(M) * K <= kFuseMaxElems && gemv2_smem_bytes(gemv_mt(M < 8 ? M : 8), K) <= kGemv2MaxSmem && M <= 8;
}

// GEMV contraction from a prepared row-major Q8_0 workspace, in chunks of 8 rows of x.
template <int FMT>
w4a8_status run_gemv(int M, int N, int K, int group, const GemvWs& a, const uint8_t* wq, const uint16_t* ws,
                     const uint16_t* wb, void* y, const Epilogue& epi, cudaStream_t stream) {
    const int B = K / 32;
    for (int m0 = 0; m0 < M; m0 += 8) {
        const int mc = (M - m0 < 8) ? (M - m0) : 8;
        const int mt = gemv_mt(mc);
        const int8_t* qx = a.qx + int64_t(m0) * K;
        const float* dx = a.dx + int64_t(m0) * B;
        const int32_t* sx = a.sx + int64_t(m0) * B;
        void* yy = static_cast<char*>(y) + int64_t(m0) * N * (epi.out_bf16 ? 2 : 4);
        cudaError_t e;
        const GvPlan p = gv_plan(mt, N, K, group, FMT == 1, false);
        if (p.ok) {
            e = launch_gv_mt<FMT, false>(p, mt, mc, N, K, group, nullptr, 0, qx, dx, sx, wq, ws, wb, yy, epi, stream);
        } else if (gemv2_smem_bytes(mt, K) <= kGemv2MaxSmem) {
            e = launch_gemv2_mt<FMT, 0>(mt, mc, N, K, group, nullptr, qx, dx, sx, wq, ws, wb, yy, epi, stream);
        } else {  // activation too large for shared memory: stream it from L1/L2
            const dim3 grid(unsigned(cdiv(N, kGemvWarps)));
            const dim3 block(kGemvWarps * 32);
            if (mt == 1)
                e = launch_pdl(gemv_kernel<1, FMT>, grid, block, 0, stream, mc, N, K, group, qx, dx, sx, wq, ws, wb, yy, epi);
            else if (mt == 2)
                e = launch_pdl(gemv_kernel<2, FMT>, grid, block, 0, stream, mc, N, K, group, qx, dx, sx, wq, ws, wb, yy, epi);
            else if (mt == 4)
                e = launch_pdl(gemv_kernel<4, FMT>, grid, block, 0, stream, mc, N, K, group, qx, dx, sx, wq, ws, wb, yy, epi);
            else
                e = launch_pdl(gemv_kernel<8, FMT>, grid, block, 0, stream, mc, N, K, group, qx, dx, sx, wq, ws, wb, yy, epi);
        }
        if (e != cudaSuccess) return cuda_status(e);
    }
    return W4A8_OK;
}

// GEMV for 6- and 8-bit affine codes from a prepared row-major Q8_0 workspace, in
// chunks of 8 rows of x.
template <int BITS>
w4a8_status run_gemv_wide(int M, int N, int K, int group, const GemvWs& a, const uint8_t* wq, const uint16_t* ws,
                          const uint16_t* wb, void* y, const Epilogue& epi, cudaStream_t stream) {
    const int B = K / 32;
    const dim3 grid(unsigned(cdiv(N, kGemvWarps)));
    const dim3 block(kGemvWarps * 32);
    for (int m0 = 0; m0 < M; m0 += 8) {
        const int mc = (M - m0 < 8) ? (M - m0) : 8;
        const int mt = gemv_mt(mc);
        const int8_t* qx = a.qx + int64_t(m0) * K;
        const float* dx = a.dx + int64_t(m0) * B;
        const int32_t* sx = a.sx + int64_t(m0) * B;
        void* yy = static_cast<char*>(y) + int64_t(m0) * N * (epi.out_bf16 ? 2 : 4);
        cudaError_t e;
        if (mt == 1)
            e = launch_pdl(gemv_wide_kernel<1, BITS>, grid, block, 0, stream, mc, N, K, group, qx, dx, sx, wq, ws, wb, yy, epi);
        else if (mt == 2)
            e = launch_pdl(gemv_wide_kernel<2, BITS>, grid, block, 0, stream, mc, N, K, group, qx, dx, sx, wq, ws, wb, yy, epi);
        else if (mt == 4)
            e = launch_pdl(gemv_wide_kernel<4, BITS>, grid, block, 0, stream, mc, N, K, group, qx, dx, sx, wq, ws, wb, yy, epi);
        else
            e = launch_pdl(gemv_wide_kernel<8, BITS>, grid, block, 0, stream, mc, N, K, group, qx, dx, sx, wq, ws, wb, yy, epi);
        if (e != cudaSuccess) return cuda_status(e);
    }
    return W4A8_OK;
}

// One-launch GEMV that quantises x itself (requires gemv_fused(M, K)).
template <int FMT>
w4a8_status run_gemv_fused(int M, int N, int K, int group, const void* x, w4a8_dtype dt, const uint8_t* wq,
                           const uint16_t* ws, const uint16_t* wb, void* y, const Epilogue& epi, cudaStream_t stream) {
    const int mt = gemv_mt(M);
    const GvPlan p = gv_plan(mt, N, K, group, FMT == 1, true);
    if (p.ok)
        return cuda_status(launch_gv_mt<FMT, true>(p, mt, M, N, K, group, x, dt == W4A8_BF16 ? 1 : 0, nullptr, nullptr,
                                                   nullptr, wq, ws, wb, y, epi, stream));
    cudaError_t e = (dt == W4A8_BF16)
                        ? launch_gemv2_mt<FMT, 2>(mt, M, N, K, group, x, nullptr, nullptr, nullptr, wq, ws, wb, y, epi, stream)
                        : launch_gemv2_mt<FMT, 1>(mt, M, N, K, group, x, nullptr, nullptr, nullptr, wq, ws, wb, y, epi, stream);
    return cuda_status(e);
}

// ------------------------------------------------------------------ split of K
// When the output tiles do not fill the SMs, K is split over blockIdx.z (at least 16
// blocks per split, splits of a multiple of 8 blocks) and a reduction kernel sums the
// partial outputs, kept in the workspace after the operand region, in split order.
struct KSplit {
    int ks;      // splits actually used
    int bsplit;  // blocks per split
};
inline int64_t tc_tiles(int M, int N) { return cdiv(N, 128) * tc_token_tiles(M); }
inline size_t partial_bytes(int ks, int M, int N) { return ks > 1 ? align256(size_t(ks) * M * N * 4) : 0; }
// Longest chain of per-block f32 additions the tensor-core epilogue makes for one output.
// Summing n terms one rounding at a time errs by at most n * 2^-24 * sum|terms|. With at
// most 128 blocks per split, the splits added in groups of 16 (at most 15 + 15 roundings
// for ks <= 256, i.e. K <= 2^20) and the two roundings of the weight operand's hi/lo parts,
// every output stays within (128 + 30 + 2) * 2^-24 < 9.6e-6 of the exact sum relative to
// sum|terms|: inside the API's 1e-5 tolerance at every K.
constexpr int kMaxChainBlocks = 128;
inline int tc_split_min(int K) { return int(cdiv(K / 32, kMaxChainBlocks)); }
int tc_split_pref(int M, int N, int K) {
    const int kmin = tc_split_min(K);
    if ((int64_t(M) * N) % 4 != 0) return kmin;  // the fast reduction works on float4
    const int64_t tiles = tc_tiles(M, N);
    const int sms = sm_count();
    if (tiles >= sms) return kmin;
    int ks = int(sms / tiles);
    const int by_k = (K / 32) / 16;
    if (ks > by_k) ks = by_k;
    return ks < kmin ? kmin : ks;
}
// The split for this call: the preferred one, reduced until its partials fit `work_bytes`,
// but never below the split that bounds the accumulation chain.
KSplit tc_split(int M, int N, int K, size_t base_bytes, size_t work_bytes) {
    const int B = K / 32;
    const int kmin = tc_split_min(K);
    int ks = tc_split_pref(M, N, K);
    while (ks > kmin && base_bytes + partial_bytes(ks, M, N) > work_bytes) --ks;
    KSplit sp{1, B};
    if (ks > 1) {
        sp.bsplit = int((cdiv(B, ks) + 7) / 8 * 8);
        sp.ks = int(cdiv(B, sp.bsplit));
        if (sp.ks < 2) sp = KSplit{1, B};
    }
    return sp;
}

// Sum of the ks partial outputs in split order (+ epilogue) into y.
w4a8_status run_splitk_reduce(const float* part, int ks, int M, int N, void* y, const Epilogue& epi,
                              cudaStream_t stream) {
    const int64_t n = int64_t(M) * N;
    const int64_t units = (n % 4 == 0) ? n / 4 : n;
    int64_t rb = cdiv(units, 256);
    if (rb > 4 * int64_t(sm_count())) rb = 4 * int64_t(sm_count());
    cudaError_t e;
    if (n % 4 == 0)
        e = launch_pdl(tc::splitk_reduce_kernel, dim3(unsigned(rb)), dim3(256), 0, stream,
                       reinterpret_cast<const float4*>(part), ks, units, N, y, epi);
    else
        e = launch_pdl(tc::splitk_reduce_scalar_kernel, dim3(unsigned(rb)), dim3(256), 0, stream, part, ks, n, N, y,
                       epi);
    return cuda_status(e);
}

// cuTensorMapEncodeTiled, resolved once through the runtime (no link against the driver
// library).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {  // initialised once, thread-safe
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        return PFN_cuTensorMapEncodeTiled_v12000(nullptr);
    }();
    return fn;
}

// 2-D tensor map over a row-major [rows][cols] array of `esize`-byte elements with row
// pitch `pitch` bytes, box [box_rows][box_cols]; zero fill outside; no swizzle unless given.
bool encode_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int esize, uint64_t cols, uint64_t rows,
               uint64_t pitch, uint32_t box_cols, uint32_t box_rows,
               CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {pitch};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    (void)esize;
    return enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int FMT, bool TOKL, int MN>
w4a8_status launch_gemm_tc(int M, int N, int K, int group, const TcWs& w, const uint8_t* wq, const uint16_t* ws,
                           const uint16_t* wb, void* y, const Epilogue& epi, bool pdl, size_t work_bytes,
                           cudaStream_t stream) {
    using Gm = tc::Geo<FMT, TOKL, MN>;
    const cudaError_t ea = smem_limit_once(tc::gemm_tc_kernel<FMT, TOKL, MN>, Gm::SMEM_BYTES);
    if (ea != cudaSuccess) return cuda_status(ea);
    // Tensor maps of the packed weights: codes as bytes [N][K/2] in boxes of 16 bytes (one
    // quant block) x NW rows; scales (affine: scales and biases) as 16-bit [N][E] in boxes
    // of 8 x NW, fetched by TMA only when the row pitch 2E is a multiple of 16 bytes.
    CUtensorMap tq, tsc, tbi;
    memset(&tsc, 0, sizeof(tsc));
    memset(&tbi, 0, sizeof(tbi));
    if (!encode_2d(&tq, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(K / 2), uint64_t(N), uint64_t(K / 2), 16,
                   Gm::NW))
        return W4A8_ERR_CUDA;
    const int E = (FMT == 0) ? K / 32 : K / group;  // scales per row
    int sc_tma = ((E * 2) % 16) == 0 ? 1 : 0;
    if (sc_tma) {
        if (!encode_2d(&tsc, ws, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, uint64_t(E), uint64_t(N), uint64_t(E) * 2, 8,
                       Gm::NW))
            return W4A8_ERR_CUDA;
        if (FMT == 1 && !encode_2d(&tbi, wb, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, uint64_t(E), uint64_t(N),
                                   uint64_t(E) * 2, 8, Gm::NW))
            return W4A8_ERR_CUDA;
    }
    const KSplit sp = tc_split(M, N, K, w.bytes, work_bytes);
    float* part = reinterpret_cast<float*>(reinterpret_cast<char*>(w.tok) + w.bytes);
    const dim3 grid(unsigned(cdiv(N, Gm::NW)), unsigned(w.tiles), unsigned(sp.ks));
    cudaError_t e = launch_pdl_if(pdl, tc::gemm_tc_kernel<FMT, TOKL, MN>, grid, dim3(Gm::NUM_THREADS),
                                  size_t(Gm::SMEM_BYTES), stream, M, N, K, group, (const __half*)w.tok,
                                  (const float*)w.dxs, (const float*)w.z, wq, ws, wb, y, tq, tsc, tbi, sc_tma,
                                  sp.bsplit, part, epi);
    if (e != cudaSuccess || sp.ks == 1) return cuda_status(e);
    return run_splitk_reduce(part, sp.ks, M, N, y, epi, stream);
}

// CTA-pair kernel for 128-token tiles: two consecutive token tiles share one 128-row
// weight tile, each CTA staging half of its rows.
template <int FMT>
w4a8_status launch_gemm_pair(int M, int N, int K, int group, const TcWs& w, const uint8_t* wq, const uint16_t* ws,
                             const uint16_t* wb, void* y, const Epilogue& epi, bool pdl, size_t work_bytes,
                             cudaStream_t stream) {
    using Gm = tc::PairGeo<FMT>;
    const cudaError_t ea = smem_limit_once(tc::gemm_pair_kernel<FMT>, Gm::SMEM_BYTES);
    if (ea != cudaSuccess) return cuda_status(ea);
    CUtensorMap tq, tsc, tbi;
    memset(&tbi, 0, sizeof(tbi));
    const int E = (FMT == 0) ? K / 32 : K / group;  // scales per row (a multiple of 8 here)
    // codes: rows of K*BITS/8 bytes; 4-bit boxes of one block, wider codes one box per stage
    const uint64_t row_bytes = uint64_t(K) * Gm::BITS / 8;
    if (!encode_2d(&tq, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, row_bytes, uint64_t(N), row_bytes,
                   Gm::BITS == 4 ? 16 : Gm::S * Gm::BPB, Gm::NWH) ||
        !encode_2d(&tsc, ws, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, uint64_t(E), uint64_t(N), uint64_t(E) * 2, 8,
                   Gm::NWT))
        return W4A8_ERR_CUDA;
    if (FMT >= 1 && !encode_2d(&tbi, wb, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, uint64_t(E), uint64_t(N),
                               uint64_t(E) * 2, 8, Gm::NWT))
        return W4A8_ERR_CUDA;
    const KSplit sp = tc_split(M, N, K, w.bytes, work_bytes);
    float* part = reinterpret_cast<float*>(reinterpret_cast<char*>(w.tok) + w.bytes);
    const dim3 grid(unsigned(w.tiles), unsigned(cdiv(N, Gm::NWT)), unsigned(sp.ks));
    cudaError_t e = launch_pdl_if(pdl, tc::gemm_pair_kernel<FMT>, grid, dim3(Gm::NUM_THREADS),
                                  size_t(Gm::SMEM_BYTES), stream, M, N, K, group, (const __half*)w.tok,
                                  (const float*)w.dxs, (const uint4*)w.sums, y, tq, tsc, tbi, sp.bsplit, part, epi);
    if (e != cudaSuccess || sp.ks == 1) return cuda_status(e);
    return run_splitk_reduce(part, sp.ks, M, N, y, epi, stream);
}

// int8 tensor-core kernel for Q4_0, 16..64 tokens per tile (use_i8).
template <int MN>
w4a8_status launch_gemm_i8(int M, int N, int K, const TcWs& w, const uint8_t* wq, const uint16_t* ws, void* y,
                           const Epilogue& epi, bool pdl, size_t work_bytes, cudaStream_t stream) {
    using Gm = i8::Geo<MN>;
    const cudaError_t ea = smem_limit_once(i8::gemm_i8_kernel<MN>, Gm::SMEM_BYTES);
    if (ea != cudaSuccess) return cuda_status(ea);
    // Codes as bytes [N][K/2] in boxes of 128 bytes (8 quant blocks) x 128 rows, 128-byte
    // swizzle (K is a multiple of 256: every stage is one whole box).
    CUtensorMap tq;
    if (!encode_2d(&tq, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(K / 2), uint64_t(N), uint64_t(K / 2), 128,
                   Gm::NW, CU_TENSOR_MAP_SWIZZLE_128B))
        return W4A8_ERR_CUDA;
    // Scales as fp16 [N][K/32] in boxes of 8 (one stage) x 128 rows.
    CUtensorMap ts;
    if (!encode_2d(&ts, ws, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, uint64_t(K / 32), uint64_t(N), uint64_t(K / 32) * 2,
                   Gm::S, Gm::NW))
        return W4A8_ERR_CUDA;
    const KSplit sp = tc_split(M, N, K, w.bytes, work_bytes);
    float* part = reinterpret_cast<float*>(reinterpret_cast<char*>(w.tok) + w.bytes);
    const dim3 grid(unsigned(cdiv(N, Gm::NW)), unsigned(w.tiles), unsigned(sp.ks));
    cudaError_t e = launch_pdl_if(pdl, i8::gemm_i8_kernel<MN>, grid, dim3(Gm::NUM_THREADS), size_t(Gm::SMEM_BYTES),
                                  stream, M, N, K, (const int8_t*)w.tok, (const float*)w.dxs, y, tq, ts,
                                  sp.bsplit, part, epi);
    if (e != cudaSuccess || sp.ks == 1) return cuda_status(e);
    return run_splitk_reduce(part, sp.ks, M, N, y, epi, stream);
}

// Orientation by token tile: tiles of 16..64 tokens put the tokens on the MMA's N; tiles
// of 128 tokens put them on the TMEM lanes with 128 weight rows per tile, on CTA pairs
// when the scale rows can be fetched by TMA (their pitch a multiple of 16 bytes).
template <int FMT>
w4a8_status run_gemm_tc(int M, int N, int K, int group, const TcWs& w, const uint8_t* wq, const uint16_t* ws,
                        const uint16_t* wb, void* y, const Epilogue& epi, bool pdl, size_t work_bytes,
                        cudaStream_t stream) {
    if (FMT == 0 && use_i8(M, K, group)) {
        switch (w.tt) {
            case 16: return launch_gemm_i8<16>(M, N, K, w, wq, ws, y, epi, pdl, work_bytes, stream);
            case 32: return launch_gemm_i8<32>(M, N, K, w, wq, ws, y, epi, pdl, work_bytes, stream);
            default: return launch_gemm_i8<64>(M, N, K, w, wq, ws, y, epi, pdl, work_bytes, stream);
        }
    }
    switch (w.tt) {
        case 16: return launch_gemm_tc<FMT, false, 16>(M, N, K, group, w, wq, ws, wb, y, epi, pdl, work_bytes, stream);
        case 32: return launch_gemm_tc<FMT, false, 32>(M, N, K, group, w, wq, ws, wb, y, epi, pdl, work_bytes, stream);
        case 64: return launch_gemm_tc<FMT, false, 64>(M, N, K, group, w, wq, ws, wb, y, epi, pdl, work_bytes, stream);
        default: {
            const int E = (FMT == 0) ? K / 32 : K / group;
            if ((E * 2) % 16 == 0)
                return launch_gemm_pair<FMT>(M, N, K, group, w, wq, ws, wb, y, epi, pdl, work_bytes, stream);
            return launch_gemm_tc<FMT, true, 128>(M, N, K, group, w, wq, ws, wb, y, epi, pdl, work_bytes, stream);
        }
    }
}

inline bool use_gemv(int M, int N, int K, int group, w4a8_path path);

// Smallest workspace a call of this shape accepts on `path`: the GEMV's activation, or the
// tensor-core operand plus the partial outputs of the split of K that bounds the
// accumulation chain (K > 4096); a larger one, up to w4a8_workspace_bytes, lets the
// tensor-core path split K further to fill the SMs.
// `split`: a call of the prepare / contract pair (the path rule without N).
size_t min_workspace_bytes(int M, int N, int K, int group, w4a8_path path, bool split = false) {
    if (use_gemv(M, split ? -1 : N, K, group, path)) return gemv_ws(nullptr, M, K).bytes;
    return tc_ws(nullptr, M, K, group).bytes + partial_bytes(tc_split_min(K), M, N);
}

w4a8_status check_gemm_args(int M, int N, int K, const void* x, w4a8_dtype dt, const void* wq, const void* ws,
                            const void* wb, bool affine, int group, const void* y, const void* work,
                            size_t work_bytes, w4a8_path path, bool split = false) {
    if (!dims_ok(M, N) || !dims_ok(K, 1) || (K % 32) != 0) return W4A8_ERR_INVALID_ARG;
    if (!x || !wq || !ws || !y || (affine && !wb)) return W4A8_ERR_INVALID_ARG;
    if (dt != W4A8_F32 && dt != W4A8_BF16) return W4A8_ERR_UNSUPPORTED;
    if (path != W4A8_PATH_AUTO && path != W4A8_PATH_GEMV && path != W4A8_PATH_GEMM) return W4A8_ERR_UNSUPPORTED;
    if (affine) {
        if (group != 32 && group != 64 && group != 128) return W4A8_ERR_UNSUPPORTED;
        if (K % group != 0) return W4A8_ERR_INVALID_ARG;
    }
    if (!aligned16(x) || !aligned16(wq) || !aligned16(ws) || !aligned16(y) || (affine && !aligned16(wb)))
        return W4A8_ERR_MISALIGNED;
    if (!work) return W4A8_ERR_WORKSPACE;
    if (!aligned16(work)) return W4A8_ERR_MISALIGNED;
    if (work_bytes < min_workspace_bytes(M, N, K, affine ? group : 0, path, split)) return W4A8_ERR_WORKSPACE;
    return W4A8_OK;
}

// The epilogue of the entry points without one: f32 output, no bias.
const Epilogue kPlain{nullptr, 0, 0};

// Checks a caller's epilogue and converts it (nullptr: f32 output, no bias).
w4a8_status make_epilogue(const w4a8_epilogue* in, Epilogue* out) {
    *out = kPlain;
    if (!in) return W4A8_OK;
    if ((in->bias_dtype != W4A8_F32 && in->bias_dtype != W4A8_BF16) ||
        (in->out_dtype != W4A8_F32 && in->out_dtype != W4A8_BF16))
        return W4A8_ERR_UNSUPPORTED;
    if (in->bias && (reinterpret_cast<uintptr_t>(in->bias) & (in->bias_dtype == W4A8_BF16 ? 1u : 3u)) != 0)
        return W4A8_ERR_MISALIGNED;
    out->bias = in->bias;
    out->bias_bf16 = in->bias_dtype == W4A8_BF16 ? 1 : 0;
    out->out_bf16 = in->out_dtype == W4A8_BF16 ? 1 : 0;
    return W4A8_OK;
}

// Whether AUTO takes the GEMV. Q4_0 shapes with the int8 tensor-core kernel switch at the
// per-call times measured on B200 (weights streamed from HBM, M = 2..8): the tensor
// kernel's time is nearly flat in M up to 16 tokens while the GEMV's grows with M, so it
// wins from M = 3 on K x N = 4096 x 14336 (M = 2: 15.1 vs 15.8 us, M = 3: 20.6 vs 15.7), from
// M = 2 on 14336 x 4096 (17.7 vs 16.4: the long rows cost the GEMV more), and from M = 5 on
// 4096 x 4096 and 8192 x 2048 (M = 4: 8.2 vs 10.0 and 9.1 vs 10.9; M = 5: 14.0 vs 10.1).
// N < 0: N is not known (the prepare / contract pair), and the rule takes M and K only.
inline bool use_gemv(int M, int N, int K, int group, w4a8_path path) {
    if (path != W4A8_PATH_AUTO) return path == W4A8_PATH_GEMV;
    if (!use_i8(M, K, group)) return M <= kGemvMaxM;
    if (N < 0) return M <= 3;
    const bool small = int64_t(N) * K <= (int64_t(1) << 25);
    if (M == 1) return true;
    if (M == 2) return K <= 8192 || small;
    return M <= 4 && small;
}

// Quantise x into the workspace layout of the chosen path.
w4a8_status prepare_impl(int M, int K, int group, const void* x, w4a8_dtype dt, void* work, bool gemv,
                         cudaStream_t stream) {
    if (gemv) {
        GemvWs a = gemv_ws(work, M, K);
        return run_quant_rowmajor(x, dt, M, K, a.qx, a.dx, a.sx, stream);
    }
    return run_quant_tc(x, dt, M, K, group, tc_ws(work, M, K, group), stream);
}

// Contraction from a prepared workspace. `after_quant`: the preceding kernel in the
// stream is this call's own activation quantisation, so the contraction may overlap its
// tail (programmatic dependent launch); otherwise it starts after all prior work.
template <int FMT>
w4a8_status contract_impl(int M, int N, int K, int group, const uint8_t* wq, const uint16_t* ws, const uint16_t* wb,
                          void* y, const Epilogue& epi, void* work, size_t work_bytes, bool gemv, bool after_quant,
                          cudaStream_t stream) {
    if (gemv) return run_gemv<FMT>(M, N, K, group, gemv_ws(work, M, K), wq, ws, wb, y, epi, stream);
    return run_gemm_tc<FMT>(M, N, K, group, tc_ws(work, M, K, FMT == 1 ? group : 0), wq, ws, wb, y, epi,
                            after_quant, work_bytes, stream);
}

template <int FMT>
w4a8_status gemm_impl(int M, int N, int K, int group, const void* x, w4a8_dtype dt, const uint8_t* wq,
                      const uint16_t* ws, const uint16_t* wb, void* y, const Epilogue& epi, void* work,
                      size_t work_bytes, w4a8_path path, cudaStream_t stream) {
    w4a8_status st = check_gemm_args(M, N, K, x, dt, wq, ws, wb, FMT == 1, group, y, work, work_bytes, path);
    if (st != W4A8_OK) return st;
    const bool gemv = use_gemv(M, N, K, FMT == 1 ? group : 0, path);
    if (gemv && gemv_fused(M, K)) return run_gemv_fused<FMT>(M, N, K, group, x, dt, wq, ws, wb, y, epi, stream);
    st = prepare_impl(M, K, FMT == 1 ? group : 0, x, dt, work, gemv, stream);
    if (st != W4A8_OK) return st;
    return contract_impl<FMT>(M, N, K, group, wq, ws, wb, y, epi, work, work_bytes, gemv, true, stream);
}

// True when the CTA-pair kernel takes 6- or 8-bit codes of this shape: 128-token tiles
// (M > 64), scale rows and code rows whose pitch is a multiple of 16 bytes (TMA).
inline bool wide_pair_ok(int M, int K, int group, int bits) {
    return tc_token_tile(M) == 128 && ((K / group) * 2) % 16 == 0 && (int64_t(K) * bits / 8) % 16 == 0;
}

// Affine 6- and 8-bit codes: CTA pairs for M > 64 (AUTO or PATH_GEMM, shapes of
// wide_pair_ok), the GEMV on a prepared row-major activation otherwise (PATH_GEMM on
// other shapes is refused: there is no small-M tensor kernel for these codes).
template <int BITS>
w4a8_status gemm_wide_impl(int M, int N, int K, int group, const void* x, w4a8_dtype dt, const uint8_t* wq,
                           const uint16_t* ws, const uint16_t* wb, void* y, const Epilogue& epi, void* work,
                           size_t work_bytes, w4a8_path path, cudaStream_t stream) {
    w4a8_status st = check_gemm_args(M, N, K, x, dt, wq, ws, wb, true, group, y, work, work_bytes, path);
    if (st != W4A8_OK) return st;
    const bool pair_ok = wide_pair_ok(M, K, group, BITS);
    if (path == W4A8_PATH_GEMM && !pair_ok) return W4A8_ERR_UNSUPPORTED;
    if (pair_ok && path != W4A8_PATH_GEMV && M > kGemvMaxM) {
        const TcWs w = tc_ws(work, M, K, group);
        st = run_quant_tc(x, dt, M, K, group, w, stream, true);
        if (st != W4A8_OK) return st;
        return launch_gemm_pair<BITS == 8 ? 2 : 3>(M, N, K, group, w, wq, ws, wb, y, epi, true, work_bytes, stream);
    }
    st = prepare_impl(M, K, group, x, dt, work, true, stream);
    if (st != W4A8_OK) return st;
    return run_gemv_wide<BITS>(M, N, K, group, gemv_ws(work, M, K), wq, ws, wb, y, epi, stream);
}

template <bool BF16>
void launch_pack_affine(int bits, const void* w, int64_t ngroups, int group, uint8_t* q, uint16_t* scale,
                        uint16_t* bias, cudaStream_t stream) {
    const dim3 grid(unsigned(cdiv(ngroups * (group / 4), 256)));
    if (bits == 4)
        pack_affine_kernel<BF16, 4><<<grid, 256, 0, stream>>>(w, ngroups, group, q, scale, bias);
    else if (bits == 6)
        pack_affine_kernel<BF16, 6><<<grid, 256, 0, stream>>>(w, ngroups, group, q, scale, bias);
    else
        pack_affine_kernel<BF16, 8><<<grid, 256, 0, stream>>>(w, ngroups, group, q, scale, bias);
}

w4a8_status pack_affine_impl(const void* w, w4a8_dtype dtype, int N, int K, int group, int bits, uint8_t* q,
                             uint16_t* scale_bf16, uint16_t* bias_bf16, cudaStream_t stream) {
    if (!dims_ok(N, K) || (K % 32) != 0 || !w || !q || !scale_bf16 || !bias_bf16) return W4A8_ERR_INVALID_ARG;
    if (group != 32 && group != 64 && group != 128) return W4A8_ERR_UNSUPPORTED;
    if (bits != 4 && bits != 6 && bits != 8) return W4A8_ERR_UNSUPPORTED;
    if (K % group != 0) return W4A8_ERR_INVALID_ARG;
    if (dtype != W4A8_F32 && dtype != W4A8_BF16) return W4A8_ERR_UNSUPPORTED;
    if (!aligned16(w) || !aligned16(q) || !aligned16(scale_bf16) || !aligned16(bias_bf16)) return W4A8_ERR_MISALIGNED;
    const int64_t ngroups = int64_t(N) * (K / group);
    if (dtype == W4A8_BF16)
        launch_pack_affine<true>(bits, w, ngroups, group, q, scale_bf16, bias_bf16, stream);
    else
        launch_pack_affine<false>(bits, w, ngroups, group, q, scale_bf16, bias_bf16, stream);
    return launch_status();
}

// ------------------------------------------------------------------ Q4_K
// Row ranges of the backward: enough CTAs (super-block columns x ranges) for four per
// SM, at least 32 rows per range, at most 2048 (a lane's f32 chain of products is then at
// most 64 long).
// Row ranges of the streamed Q4_K backward: with the K/256 super-block columns, about one
// CTA per SM (at least 16 rows per range), more ranges when a range would exceed
// kBwdMaxRows rows (the bound on a lane's chain of sums).
inline int q4k_bwd_ranges(int N, int K) {
    const int nb = K / 256;
    int64_t R = cdiv(sm_count(), nb);
    const int64_t rmax = cdiv(N, 16);
    if (R > rmax) R = rmax;
    const int64_t rmin = cdiv(N, q4k::kBwdMaxRows);
    if (R < rmin) R = rmin;
    return int(R < 1 ? 1 : R);
}
inline size_t q4k_bwd_bytes(int M, int N, int K) {
    const int R = q4k_bwd_ranges(N, K);
    return R > 1 ? size_t(R) * (M < 2 ? M : 2) * K * 4 : 0;
}
template <int MT>
w4a8_status launch_q4k_bwd(int N, int K, const float* dy, const uint8_t* w, float* out, int R, cudaStream_t stream) {
    constexpr size_t smem = q4k::bwd_smem_bytes(MT);
    const cudaError_t ea = smem_limit_once(q4k::bwd_stream_kernel<MT>, int(smem));
    if (ea != cudaSuccess) return cuda_status(ea);
    // the weights as 8-byte elements [N][K/256 * 18], one box = one super-block column of 64 rows
    CUtensorMap tm;
    const uint64_t cols = uint64_t(K / 256) * (q4k::kBlockBytes / 8);
    if (!encode_2d(&tm, w, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, cols, uint64_t(N), cols * 8, q4k::kBlockBytes / 8,
                   q4k::kBwdSlotRows))
        return W4A8_ERR_CUDA;
    return cuda_status(launch_pdl(q4k::bwd_stream_kernel<MT>, dim3(unsigned((K / 256) * R)),
                                  dim3(q4k::kStreamThreads), smem, stream, MT, N, K, dy, tm, out, R));
}

template <int MT, int MINB>
w4a8_status launch_q4k_stream_b(int N, int K, const float* x, const uint8_t* w, float* y, const q4k::StreamPlan& sp,
                                cudaStream_t stream) {
    const cudaError_t ea = smem_limit_once(q4k::fwd_stream_kernel<MT, MINB>, int(tc::SMEM_LIMIT));
    if (ea != cudaSuccess) return cuda_status(ea);
    const int G = N < sm_count() ? N : sm_count();
    return cuda_status(launch_pdl(q4k::fwd_stream_kernel<MT, MINB>, dim3(unsigned(G)), dim3(q4k::kStreamThreads),
                                  sp.smem, stream, MT, N, K, x, w, y, sp.kc, sp.nst));
}
template <int MT>
w4a8_status launch_q4k_stream(int N, int K, const float* x, const uint8_t* w, float* y, const q4k::StreamPlan& sp,
                              cudaStream_t stream) {
    return sp.two_per_sm ? launch_q4k_stream_b<MT, 2>(N, K, x, w, y, sp, stream)
                         : launch_q4k_stream_b<MT, 1>(N, K, x, w, y, sp, stream);
}
w4a8_status check_q4k(int M, int N, int K, const void* a, const void* w, const void* out) {
    if (!dims_ok(M, N) || !dims_ok(K, 1) || (K % 256) != 0 || !a || !w || !out) return W4A8_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(w) || !aligned16(out)) return W4A8_ERR_MISALIGNED;
    return W4A8_OK;
}

}  // namespace

extern "C" {

w4a8_status w4a8_gemv_q4_k(int M, int N, int K, const float* x, const uint8_t* w_q4k, float* y,
                           cudaStream_t stream) {
    const w4a8_status st = check_q4k(M, N, K, x, w_q4k, y);
    if (st != W4A8_OK) return st;
    const dim3 grid(unsigned(cdiv(N, 16)));  // 16 rows per CTA
    for (int m0 = 0; m0 < M; m0 += 2) {
        const int mt = (M - m0 < 2) ? (M - m0) : 2;
        // The streamed kernel where x of the launch's tokens fits in shared memory beside
        // the weight ring; the 16-rows-per-CTA kernel otherwise.
        const q4k::StreamPlan sp = q4k::stream_plan(mt, K, size_t(tc::SMEM_LIMIT), size_t(kSmemPerSm));
        if (sp.ok) {
            const w4a8_status ls = mt == 1 ? launch_q4k_stream<1>(N, K, x + int64_t(m0) * K, w_q4k,
                                                                  y + int64_t(m0) * N, sp, stream)
                                           : launch_q4k_stream<2>(N, K, x + int64_t(m0) * K, w_q4k,
                                                                  y + int64_t(m0) * N, sp, stream);
            if (ls != W4A8_OK) return ls;
            continue;
        }
        if (mt == 1)
            q4k::gemv_kernel<1><<<grid, q4k::kThreads, 0, stream>>>(1, N, K, x + int64_t(m0) * K, w_q4k,
                                                                   y + int64_t(m0) * N);
        else
            q4k::gemv_kernel<2><<<grid, q4k::kThreads, 0, stream>>>(2, N, K, x + int64_t(m0) * K, w_q4k,
                                                                   y + int64_t(m0) * N);
        const w4a8_status ls = launch_status();
        if (ls != W4A8_OK) return ls;
    }
    return W4A8_OK;
}

size_t w4a8_q4_k_backward_workspace_bytes(int M, int N, int K) {
    if (!dims_ok(M, N) || !dims_ok(K, 1) || (K % 256) != 0) return 0;
    const size_t b = q4k_bwd_bytes(M, N, K);
    return b ? b : 16;
}

w4a8_status w4a8_gemv_q4_k_backward(int M, int N, int K, const float* dy, const uint8_t* w_q4k, float* dx,
                                    void* ws, size_t ws_bytes, cudaStream_t stream) {
    w4a8_status st = check_q4k(M, N, K, dy, w_q4k, dx);
    if (st != W4A8_OK) return st;
    const int R = q4k_bwd_ranges(N, K);
    const size_t need = q4k_bwd_bytes(M, N, K);
    if (need > 0) {
        if (!ws || ws_bytes < need) return W4A8_ERR_WORKSPACE;
        if (!aligned16(ws)) return W4A8_ERR_MISALIGNED;
    }
    float* part = static_cast<float*>(ws);
    for (int m0 = 0; m0 < M; m0 += 2) {
        const int mt = (M - m0 < 2) ? (M - m0) : 2;
        const float* dyc = dy + int64_t(m0) * N;
        float* dxc = dx + int64_t(m0) * K;
        float* out = R > 1 ? part : dxc;
        st = mt == 1 ? launch_q4k_bwd<1>(N, K, dyc, w_q4k, out, R, stream)
                     : launch_q4k_bwd<2>(N, K, dyc, w_q4k, out, R, stream);
        if (st != W4A8_OK) return st;
        if (R > 1) {
            const int64_t count = int64_t(mt) * K;
            int64_t nblk = cdiv(count, 256);
            if (nblk > 4 * int64_t(sm_count())) nblk = 4 * int64_t(sm_count());
            q4k::bwd_reduce_kernel<<<unsigned(nblk), 256, 0, stream>>>(part, R, count, dxc);
            st = launch_status();
            if (st != W4A8_OK) return st;
        }
    }
    return W4A8_OK;
}

w4a8_status w4a8_pack_q4_0(const void* w, w4a8_dtype dtype, int N, int K, uint8_t* qs, uint16_t* d_fp16,
                           cudaStream_t stream) {
    if (!dims_ok(N, K) || (K % 32) != 0 || !w || !qs || !d_fp16) return W4A8_ERR_INVALID_ARG;
    if (dtype != W4A8_F32 && dtype != W4A8_BF16) return W4A8_ERR_UNSUPPORTED;
    if (!aligned16(w) || !aligned16(qs) || !aligned16(d_fp16)) return W4A8_ERR_MISALIGNED;
    const int64_t nblocks = int64_t(N) * (K / 32);
    const dim3 grid(unsigned(cdiv(nblocks * 8, 256)));
    if (dtype == W4A8_BF16)
        pack_q4_0_kernel<true><<<grid, 256, 0, stream>>>(w, nblocks, qs, d_fp16);
    else
        pack_q4_0_kernel<false><<<grid, 256, 0, stream>>>(w, nblocks, qs, d_fp16);
    return launch_status();
}

w4a8_status w4a8_quant_act_q8_0(const void* x, w4a8_dtype dtype, int M, int K, int8_t* qx, float* dx, int32_t* sx,
                                cudaStream_t stream) {
    if (!dims_ok(M, K) || (K % 32) != 0 || !x || !qx || !dx) return W4A8_ERR_INVALID_ARG;
    if (dtype != W4A8_F32 && dtype != W4A8_BF16) return W4A8_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(qx) || !aligned16(dx) || (sx && !aligned16(sx))) return W4A8_ERR_MISALIGNED;
    return run_quant_rowmajor(x, dtype, M, K, qx, dx, sx, stream);
}

size_t w4a8_workspace_bytes(int M, int N, int K, int group) {
    if (!dims_ok(M, N) || !dims_ok(K, 1) || (K % 32) != 0) return 0;
    if (group != 0 && (group != 32 && group != 64 && group != 128)) return 0;
    if (group != 0 && (K % group) != 0) return 0;
    const size_t a = gemv_ws(nullptr, M, K).bytes;
    const size_t b = tc_ws(nullptr, M, K, group).bytes + partial_bytes(tc_split_pref(M, N, K), M, N);
    return a > b ? a : b;
}

int w4a8_gemm_path(int M, int N, int K, int group, w4a8_path path) {
    if (!dims_ok(M, N) || !dims_ok(K, 1) || (K % 32) != 0) return 0;
    if (group != 0 && ((group != 32 && group != 64 && group != 128) || (K % group) != 0)) return 0;
    if (path != W4A8_PATH_AUTO && path != W4A8_PATH_GEMV && path != W4A8_PATH_GEMM) return 0;
    if (use_gemv(M, N, K, group, path)) return W4A8_KERNEL_GEMV;
    if (group == 0 && use_i8(M, K, group)) return W4A8_KERNEL_TC_INT8;
    if (tc_token_tile(M) <= 64) return W4A8_KERNEL_TC_FP16;
    const int E = group == 0 ? K / 32 : K / group;
    return (E * 2) % 16 == 0 ? W4A8_KERNEL_TC_PAIR : W4A8_KERNEL_TC_FP16;
}

w4a8_status w4a8_gemm_ex(int M, int N, int K, const void* x, w4a8_dtype dtype, const uint8_t* qs,
                         const uint16_t* d_fp16, float* y, void* ws, size_t ws_bytes, w4a8_path path,
                         cudaStream_t stream) {
    return gemm_impl<0>(M, N, K, 0, x, dtype, qs, d_fp16, nullptr, y, kPlain, ws, ws_bytes, path, stream);
}

w4a8_status w4a8_gemm(int M, int N, int K, const void* x, w4a8_dtype dtype, const uint8_t* qs,
                      const uint16_t* d_fp16, float* y, void* ws, size_t ws_bytes, cudaStream_t stream) {
    return w4a8_gemm_ex(M, N, K, x, dtype, qs, d_fp16, y, ws, ws_bytes, W4A8_PATH_AUTO, stream);
}

w4a8_status w4a8_pack_affine(const void* w, w4a8_dtype dtype, int N, int K, int group, uint32_t* q,
                             uint16_t* scale_bf16, uint16_t* bias_bf16, cudaStream_t stream) {
    return pack_affine_impl(w, dtype, N, K, group, 4, reinterpret_cast<uint8_t*>(q), scale_bf16, bias_bf16, stream);
}

w4a8_status w4a8_pack_affine_nbit(const void* w, w4a8_dtype dtype, int N, int K, int group, int bits, uint8_t* q,
                                  uint16_t* scale_bf16, uint16_t* bias_bf16, cudaStream_t stream) {
    return pack_affine_impl(w, dtype, N, K, group, bits, q, scale_bf16, bias_bf16, stream);
}

w4a8_status w4a8_gemm_affine_nbit(int M, int N, int K, int group, int bits, const void* x, w4a8_dtype dtype,
                                  const uint8_t* q, const uint16_t* scale_bf16, const uint16_t* bias_bf16,
                                  const w4a8_epilogue* epi, void* y, void* ws, size_t ws_bytes, w4a8_path path,
                                  cudaStream_t stream) {
    Epilogue e;
    const w4a8_status st = make_epilogue(epi, &e);
    if (st != W4A8_OK) return st;
    switch (bits) {
        case 4:
            return gemm_impl<1>(M, N, K, group, x, dtype, q, scale_bf16, bias_bf16, y, e, ws, ws_bytes, path, stream);
        case 6:
            return gemm_wide_impl<6>(M, N, K, group, x, dtype, q, scale_bf16, bias_bf16, y, e, ws, ws_bytes, path,
                                     stream);
        case 8:
            return gemm_wide_impl<8>(M, N, K, group, x, dtype, q, scale_bf16, bias_bf16, y, e, ws, ws_bytes, path,
                                     stream);
        default:
            return W4A8_ERR_UNSUPPORTED;
    }
}

w4a8_status w4a8_gemm_affine_ex(int M, int N, int K, int group, const void* x, w4a8_dtype dtype, const uint32_t* q,
                                const uint16_t* scale_bf16, const uint16_t* bias_bf16, float* y, void* ws,
                                size_t ws_bytes, w4a8_path path, cudaStream_t stream) {
    return gemm_impl<1>(M, N, K, group, x, dtype, reinterpret_cast<const uint8_t*>(q), scale_bf16, bias_bf16, y, kPlain, ws,
                        ws_bytes, path, stream);
}

w4a8_status w4a8_gemm_affine(int M, int N, int K, int group, const void* x, w4a8_dtype dtype, const uint32_t* q,
                             const uint16_t* scale_bf16, const uint16_t* bias_bf16, float* y, void* ws,
                             size_t ws_bytes, cudaStream_t stream) {
    return w4a8_gemm_affine_ex(M, N, K, group, x, dtype, q, scale_bf16, bias_bf16, y, ws, ws_bytes, W4A8_PATH_AUTO,
                               stream);
}

w4a8_status w4a8_prepare_act(int M, int K, int group, const void* x, w4a8_dtype dtype, void* ws, size_t ws_bytes,
                             w4a8_path path, cudaStream_t stream) {
    const bool affine = group != 0;
    // the weight pointers are not used here; pass x so their null / alignment checks pass
    w4a8_status st = check_gemm_args(M, 1, K, x, dtype, x, x, x, affine, group, static_cast<const float*>(x), ws,
                                     ws_bytes, path, true);
    if (st != W4A8_OK) return st;
    return prepare_impl(M, K, group, x, dtype, ws, use_gemv(M, -1, K, group, path), stream);
}

w4a8_status w4a8_gemm_epi(int M, int N, int K, const void* x, w4a8_dtype dtype, const uint8_t* qs,
                          const uint16_t* d_fp16, const w4a8_epilogue* epi, void* y, void* ws, size_t ws_bytes,
                          w4a8_path path, cudaStream_t stream) {
    Epilogue e;
    const w4a8_status st = make_epilogue(epi, &e);
    if (st != W4A8_OK) return st;
    return gemm_impl<0>(M, N, K, 0, x, dtype, qs, d_fp16, nullptr, y, e, ws, ws_bytes, path, stream);
}

w4a8_status w4a8_gemm_affine_epi(int M, int N, int K, int group, const void* x, w4a8_dtype dtype, const uint32_t* q,
                                 const uint16_t* scale_bf16, const uint16_t* bias_bf16, const w4a8_epilogue* epi,
                                 void* y, void* ws, size_t ws_bytes, w4a8_path path, cudaStream_t stream) {
    Epilogue e;
    const w4a8_status st = make_epilogue(epi, &e);
    if (st != W4A8_OK) return st;
    return gemm_impl<1>(M, N, K, group, x, dtype, reinterpret_cast<const uint8_t*>(q), scale_bf16, bias_bf16, y, e,
                        ws, ws_bytes, path, stream);
}

w4a8_status w4a8_gemm_prepared(int M, int N, int K, const uint8_t* qs, const uint16_t* d_fp16, float* y,
                               const void* ws, size_t ws_bytes, w4a8_path path, cudaStream_t stream) {
    w4a8_status st =
        check_gemm_args(M, N, K, qs, W4A8_F32, qs, d_fp16, nullptr, false, 0, y, ws, ws_bytes, path, true);
    if (st != W4A8_OK) return st;
    return contract_impl<0>(M, N, K, 0, qs, d_fp16, nullptr, y, kPlain, const_cast<void*>(ws), ws_bytes,
                            use_gemv(M, -1, K, 0, path), false, stream);
}

w4a8_status w4a8_gemm_affine_prepared(int M, int N, int K, int group, const uint32_t* q, const uint16_t* scale_bf16,
                                      const uint16_t* bias_bf16, float* y, const void* ws, size_t ws_bytes,
                                      w4a8_path path, cudaStream_t stream) {
    const uint8_t* wq = reinterpret_cast<const uint8_t*>(q);
    w4a8_status st =
        check_gemm_args(M, N, K, wq, W4A8_F32, wq, scale_bf16, bias_bf16, true, group, y, ws, ws_bytes, path, true);
    if (st != W4A8_OK) return st;
    return contract_impl<1>(M, N, K, group, wq, scale_bf16, bias_bf16, y, kPlain, const_cast<void*>(ws), ws_bytes,
                            use_gemv(M, -1, K, group, path), false, stream);
}

// Scratch of w4a8_gemm_noalloc. In host code this name is only a stand-in for the
// device array; its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_noalloc_scratch[W4A8_NOALLOC_SCRATCH_BYTES];

}  // extern "C"

namespace {

// Device address of g_noalloc_scratch in the current context of device `dev`. The address
// belongs to a context, not to a device: after cudaDeviceReset the next context loads the
// library's device code again and the array may sit elsewhere. So the looked-up address is
// kept per device together with the ID of the context it was looked up in, and looked up
// again whenever the current context differs (or cannot be identified). The cache is read
// and filled under a lock, so first calls from several host threads do not race.
cudaError_t noalloc_scratch_address(int dev, void** out) {
    static std::mutex mu;
    static bool valid[64] = {false};
    static unsigned long long ctx_of[64] = {0};
    static void* addr_of[64] = {nullptr};
    std::lock_guard<std::mutex> lock(mu);
    unsigned long long id = 0;
    if (valid[dev] && current_context_id(&id) && id == ctx_of[dev]) {
        *out = addr_of[dev];
        return cudaSuccess;
    }
    void* p = nullptr;  // this lookup also creates the device's primary context if needed
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    valid[dev] = current_context_id(&id);
    ctx_of[dev] = id;
    addr_of[dev] = p;
    *out = p;
    return cudaSuccess;
}

}  // namespace

extern "C" {

w4a8_status w4a8_gemm_noalloc(int M, int N, int K, const void* x, w4a8_dtype dtype, const uint8_t* qs,
                              const uint16_t* d_fp16, float* y, cudaStream_t stream) {
    const size_t need =
        (dims_ok(M, N) && dims_ok(K, 1) && K % 32 == 0) ? min_workspace_bytes(M, N, K, 0, W4A8_PATH_AUTO) : 0;
    if (need == 0) return W4A8_ERR_INVALID_ARG;
    if (need > W4A8_NOALLOC_SCRATCH_BYTES) return W4A8_ERR_WORKSPACE;
    int dev = 0;
    const cudaError_t ed = cudaGetDevice(&dev);
    if (ed != cudaSuccess) return cuda_status(ed);
    if (dev < 0 || dev >= 64) return W4A8_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    const cudaError_t es = noalloc_scratch_address(dev, &scratch);
    if (es != cudaSuccess) return cuda_status(es);
    return gemm_impl<0>(M, N, K, 0, x, dtype, qs, d_fp16, nullptr, y, kPlain, scratch, W4A8_NOALLOC_SCRATCH_BYTES,
                        W4A8_PATH_AUTO, stream);
}

// Outcome word of w4a8_selftest_bounded_wait.
static __device__ unsigned int g_selftest_outcome;

w4a8_status w4a8_selftest_bounded_wait(unsigned long long limit_ns, unsigned int* outcome, cudaStream_t stream) {
    if (!outcome || limit_ns < 1000ull || limit_ns > 1000000000ull) return W4A8_ERR_INVALID_ARG;
    const unsigned int zero = 0;
    cudaError_t e = cudaMemcpyToSymbolAsync(g_selftest_outcome, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return cuda_status(e);
    unsigned int* dev_outcome = nullptr;
    e = cudaGetSymbolAddress(reinterpret_cast<void**>(&dev_outcome), g_selftest_outcome);
    if (e != cudaSuccess) return cuda_status(e);
    w4a8::selftest_wait_kernel<<<1, 64, 0, stream>>>(limit_ns, dev_outcome);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_status(e);
    e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_status(e);
    e = cudaMemcpyFromSymbol(outcome, g_selftest_outcome, sizeof(*outcome));
    return cuda_status(e);
}

w4a8_status w4a8_last_device_error(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return W4A8_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, w4a8::g_device_status, sizeof(v)) != cudaSuccess) return W4A8_ERR_CUDA;
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(w4a8::g_device_status, &zero, sizeof(zero)) != cudaSuccess) return W4A8_ERR_CUDA;
    if (v & w4a8::kDevErrChecked) return W4A8_ERR_CHECK;  // the cause of any timeout that follows
    if (v & w4a8::kDevErrTimeout) return W4A8_ERR_DEVICE_TIMEOUT;
    return v ? W4A8_ERR_RANGE : W4A8_OK;
}

const char* w4a8_last_cuda_error_string(void) { return cudaGetErrorString(t_last_cuda_error); }

const char* w4a8_status_string(w4a8_status s) {
    switch (s) {
        case W4A8_OK: return "W4A8_OK";
        case W4A8_ERR_INVALID_ARG: return "W4A8_ERR_INVALID_ARG";
        case W4A8_ERR_UNSUPPORTED: return "W4A8_ERR_UNSUPPORTED";
        case W4A8_ERR_WORKSPACE: return "W4A8_ERR_WORKSPACE";
        case W4A8_ERR_CUDA: return "W4A8_ERR_CUDA";
        case W4A8_ERR_DEVICE_TIMEOUT: return "W4A8_ERR_DEVICE_TIMEOUT";
        case W4A8_ERR_MISALIGNED: return "W4A8_ERR_MISALIGNED";
        case W4A8_ERR_RANGE: return "W4A8_ERR_RANGE";
        case W4A8_ERR_CHECK: return "W4A8_ERR_CHECK";
    }
    return "W4A8_UNKNOWN_STATUS";
}

}  // extern "C"
