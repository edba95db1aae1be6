// Small-M path with the weights resident in shared memory: the decode GEMV of tract PR
// #2432 (follow-up "decode regime (m=1)"), where the weight stream is the whole cost.
//
// Each CTA owns a contiguous range of weight rows whose codes and scales (affine: and
// biases) fit in shared memory at once. One thread issues bulk asynchronous copies of them
// (the copy engine, not the load/store path) BEFORE the grid waits on the preceding kernel.
// A CTA takes less than half an SM, so under programmatic dependent launch the CTA of the
// next call in the stream sits beside the CTA of the current call and streams its weights
// while the current call waits for its input, quantises it and contracts it. Everything
// that reads the activation or writes the output comes after griddepcontrol.wait.
//
// Work split inside a CTA: the K blocks of a row are cut into slices of 32 blocks; the
// NSW warps of a row group take slices sw, sw + NSW, ... (XS each; lane l: block l of each
// slice), and the H = warps / NSW row groups take rows h, h + H, h + 2H, ... of the CTA's
// range. A lane keeps the Q8_0 codes, scale and block sum of its XS blocks for all MT
// tokens in registers and walks the rows of its group, so shared memory is read once per
// weight byte. The 32 lanes' partial sums of RW rows x MT tokens are combined by a shuffle
// reduce-scatter; when a row's slices are on several warps (NSW > 1) their partials are
// added in slice order after a block barrier.
//
// Block dot on dp4a with the codes unsigned and x signed: the low nibbles (w & 0x0F0F0F0F)
// pair with the first 16 elements of the block (Q4_0) or the even elements of each word
// (affine); the high nibbles are taken in place (w & 0xF0F0F0F0, i.e. 16 * code) and their
// dot is divided by 16 exactly. Q4_0 starts the low dot at -8 * sum(q_x), so
// D = sum((q - 8) * q_x) comes out exact.
#pragma once

#include "device_common.cuh"

namespace w4a8 {
namespace gv {

// Warps per CTA: 16 for one token (registers are light, and more warps hide the
// latencies of the short post-wait critical path), 8 for 2..8 tokens.
__host__ __device__ constexpr int warps_for(int MT) { return MT == 1 ? 16 : 8; }
constexpr int kVals = 8;                     // at most RW * MT values per warp and pass
constexpr int kHeaderBytes = 2048;           // barriers, flags, pass partials

// Rows per warp and pass: the pass body (RW rows x XS blocks, unrolled) is kept to eight
// block dots per token so that the code executed once per call stays small.
__host__ __device__ constexpr int rows_per_pass(int MT, int XS) { return (8 / (XS * MT)) > 0 ? 8 / (XS * MT) : 1; }

// Shared-memory bytes of the quantised activation (x codes [MT][K] as two 16-byte halves
// per block, d_x [MT][B] f32, sum(q_x) [MT][B] s32) when the kernel quantises x itself.
__host__ __device__ constexpr size_t xregion_bytes(int MT, int K, bool quantise) {
    return quantise ? ((size_t(MT) * K + size_t(MT) * (K / 32) * 8 + 127) & ~size_t(127)) : 0;
}
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// Bulk copy global -> shared (this CTA only) with an L2 eviction-priority hint: the weights
// are read once per call, so they should not push the activations and outputs out of L2.
__device__ __forceinline__ void bulk_g2s_hint(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                              uint64_t policy) {
    if (!checked((dst & 15u) == 0 && (reinterpret_cast<uintptr_t>(src) & 15u) == 0 && (bytes & 15u) == 0)) return;
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
            "r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

// dp4a with the first operand's bytes unsigned and the second's signed.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Shared-memory loads at a 32-bit shared address, written as ordinary loads so that the
// compiler keeps them after the barrier waits that guard the data.
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    extern __shared__ __align__(128) uint8_t smem[];
    return *reinterpret_cast<const uint4*>(smem + (addr - smem_addr(smem)));
}
__device__ __forceinline__ uint32_t lds16(uint32_t addr) {
    extern __shared__ __align__(128) uint8_t smem[];
    return *reinterpret_cast<const unsigned short*>(smem + (addr - smem_addr(smem)));
}

// Reduce-scatter of V values (V = 1, 2, 4 or 8) over the warp: afterwards every lane l
// holds the sum over the 32 lanes of value l / (32 / V).
template <int V>
__device__ __forceinline__ float reduce_scatter(float (&v)[V], int lane) {
#pragma unroll
    for (int off = 16, n = V; off >= 1; off >>= 1) {
        if (n > 1) {
            const int half = n >> 1;
            const bool up = lane & off;
#pragma unroll
            for (int k = 0; k < half; ++k) {
                const float send = up ? v[k] : v[k + half];
                const float keep = up ? v[k + half] : v[k];
                v[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
            }
            n = half;
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
        }
    }
    return v[0];
}

// Q8_0 quantisation of the M x K activation into shared memory (codes of token m, block b:
// bytes 0-15 at m*K + 16b, bytes 16-31 at m*K + K/2 + 16b; d_x at dxs[m*B + b], sum(q_x) at
// sxs[m*B + b]). THREADS threads, PIECES = 32 / EPT adjacent lanes per block. The arithmetic
// is the pages' Q8_0 step: d = amax / 127 (f32 division), id = 1 / d, q = round half away
// from zero of fl(x * id). The rounding is trunc(|t| + 0.5) with the sign of t, exact here:
// |t| < 2^23, and |t| + 0.5 lies in |t|'s binade or the next one, so the addition rounds
// only where no representable |t| can reach the wrong side of k + 0.5. No clamp is needed:
// |t| <= amax * id <= 127 * (1 + 3 * 2^-24) < 127.5.
template <int THREADS, int EPT>
__device__ __forceinline__ void quantise_x_smem(const void* __restrict__ x, int xbf16, int M, int K, int8_t* xq,
                                                float* dxs, int32_t* sxs) {
    constexpr int PIECES = 32 / EPT;
    const int B = K >> 5;
    for (int m = 0; m < M; ++m) {
        for (int base = 0; base < PIECES * B; base += THREADS) {
            const int p = base + int(threadIdx.x);  // piece p % PIECES of block p / PIECES of token m
            const bool valid = p < PIECES * B;
            const int b = p / PIECES, pc = p % PIECES;
            float v[EPT];
#pragma unroll
            for (int i = 0; i < EPT; ++i) v[i] = 0.0f;
            if (valid) {
                const int64_t e0 = int64_t(m) * K + b * 32 + pc * EPT;
#pragma unroll
                for (int qq = 0; qq < EPT / 4; ++qq) {
                    float t[4];
                    if (xbf16)
                        load4<true>(x, e0 + 4 * qq, t);
                    else
                        load4<false>(x, e0 + 4 * qq, t);
                    v[4 * qq] = t[0]; v[4 * qq + 1] = t[1]; v[4 * qq + 2] = t[2]; v[4 * qq + 3] = t[3];
                }
            }
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < EPT; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
            for (int o = 1; o < PIECES; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            const float d = __fdiv_rn(amax, 127.0f);
            const float id = (d != 0.0f) ? __frcp_rn(d) : 0.0f;
            int sum = 0;
            uint32_t w[EPT / 4];
#pragma unroll
            for (int qq = 0; qq < EPT / 4; ++qq) {
                int q[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float t = __fmul_rn(v[4 * qq + i], id);
                    q[i] = __float2int_rz(copysignf(__fadd_rn(fabsf(t), 0.5f), t));
                }
                w[qq] = __byte_perm(__byte_perm(uint32_t(q[0]), uint32_t(q[1]), 0x0040),
                                    __byte_perm(uint32_t(q[2]), uint32_t(q[3]), 0x0040), 0x5410);
                sum = __dp4a(int(w[qq]), 0x01010101, sum);
            }
#pragma unroll
            for (int o = 1; o < PIECES; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            if (valid) {
                // elements 0-15 of the block go to half 0, 16-31 to half 1
                int8_t* dst = xq + m * K + ((pc * EPT) >> 4) * (K >> 1) + b * 16 + ((pc * EPT) & 15);
                if constexpr (EPT == 16)
                    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
                else
                    *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
                if (pc == 0) {
                    dxs[m * B + b] = d;
                    sxs[m * B + b] = sum;
                }
            }
        }
    }
}

// This lane's activation for XS blocks (slices sw, sw + NSW, ... of 32 blocks; lane = block
// within the slice) and MT tokens: codes as the dp4a partners of the low nibbles (xa) and
// of the high nibbles (xb), the dot's starting value (Q4_0: -8 * sum(q_x)), d_x and sum(q_x).
template <int MT, int FMT, bool QX, int XS>
struct XRegs {
    uint32_t a[XS][MT][4], b[XS][MT][4];
    int init[XS][MT];
    float d[XS][MT], s[XS][MT];
    bool valid[XS];
    __device__ __forceinline__ void load(int M, int K, int sw, int lnsw, int lane, const int8_t* xq_smem,
                                         const float* dxs, const int32_t* sxs, const int8_t* __restrict__ qx,
                                         const float* __restrict__ dx, const int32_t* __restrict__ sx) {
        const int B = K >> 5, NS = (B + 31) >> 5;
#pragma unroll
        for (int xi = 0; xi < XS; ++xi) {
            const int slice = sw + (xi << lnsw);
            const int bb = slice * 32 + lane;
            valid[xi] = slice < NS && bb < B;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
                float dv = 0.0f;
                int S = 0;
                if (valid[xi] && m < M) {
                    if (QX) {
                        lo = *reinterpret_cast<const uint4*>(xq_smem + m * K + bb * 16);
                        hi = *reinterpret_cast<const uint4*>(xq_smem + m * K + (K >> 1) + bb * 16);
                        dv = dxs[m * B + bb];
                        S = sxs[m * B + bb];
                    } else {
                        const uint4* p = reinterpret_cast<const uint4*>(qx + int64_t(m) * K + int64_t(bb) * 32);
                        lo = p[0];
                        hi = p[1];
                        dv = dx[int64_t(m) * B + bb];
                        S = sx[int64_t(m) * B + bb];
                    }
                }
                if (FMT == 0) {  // word k: elements 4k..4k+3 (low nibbles) and 16+4k.. (high nibbles)
                    a[xi][m][0] = lo.x; a[xi][m][1] = lo.y; a[xi][m][2] = lo.z; a[xi][m][3] = lo.w;
                    b[xi][m][0] = hi.x; b[xi][m][1] = hi.y; b[xi][m][2] = hi.z; b[xi][m][3] = hi.w;
                    init[xi][m] = -8 * S;
                } else {  // word k: elements 8k, 8k+2, 8k+4, 8k+6 (low nibbles) and the odd ones (high)
                    const uint32_t e[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        a[xi][m][k] = __byte_perm(e[2 * k], e[2 * k + 1], 0x6420);
                        b[xi][m][k] = __byte_perm(e[2 * k], e[2 * k + 1], 0x7531);
                    }
                    init[xi][m] = 0;
                }
                d[xi][m] = dv;
                s[xi][m] = float(S);
            }
        }
    }
    // acc[m] += this block's term for weight codes `wv` (16 bytes) with scale ws (affine:
    // and bias wb), token m.
    __device__ __forceinline__ void dot(int xi, uint4 wv, float ws, float wb, float (&acc)[MT]) const {
        const uint32_t w[4] = {wv.x, wv.y, wv.z, wv.w};
        uint32_t lo[4], hi[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            lo[k] = w[k] & 0x0F0F0F0Fu;
            hi[k] = w[k] & 0xF0F0F0F0u;
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            int dl = init[xi][m], dh = 0;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                dl = dp4a_us(lo[k], a[xi][m][k], dl);
                dh = dp4a_us(hi[k], b[xi][m][k], dh);
            }
            const int D = dl + (dh >> 4);  // dh is 16 x an integer: exact
            if (FMT == 0)
                acc[m] = fmaf(__fmul_rn(ws, d[xi][m]), float(D), acc[m]);
            else
                acc[m] = fmaf(d[xi][m], fmaf(ws, float(D), __fmul_rn(wb, s[xi][m])), acc[m]);
        }
    }
};

// ------------------------------------------------------------------ kernel
// Shared memory: [0, 8) barrier, [8] abort flag, [256, 1280) pass partials [2][warps][8]
// f32, from kHeaderBytes the quantised activation (QX), then codes [RC][K/2], scales
// [RC][E] and (affine) biases [RC][E] -- all 16-byte aligned since E is a multiple of 8.
// MT: tokens per launch (1, 2, 4, 8); FMT 0 Q4_0, 1 affine 4-bit; QX: quantise x in the
// kernel (f32 or bf16 per `xbf16`) instead of reading a prepared row-major Q8_0 activation;
// XS: blocks per lane and row; lnsw: log2 of the slice warps per row group. Launch:
// gridDim.x <= N CTAs (an even split of the rows), WARPS * 32 threads.
__host__ __device__ constexpr size_t resident_weight_bytes(int rows, int K, int E, bool affine) {
    return size_t(rows) * (K / 2) + size_t(rows) * E * 2 * (affine ? 2 : 1);
}

template <int MT, int FMT, bool QX, int XS, int WARPS = warps_for(MT)>
__global__ void __launch_bounds__(WARPS * 32, 2)
    gemv_resident_kernel(int M, int N, int K, int group, const void* __restrict__ x, int xbf16,
                    const int8_t* __restrict__ qx, const float* __restrict__ dx, const int32_t* __restrict__ sx,
                    const uint8_t* __restrict__ wq, const uint16_t* __restrict__ wscale,
                    const uint16_t* __restrict__ wbias, void* __restrict__ y, Epilogue epi, int lnsw) {
    constexpr int RW = rows_per_pass(MT, XS);
    constexpr int V = RW * MT, LPV = 32 / V;
    constexpr int kWarps = WARPS, kThreads = WARPS * 32;
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t bar = smem_addr(smem);
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + 8);
    float* part = reinterpret_cast<float*>(smem + 256);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = K >> 5;
    const int bsh = (FMT == 1) ? group_shift(group) : 0;
    const int E = B >> bsh;  // scales per row
    const int NSW = 1 << lnsw, lH = (kWarps == 16 ? 4 : 3) - lnsw, H = 1 << lH;
    const int q = N / int(gridDim.x), rem = N - q * int(gridDim.x);
    const int c = int(blockIdx.x);
    const int64_t n0 = int64_t(c) * q + (c < rem ? c : rem);
    const int RC = q + (c < rem ? 1 : 0);
    const int codes_row = K >> 1;
    const uint32_t wbase = smem_addr(smem) + kHeaderBytes + uint32_t(xregion_bytes(MT, K, QX));
    const uint32_t sbase = wbase + uint32_t(RC * codes_row);
    const uint32_t bbase = sbase + uint32_t(RC * E * 2);

    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        *abort_flag = 0u;
        mbar_init_fence();
        const uint64_t pol = l2_evict_first_policy();
        mbar_arrive_expect_tx(bar, uint32_t(resident_weight_bytes(RC, K, E, FMT == 1)));
        // (checked build: this CTA's rows lie within the N rows of the weights)
        if (in_range(n0, RC, N)) bulk_g2s_hint(wbase, wq + n0 * codes_row, uint32_t(RC * codes_row), bar, pol);
        bulk_g2s_hint(sbase, reinterpret_cast<const uint8_t*>(wscale) + n0 * E * 2, uint32_t(RC * E * 2), bar, pol);
        if (FMT == 1)
            bulk_g2s_hint(bbase, reinterpret_cast<const uint8_t*>(wbias) + n0 * E * 2, uint32_t(RC * E * 2), bar, pol);
    }
    __syncthreads();
    const int sw = warp & (NSW - 1), h = warp >> lnsw;

    // x (or its prepared quantisation) may be written by the preceding kernel.
    pdl_wait_primary();
    // Probe the weights' barrier now (usually complete: the copies were issued long before
    // the grid could start waiting), so that its latency overlaps the activation's loads.
    bool ok = mbar_try_wait_nohint(bar, 0);
    int8_t* xq_smem = reinterpret_cast<int8_t*>(smem + kHeaderBytes);
    float* dxs = reinterpret_cast<float*>(smem + kHeaderBytes + size_t(MT) * K);
    int32_t* sxs = reinterpret_cast<int32_t*>(dxs + MT * B);
    if (QX) {
        quantise_x_smem<kThreads, (kThreads >= 512 ? 8 : 16)>(x, xbf16, M, K, xq_smem, dxs, sxs);
        __syncthreads();
    }
    XRegs<MT, FMT, QX, XS> xr;
    xr.load(M, K, sw, lnsw, lane, xq_smem, dxs, sxs, qx, dx, sx);
    // A dependent launch may start its own weight prefetch now (it still waits for this grid
    // to complete before it reads anything this grid writes). Not earlier: its weight stream
    // would compete with this call's activation loads, the critical path (measured: 3.60 ->
    // 3.43 us per back-to-back decode call at 4096 x 4096).
    pdl_launch_dependents();

    ok = __all_sync(0xffffffffu, ok);
    if (!ok) ok = bounded_wait_warp(bar, 0, abort_flag);

    // rows of this warp's group: r = h + H*t
    const int Tmax = (RC + H - 1) >> lH;
    int pass = 0;
#pragma unroll 1
    for (int t0 = 0; t0 < Tmax; t0 += RW, ++pass) {
        float acc[RW][MT];
#pragma unroll
        for (int i = 0; i < RW; ++i)
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[i][m] = 0.0f;
#pragma unroll
        for (int i = 0; i < RW; ++i) {
            const int r = h + ((t0 + i) << lH);
            if (ok && r < RC) {
#pragma unroll
                for (int xi = 0; xi < XS; ++xi) {
                    if (!xr.valid[xi]) continue;
                    const int b = (sw + (xi << lnsw)) * 32 + lane;
                    const uint4 wv = lds128(wbase + uint32_t(r * codes_row + b * 16));
                    float ws, wb = 0.0f;
                    if (FMT == 0) {
                        ws = __half2float(__ushort_as_half((unsigned short)lds16(sbase + uint32_t((r * E + b) * 2))));
                    } else {
                        const int g = b >> bsh;
                        ws = __bfloat162float(__ushort_as_bfloat16((unsigned short)lds16(sbase + uint32_t((r * E + g) * 2))));
                        wb = __bfloat162float(__ushort_as_bfloat16((unsigned short)lds16(bbase + uint32_t((r * E + g) * 2))));
                    }
                    xr.dot(xi, wv, ws, wb, acc[i]);
                }
            }
        }
        float v[V];
#pragma unroll
        for (int i = 0; i < RW; ++i)
#pragma unroll
            for (int m = 0; m < MT; ++m) v[i * MT + m] = acc[i][m];
        const float red = reduce_scatter<V>(v, lane);
        if (lnsw == 0) {  // this warp holds whole rows: store directly, no barrier
            const int vv = lane / LPV, i = vv / MT, m = vv - i * MT;
            const int r = h + H * (t0 + i);
            if ((lane % LPV) == 0 && r < RC && m < M) epi_store(y, int64_t(m) * N + n0 + r, int(n0 + r), red, epi);
            continue;
        }
        const int buf = pass & 1;
        if ((lane % LPV) == 0) part[(buf * kWarps + warp) * kVals + lane / LPV] = red;
        __syncthreads();
        const int tid = threadIdx.x;
        if (tid < H * V) {
            const int hh = tid / V, vv = tid - hh * V;
            const int i = vv / MT, m = vv - i * MT;
            const int r = hh + H * (t0 + i);
            if (r < RC && m < M) {
                float sum = 0.0f;
                for (int qq = 0; qq < NSW; ++qq) sum += part[(buf * kWarps + (hh << lnsw) + qq) * kVals + vv];
                epi_store(y, int64_t(m) * N + n0 + r, int(n0 + r), sum, epi);
            }
        }
    }
    // A warp whose wait ran out must not let the CTA exit while the copy may still land.
    if (!ok) drain_wait_warp(bar, 0, 200000ull);
}

}  // namespace gv
}  // namespace w4a8
