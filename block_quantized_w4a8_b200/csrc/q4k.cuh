// Q4_K weights with FP32 activations: the GEMV y = x W^T and the input gradient
// dX = dY W of a frozen layer (C-Kernel-Engine gemm_kernels_q4k.c, "GEMV: y = W @ x" and
// "Backward Pass: Gradient w.r.t. Input"). Both stream the packed weights once and
// dequantise in registers: w = d*sc*q - dmin*m per 32-element sub-block, computed as one
// fused multiply-add fma(d*sc, q, -dmin*m) (d*sc*q is exact in f32, so this is the
// page's d1*q - m1 rounded once).
//
// Layout (per row: K/256 super-blocks of 144 bytes): d (fp16), dmin (fp16), 12 bytes of
// packed 6-bit scales and mins, 128 code bytes. Code byte 32i + l holds element 64i + l
// (low nibble, sub-block 2i) and element 64i + 32 + l (high nibble, sub-block 2i + 1).
//
// Work split shared by both kernels: a warp takes four rows of one super-block per step;
// lane l reads the 16-byte code chunk c = l % 8 of row l / 8 (coalesced: a warp's
// chunks are four contiguous 128-byte runs) and the row's 16-byte header (one broadcast
// load per 8 lanes). Chunk c covers code bytes 16c..16c+15: elements 64i + l0 + t (low
// nibbles, sub-block 2i) and 64i + 32 + l0 + t (high nibbles, sub-block 2i + 1) for
// t < 16, with i = c / 2 and l0 = 16 (c % 2).
#pragma once

#include <cuda.h>  // CUtensorMap (the type only; maps are encoded by the host code)

#include "device_common.cuh"

namespace w4a8 {
namespace q4k {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kBlockBytes = 144;

// Sub-block scale and min (6 bits each) of sub-block j from the header words s03 (scale
// bytes 0-3), s47 (4-7), s811 (8-11): the llama.cpp Q4_K packing.
__device__ __forceinline__ void scale_min(int j, uint32_t s03, uint32_t s47, uint32_t s811, int& sc, int& m) {
    if (j < 4) {
        sc = int((s03 >> (8 * j)) & 63u);
        m = int((s47 >> (8 * j)) & 63u);
    } else {
        const int jj = 8 * (j - 4);
        const uint32_t lo = (s811 >> jj) & 0xFFu;
        sc = int((lo & 15u) | (((s03 >> (jj + 6)) & 3u) << 4));
        m = int((lo >> 4) | (((s47 >> (jj + 6)) & 3u) << 4));
    }
}

// Code (0..15) as a float: 2^23 + q from the bit pattern, minus 2^23 (exact).
__device__ __forceinline__ float code_f(uint32_t word, int shift) {
    return __int_as_float(int(((word >> shift) & 15u) | 0x4B000000u)) - 8388608.0f;
}

// The two sub-blocks of a chunk: (d*sc, dmin*m) for its low and its high nibbles.
struct ChunkScales {
    float d_lo, m_lo, d_hi, m_hi;
};
__device__ __forceinline__ ChunkScales chunk_scales(const uint4& h, int c) {
    const float d = __half2float(__ushort_as_half(uint16_t(h.x & 0xFFFFu)));
    const float dmin = __half2float(__ushort_as_half(uint16_t(h.x >> 16)));
    const int j0 = 2 * (c >> 1);
    int sc0, m0, sc1, m1;
    scale_min(j0, h.y, h.z, h.w, sc0, m0);
    scale_min(j0 + 1, h.y, h.z, h.w, sc1, m1);
    return ChunkScales{__fmul_rn(d, float(sc0)), __fmul_rn(dmin, float(m0)), __fmul_rn(d, float(sc1)),
                       __fmul_rn(dmin, float(m1))};
}

// ------------------------------------------------------------------ forward
// y[m][n] = sum_k w[n][k] x[m][k] for MT tokens (x: MT x K f32, row-major). CTA b owns
// rows 16b..16b+15 (four row groups of four); warp w takes super-blocks w, w + 8, ...
// For each of them the warp reads its lanes' slice of x once into registers (the same
// 32 elements serve all four row groups) and issues the loads of the four groups' code
// chunks together, so x costs the L1 one read per CTA rather than one per row group.
// The 8 lanes of a row add their partial sums by shuffles, the 8 warps' sums are added
// in warp order through shared memory.
template <int MT>
__global__ void __launch_bounds__(kThreads) gemv_kernel(int M, int N, int K, const float* __restrict__ x,
                                                      const uint8_t* __restrict__ W, float* __restrict__ y) {
    constexpr int RG = 4;  // row groups of four rows per CTA
    __shared__ float red[kWarps][4 * RG][MT];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rr = lane >> 3, c = lane & 7;
    const int nb = K >> 8;
    const int n0 = blockIdx.x * 4 * RG;
    const int e0 = 64 * (c >> 1) + 16 * (c & 1);  // first element of the chunk's low nibbles
    // Three levels of f32 sums keep every output's rounding chain short at any K: a
    // super-block's 32 products (sb_acc), 16 super-blocks of a warp (mid), the rest (acc).
    float acc[RG][MT], mid[RG][MT];
#pragma unroll
    for (int g = 0; g < RG; ++g)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[g][m] = mid[g][m] = 0.0f;
    int step = 0;
    for (int sb = warp; sb < nb; sb += kWarps, ++step) {
        float xs[MT][32];  // x[m][sb*256 + e0 + t] (t < 16) and x[m][sb*256 + e0 + 32 + t]
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const float* xp = x + int64_t(m < M ? m : 0) * K + sb * 256 + e0;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const float4 a = __ldg(reinterpret_cast<const float4*>(xp) + v);
                const float4 b = __ldg(reinterpret_cast<const float4*>(xp + 32) + v);
                xs[m][4 * v] = a.x; xs[m][4 * v + 1] = a.y; xs[m][4 * v + 2] = a.z; xs[m][4 * v + 3] = a.w;
                xs[m][16 + 4 * v] = b.x; xs[m][16 + 4 * v + 1] = b.y;
                xs[m][16 + 4 * v + 2] = b.z; xs[m][16 + 4 * v + 3] = b.w;
            }
        }
        uint4 h[RG], q[RG];
#pragma unroll
        for (int g = 0; g < RG; ++g) {
            const int n = n0 + 4 * g + rr;
            h[g] = make_uint4(0u, 0u, 0u, 0u);
            q[g] = h[g];
            if (n < N) {
                const uint8_t* blk = W + (int64_t(n) * nb + sb) * kBlockBytes;
                h[g] = __ldcs(reinterpret_cast<const uint4*>(blk));
                q[g] = __ldcs(reinterpret_cast<const uint4*>(blk + 16 + 16 * c));
            }
        }
#pragma unroll
        for (int g = 0; g < RG; ++g) {
            const ChunkScales cs = chunk_scales(h[g], c);
            const uint32_t qw[4] = {q[g].x, q[g].y, q[g].z, q[g].w};
            float sb_acc[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) sb_acc[m] = 0.0f;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const float wl = fmaf(cs.d_lo, code_f(qw[v], 8 * b), -cs.m_lo);
                    const float wh = fmaf(cs.d_hi, code_f(qw[v], 8 * b + 4), -cs.m_hi);
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        sb_acc[m] = fmaf(wl, xs[m][4 * v + b], sb_acc[m]);
                        sb_acc[m] = fmaf(wh, xs[m][16 + 4 * v + b], sb_acc[m]);
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) mid[g][m] += sb_acc[m];
        }
        if ((step & 15) == 15) {
#pragma unroll
            for (int g = 0; g < RG; ++g)
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    acc[g][m] += mid[g][m];
                    mid[g][m] = 0.0f;
                }
        }
    }
#pragma unroll
    for (int g = 0; g < RG; ++g)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[g][m] += mid[g][m];
#pragma unroll
    for (int g = 0; g < RG; ++g)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            float v = acc[g][m];
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            v += __shfl_xor_sync(0xffffffffu, v, 2);
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            if (c == 0) red[warp][4 * g + rr][m] = v;
        }
    __syncthreads();
    for (int i = threadIdx.x; i < 4 * RG * MT; i += kThreads) {
        const int r2 = i / MT, m = i % MT;
        const int n2 = n0 + r2;
        if (n2 < N && m < M) {
            float v = 0.0f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) v += red[w][r2][m];
            y[int64_t(m) * N + n2] = v;
        }
    }
}

// ------------------------------------------------------------------ forward, streamed
// y[m][n] = sum_k w[n][k] x[m][k] for MT tokens, one CTA per SM (grid = min(N, SMs)),
// CTA c owning a contiguous range of rc rows. The rows' super-blocks stream through a
// ring of NST shared-memory slots, one slot = 16 rows x KC super-blocks (KC = min(K/256,
// 16)), each row's piece one bulk copy; a copy warp keeps the ring full from the start,
// before the grid dependency (the weights are not written by a kernel that triggers this
// launch early). x is staged once in shared memory after the grid dependency, each
// 32-float segment's 16-byte chunks rotated by the segment index so that the eight
// sub-blocks a quarter-warp reads at once fall on distinct banks.
// Compute warp w takes row 16 g + w of row group g; lane l works on sub-block j = l % 8
// (elements 32 j .. 32 j + 31: the low nibbles of code bytes 32 (j/2) .. + 31 for even j,
// the high nibbles for odd j) of super-block 4 s + l / 8 of the slot, so the 6-bit scale
// decode happens once per 32 weights. Each code nibble becomes the float 2^23 + q by one
// byte permute; w = fma(d*sc, q, -dmin*m) (the page's d1*q - m1, rounded once) and the dot
// run as packed f32x2 operations. Sums: a super-block's 32 products per lane, then the
// row's super-blocks, then the 32 lanes by shuffles (a few dozen roundings in any chain).
constexpr int kStreamWarps = 16;                     // compute warps
constexpr int kStreamThreads = (kStreamWarps + 1) * 32;  // + the copy warp
constexpr int kStreamMaxStages = 4;

struct StreamPlan {
    bool ok;
    bool two_per_sm;  // two CTAs (consecutive calls) may share an SM: the next call's
                      // weight copies overlap this call's work
    int kc, nst;
    size_t smem;
};
// Slot size, ring depth and shared memory of the streamed forward (x of MT tokens
// staged): a two-slot ring within half of the SM's shared memory when it fits, else the
// deepest ring (up to four slots) within one CTA's limit.
inline StreamPlan stream_plan(int MT, int K, size_t smem_limit, size_t sm_smem) {
    StreamPlan p{false, false, 0, 0, 0};
    const int nb = K >> 8;
    p.kc = nb < 16 ? nb : 16;
    const size_t slot = size_t(16) * p.kc * kBlockBytes;
    const size_t xbytes = size_t(MT) * K * 4;
    const size_t ctrl = 128, reserved = 1024;  // per-CTA shared memory the runtime keeps
    const size_t half = sm_smem / 2 - reserved;
    if (xbytes + ctrl + 2 * slot <= half) {
        p.two_per_sm = true;
        p.nst = 2;
    } else {
        if (xbytes + ctrl + 2 * slot > smem_limit) return p;
        const size_t nst = (smem_limit - xbytes - ctrl) / slot;
        p.nst = int(nst < size_t(kStreamMaxStages) ? nst : size_t(kStreamMaxStages));
    }
    p.smem = size_t(p.nst) * slot + xbytes + ctrl;
    p.ok = true;
    return p;
}

// The 6-bit scale and min of sub-block j (0..7) of a super-block header, without a branch.
__device__ __forceinline__ void scale_min_sel(int j, uint32_t s03, uint32_t s47, uint32_t s811, int& sc, int& m) {
    const int sh = 8 * (j & 3);
    const uint32_t b = (s811 >> sh) & 0xFFu;
    const uint32_t sc_hi = (b & 15u) | (((s03 >> (sh + 6)) & 3u) << 4);
    const uint32_t m_hi = (b >> 4) | (((s47 >> (sh + 6)) & 3u) << 4);
    sc = int(j < 4 ? ((s03 >> sh) & 63u) : sc_hi);
    m = int(j < 4 ? ((s47 >> sh) & 63u) : m_hi);
}

// acc += (fma(d2, q2 - 2^23, -m2)) * x2 lane-wise: f2 holds the floats 2^23 + q (exact), the
// subtraction is exact, the dequantised weight rounds once, the product-sum once.
__device__ __forceinline__ void q4k_fma2(unsigned long long& acc, uint32_t f0, uint32_t f1, float x0, float x1,
                                         unsigned long long d2, unsigned long long nm2) {
    asm("{\n\t.reg .b64 ff, qq, ww, xx, cc;\n\t"
        "mov.b64 ff, {%1, %2};\n\t"
        "mov.b64 cc, {%7, %7};\n\t"
        "add.rn.f32x2 qq, ff, cc;\n\t"
        "fma.rn.f32x2 ww, qq, %5, %6;\n\t"
        "mov.b64 xx, {%3, %4};\n\t"
        "fma.rn.f32x2 %0, ww, xx, %0;\n\t}\n"
        : "+l"(acc)
        : "r"(f0), "r"(f1), "f"(x0), "f"(x1), "l"(d2), "l"(nm2), "f"(-8388608.0f));
}

template <int MT, int MINB>
__global__ void __launch_bounds__(kStreamThreads, MINB)
    fwd_stream_kernel(int M, int N, int K, const float* __restrict__ x, const uint8_t* __restrict__ W,
                      float* __restrict__ y, int KC, int NST) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nb = K >> 8;
    const int q = N / int(gridDim.x), rem = N - q * int(gridDim.x);
    const int c = int(blockIdx.x);
    const int n0 = c * q + (c < rem ? c : rem);
    const int rc = q + (c < rem ? 1 : 0);
    const int RG = (rc + 15) >> 4, NC = (nb + KC - 1) / KC, S = RG * NC;
    const int slot_bytes = 16 * KC * kBlockBytes;
    const uint32_t ring = smem_addr(smem);
    float* xs = reinterpret_cast<float*>(smem + size_t(NST) * slot_bytes);
    unsigned long long* full = reinterpret_cast<unsigned long long*>(smem + size_t(NST) * slot_bytes +
                                                                       size_t(MT) * K * 4);
    unsigned long long* empty = full + kStreamMaxStages;
    volatile uint32_t* abort = reinterpret_cast<volatile uint32_t*>(empty + kStreamMaxStages);
    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(smem_addr(&full[i]), 1);
            mbar_init(smem_addr(&empty[i]), kStreamWarps);
        }
        *abort = 0u;
        mbar_init_fence();
    }
    __syncthreads();
    pdl_launch_dependents();

    if (warp == kStreamWarps) {
        // ------------------------------------------------ copy warp: the weight ring
        if (lane == 0) {
            int issued = 0;
            for (int st = 0; st < S; ++st) {
                const int slot = st % NST;
                if (!bounded_wait(smem_addr(&empty[slot]), ((st / NST) & 1) ^ 1, abort)) break;
                const int rg = st / NC, kc = st - rg * NC;
                const int rows = min(16, rc - rg * 16), kcn = min(KC, nb - kc * KC);
                const uint32_t fb = smem_addr(&full[slot]);
                mbar_arrive_expect_tx(fb, uint32_t(rows * kcn * kBlockBytes));
                for (int i = 0; i < rows; ++i) {
                    const int64_t n = int64_t(n0) + rg * 16 + i;
                    // (checked build: the row lies within the N rows of the weights)
                    if (in_range(n, 1, N))
                        bulk_g2s(ring + uint32_t(slot * slot_bytes + i * KC * kBlockBytes),
                                 W + (n * nb + int64_t(kc) * KC) * kBlockBytes, uint32_t(kcn * kBlockBytes), fb);
                }
                issued = st + 1;
            }
            // let the copies land before the CTA can exit (capped after an abort)
            for (int st = max(0, issued - NST); st < issued; ++st) {
                const uint32_t fb = smem_addr(&full[st % NST]);
                const unsigned long long t0 = global_timer_ns();
                while (!mbar_try_wait(fb, (st / NST) & 1) && global_timer_ns() - t0 < 200000ull) {
                }
            }
        }
        return;
    }

    // ---------------------------------------------------- compute warps
    pdl_wait_primary();  // x is written by the preceding kernel
    for (int i = threadIdx.x; i < MT * (K >> 2); i += kStreamWarps * 32) {
        const int m = i / (K >> 2), f = i - m * (K >> 2);  // float4 f of token m
        const int sgm = f >> 3, v = f & 7;
        const float4 val = (m < M) ? __ldg(reinterpret_cast<const float4*>(x + int64_t(m) * K) + f)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(xs + size_t(m) * K + sgm * 32 + ((v + sgm) & 7) * 4) = val;
    }
    named_barrier(1, kStreamWarps * 32);

    const int j = lane & 7, h = j & 1, quarter = lane >> 3;
    const int code_off = 16 + 32 * (j >> 1);
    unsigned long long racc[MT];
    for (int st = 0; st < S; ++st) {
        const int slot = st % NST;
        const int rg = st / NC, kc = st - rg * NC;
        if (kc == 0)
#pragma unroll
            for (int m = 0; m < MT; ++m) racc[m] = 0ull;
        if (!bounded_wait_warp(smem_addr(&full[slot]), (st / NST) & 1, abort)) break;
        const int row = rg * 16 + warp;
        const int kcn = min(KC, nb - kc * KC);
        if (row < rc) {
            const uint8_t* base = smem + size_t(slot) * slot_bytes + size_t(warp) * KC * kBlockBytes;
            for (int g = 0; g < kcn; g += 4) {
                const int sl = g + quarter;
                if (sl < kcn) {
                    const uint8_t* blk = base + sl * kBlockBytes;
                    const uint4 hd = *reinterpret_cast<const uint4*>(blk);
                    int sc, mn;
                    scale_min_sel(j, hd.y, hd.z, hd.w, sc, mn);
                    const float d1 = __fmul_rn(__half2float(__ushort_as_half(uint16_t(hd.x & 0xFFFFu))), float(sc));
                    const float m1 = __fmul_rn(__half2float(__ushort_as_half(uint16_t(hd.x >> 16))), float(mn));
                    const unsigned long long d2 = pack2(d1, d1), nm2 = pack2(-m1, -m1);
                    const uint4 c0 = *reinterpret_cast<const uint4*>(blk + code_off);
                    const uint4 c1 = *reinterpret_cast<const uint4*>(blk + code_off + 16);
                    const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                    const int sgm = (kc * KC + sl) * 8 + j;  // x segment of this sub-block
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        const float* xseg = xs + size_t(m) * K + sgm * 32;
                        unsigned long long sacc = 0ull;
#pragma unroll
                        for (int v = 0; v < 8; ++v) {
                            const float4 xv = *reinterpret_cast<const float4*>(xseg + ((v + j) & 7) * 4);
                            const uint32_t u = (cw[v] >> (4 * h)) & 0x0F0F0F0Fu;  // codes of elements 4v..4v+3
                            q4k_fma2(sacc, __byte_perm(u, 0x4B000000u, 0x7540u), __byte_perm(u, 0x4B000000u, 0x7541u),
                                     xv.x, xv.y, d2, nm2);
                            q4k_fma2(sacc, __byte_perm(u, 0x4B000000u, 0x7542u), __byte_perm(u, 0x4B000000u, 0x7543u),
                                     xv.z, xv.w, d2, nm2);
                        }
                        float a0, a1, r0, r1;
                        unpack2(sacc, a0, a1);
                        unpack2(racc[m], r0, r1);
                        racc[m] = pack2(r0 + a0, r1 + a1);
                    }
                }
            }
            if (kc == NC - 1) {
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    float a0, a1;
                    unpack2(racc[m], a0, a1);
                    float v = a0 + a1;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                    if (lane == 0 && m < M) y[int64_t(m) * N + n0 + row] = v;
                }
            }
        }
        // the slot's loads were consumed above: hand it back
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&empty[slot]));
    }
}

// ------------------------------------------------------------------ backward, streamed
// dX[m][k] = sum_n w[n][k] dY[m][n] for MT tokens. CTA c takes super-block column c % nb
// (256 elements of k) of row range c / nb (at most kBwdMaxRows rows); the range's
// super-blocks of that column stream through a ring of shared-memory slots of 64 rows, one
// 2-D TMA box per slot (the weights seen as 8-byte elements, [N][nb * 18], box 18 x 64:
// the x offset col * 144 bytes is a multiple of 16; rows past N read as zeros, rows of the
// next range are read and ignored), and the range's dY values are staged once in shared
// memory.
// Compute warp w takes rows 4 w .. 4 w + 3 of each slot; lane l takes row l / 8 of those
// and sub-block j = l % 8, and keeps the 32 sums of its sub-block's elements over the rows
// it visits in registers (one row per lane and slot). At the end
// the four row lanes are added by shuffles, the 16 warps in order through shared memory,
// and the CTA writes its partial sums to part[r][m][k] (or dX directly when one range
// covers all rows); bwd_reduce_kernel adds the ranges in a fixed order, so the result does
// not depend on scheduling.
constexpr int kBwdMaxRows = 512;
constexpr int kBwdSlotRows = 64;
constexpr int kBwdStages = 4;
constexpr size_t bwd_smem_bytes(int MT) {
    return 128 + size_t(kBwdStages) * kBwdSlotRows * kBlockBytes + size_t(kStreamWarps) * MT * 256 * 4 +
           size_t(MT) * kBwdMaxRows * 4 + 128;  // (the first 128: alignment of the TMA ring)
}

template <int MT>
__global__ void __launch_bounds__(kStreamThreads, 1)
    bwd_stream_kernel(int M, int N, int K, const float* __restrict__ dy, const __grid_constant__ CUtensorMap tm_w,
                      float* __restrict__ out, int R) {
    constexpr int NST = kBwdStages, SR = kBwdSlotRows;
    constexpr int slot_bytes = SR * kBlockBytes;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nb = K >> 8;
    const int c = int(blockIdx.x);
    const int col = c % nb, r = c / nb;
    const int q = N / R, rem = N - q * R;
    const int n0 = r * q + (r < rem ? r : rem);
    const int rc = q + (r < rem ? 1 : 0);
    const int RG = (rc + SR - 1) / SR;
    const uint32_t ring = smem_addr(smem);
    float* red = reinterpret_cast<float*>(smem + NST * slot_bytes);      // [16 warps][MT][256]
    float* dys = red + kStreamWarps * MT * 256;                           // [MT][kBwdMaxRows]
    unsigned long long* full = reinterpret_cast<unsigned long long*>(dys + MT * kBwdMaxRows);
    unsigned long long* empty = full + NST;
    volatile uint32_t* abort = reinterpret_cast<volatile uint32_t*>(empty + NST);
    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(smem_addr(&full[i]), 1);
            mbar_init(smem_addr(&empty[i]), kStreamWarps);
        }
        *abort = 0u;
        mbar_init_fence();
    }
    __syncthreads();
    pdl_launch_dependents();

    if (warp == kStreamWarps) {
        // ------------------------------------------------ copy warp
        if (lane == 0) {
            int issued = 0;
            for (int st = 0; st < RG; ++st) {
                const int slot = st % NST;
                if (!bounded_wait(smem_addr(&empty[slot]), ((st / NST) & 1) ^ 1, abort)) break;
                const uint32_t fb = smem_addr(&full[slot]);
                mbar_arrive_expect_tx(fb, uint32_t(slot_bytes));  // the whole box, zero fill included
                tma_load_2d<8>(ring + uint32_t(slot * slot_bytes), &tm_w, col * (kBlockBytes / 8), n0 + st * SR, fb);
                issued = st + 1;
            }
            for (int st = max(0, issued - NST); st < issued; ++st) {
                const uint32_t fb = smem_addr(&full[st % NST]);
                const unsigned long long t0 = global_timer_ns();
                while (!mbar_try_wait(fb, (st / NST) & 1) && global_timer_ns() - t0 < 200000ull) {
                }
            }
        }
        return;
    }

    // ---------------------------------------------------- compute warps
    pdl_wait_primary();  // dY is written by the preceding kernel
    for (int i = threadIdx.x; i < MT * rc; i += kStreamWarps * 32) {
        const int m = i / rc, rr = i - m * rc;
        dys[m * kBwdMaxRows + rr] = (m < M) ? __ldg(dy + int64_t(m) * N + n0 + rr) : 0.0f;
    }
    named_barrier(1, kStreamWarps * 32);
    const int j = lane & 7, h = j & 1, rl = lane >> 3;
    const int code_off = 16 + 32 * (j >> 1);
    float acc[MT][32];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int t = 0; t < 32; ++t) acc[m][t] = 0.0f;
    bool ok = true;
    for (int st = 0; st < RG; ++st) {
        const int slot = st % NST;
        if (!bounded_wait_warp(smem_addr(&full[slot]), (st / NST) & 1, abort)) {
            ok = false;
            break;
        }
        const int rr = 4 * warp + rl;  // row within the slot
        if (rr < min(SR, rc - st * SR)) {
            const uint8_t* blk = smem + size_t(slot) * slot_bytes + size_t(rr) * kBlockBytes;
            const uint4 hd = *reinterpret_cast<const uint4*>(blk);
            int sc, mn;
            scale_min_sel(j, hd.y, hd.z, hd.w, sc, mn);
            const float d1 = __fmul_rn(__half2float(__ushort_as_half(uint16_t(hd.x & 0xFFFFu))), float(sc));
            const float m1 = __fmul_rn(__half2float(__ushort_as_half(uint16_t(hd.x >> 16))), float(mn));
            const uint4 c0 = *reinterpret_cast<const uint4*>(blk + code_off);
            const uint4 c1 = *reinterpret_cast<const uint4*>(blk + code_off + 16);
            const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            float g[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) g[m] = dys[m * kBwdMaxRows + st * SR + rr];
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const uint32_t u = (cw[v] >> (4 * h)) & 0x0F0F0F0Fu;  // codes of elements 4v..4v+3
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const float qf = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540u + b)) - 8388608.0f;
                    const float wv = fmaf(d1, qf, -m1);  // the page's d1*q - m1, rounded once
#pragma unroll
                    for (int m = 0; m < MT; ++m) acc[m][4 * v + b] = fmaf(wv, g[m], acc[m][4 * v + b]);
                }
            }
        }
        // the slot's loads were consumed above: hand it back
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&empty[slot]));
    }
    // the four row lanes of each sub-block, then the 16 warps in order
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            float v = acc[m][t];
            v += __shfl_xor_sync(0xffffffffu, v, 8);
            v += __shfl_xor_sync(0xffffffffu, v, 16);
            acc[m][t] = v;
        }
    if (rl == 0) {
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int t = 0; t < 32; t += 4)
                *reinterpret_cast<float4*>(red + (warp * MT + m) * 256 + 32 * j + t) =
                    make_float4(acc[m][t], acc[m][t + 1], acc[m][t + 2], acc[m][t + 3]);
    }
    named_barrier(1, kStreamWarps * 32);
    if (!ok || *abort) return;
    const bool direct = R == 1;
    for (int i = threadIdx.x; i < MT * 256; i += kStreamWarps * 32) {
        const int m = i >> 8, e = i & 255;
        if (m >= M) continue;
        float v = red[m * 256 + e];
#pragma unroll
        for (int w = 1; w < kStreamWarps; ++w) v += red[(w * MT + m) * 256 + e];
        const int64_t k = int64_t(col) * 256 + e;
        if (direct)
            out[int64_t(m) * K + k] = v;
        else
            out[(int64_t(r) * M + m) * K + k] = v;
    }
}

// dX[i] = sum over row ranges r = 0..R-1 of part[r][i], i < M*K: in order, in groups of 16,
// their sums in groups of 16, and those in order (at most 15 + 15 + R/256 roundings in a
// chain).
__global__ void __launch_bounds__(256) bwd_reduce_kernel(const float* __restrict__ part, int R, int64_t count,
                                                         float* __restrict__ dx) {
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < count; i += int64_t(gridDim.x) * blockDim.x) {
        float v = 0.0f;
        for (int r1 = 0; r1 < R; r1 += 256) {
            float u = 0.0f;
            for (int r0 = r1; r0 < R && r0 < r1 + 256; r0 += 16) {
                float g = part[int64_t(r0) * count + i];
                for (int r = r0 + 1; r < R && r < r0 + 16; ++r) g += part[int64_t(r) * count + i];
                u = (r0 == r1) ? g : u + g;
            }
            v = (r1 == 0) ? u : v + u;
        }
        dx[i] = v;
    }
}

}  // namespace q4k
}  // namespace w4a8
