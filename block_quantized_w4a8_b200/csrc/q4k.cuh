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

// ------------------------------------------------------------------ backward
// dX[m][k] = sum_n w[n][k] dY[m][n] for MT tokens. CTA (sb, r) owns super-block column sb
// and the rows [r*rows, (r+1)*rows); warp w takes row groups w, w + 8, ... of four rows,
// four groups per step with all their loads issued first. Each lane accumulates its
// chunk's 32 elements over the rows it visits; the four lanes that hold the same chunk
// (one per row of a group) and then the 8 warps are added in a fixed order, and the CTA
// writes its partial sums to part[r][m][k] (or dX directly when there is one row range),
// so the result does not depend on scheduling. A row range holds at most 2048 rows, so a
// lane's chain of products is at most 64 long.
template <int MT>
__global__ void __launch_bounds__(kThreads) bwd_kernel(int M, int N, int K, int rows, const float* __restrict__ dy,
                                                     const uint8_t* __restrict__ W, float* __restrict__ out) {
    constexpr int U = 4;  // row groups per step
    __shared__ float red[kWarps][MT][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sb = blockIdx.x, r = blockIdx.y;
    const int c = lane & 7;
    const int nb = K >> 8;
    const int n_begin = r * rows, n_end = min(N, n_begin + rows);
    const int e0 = 64 * (c >> 1) + 16 * (c & 1);
    float acc[MT][32];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int t = 0; t < 32; ++t) acc[m][t] = 0.0f;
    for (int g0 = n_begin + warp * 4; g0 < n_end; g0 += U * kWarps * 4) {
        uint4 h[U], q[U];
        float dyv[U][MT];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int n = g0 + u * kWarps * 4 + (lane >> 3);
            const bool row_ok = n < n_end;
            h[u] = make_uint4(0u, 0u, 0u, 0u);
            q[u] = h[u];
            if (row_ok) {
                const uint8_t* blk = W + (int64_t(n) * nb + sb) * kBlockBytes;
                h[u] = __ldcs(reinterpret_cast<const uint4*>(blk));
                q[u] = __ldcs(reinterpret_cast<const uint4*>(blk + 16 + 16 * c));
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) dyv[u][m] = (row_ok && m < M) ? __ldg(dy + int64_t(m) * N + n) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const ChunkScales cs = chunk_scales(h[u], c);
            const uint32_t qw[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
            for (int v = 0; v < 4; ++v) {
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const float wl = fmaf(cs.d_lo, code_f(qw[v], 8 * b), -cs.m_lo);
                    const float wh = fmaf(cs.d_hi, code_f(qw[v], 8 * b + 4), -cs.m_hi);
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        acc[m][4 * v + b] = fmaf(wl, dyv[u][m], acc[m][4 * v + b]);
                        acc[m][16 + 4 * v + b] = fmaf(wh, dyv[u][m], acc[m][16 + 4 * v + b]);
                    }
                }
            }
        }
    }
    // lanes c, c + 8, c + 16, c + 24 hold the same elements for different rows
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            float v = acc[m][t];
            v += __shfl_xor_sync(0xffffffffu, v, 8);
            v += __shfl_xor_sync(0xffffffffu, v, 16);
            acc[m][t] = v;
        }
    if (lane < 8) {
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                red[warp][m][e0 + t] = acc[m][t];
                red[warp][m][e0 + 32 + t] = acc[m][16 + t];
            }
    }
    __syncthreads();
    const bool direct = gridDim.y == 1;
    for (int i = threadIdx.x; i < MT * 256; i += kThreads) {
        const int m = i >> 8, e = i & 255;
        if (m >= M) continue;
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v += red[w][m][e];
        const int64_t k = int64_t(sb) * 256 + e;
        if (direct)
            out[int64_t(m) * K + k] = v;
        else
            out[(int64_t(r) * M + m) * K + k] = v;
    }
}

// dX[i] = sum over row ranges r = 0..R-1 of part[r][i], i < M*K: in order, in groups of 16
// whose sums are added in order (at most 15 + R/16 roundings in a chain).
__global__ void __launch_bounds__(256) bwd_reduce_kernel(const float* __restrict__ part, int R, int64_t count,
                                                         float* __restrict__ dx) {
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < count; i += int64_t(gridDim.x) * blockDim.x) {
        float v = 0.0f;
        for (int r0 = 0; r0 < R; r0 += 16) {
            float g = part[int64_t(r0) * count + i];
            for (int r = r0 + 1; r < R && r < r0 + 16; ++r) g += part[int64_t(r) * count + i];
            v = (r0 == 0) ? g : v + g;
        }
        dx[i] = v;
    }
}

}  // namespace q4k
}  // namespace w4a8
