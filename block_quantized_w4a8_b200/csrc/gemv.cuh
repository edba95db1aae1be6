// Small-M path: the packed weights are streamed once with 128-bit loads, nibbles are
// decoded in registers, block dots use dp4a and each output is reduced across the warp
// with shuffles. This is the memory-bound decode case of tract PR #2432 (follow-up
// "decode regime (m=1)"): at M = 1 the weight stream is the whole cost.
//
// One warp per weight row; lane l takes blocks l, l+32, l+64, ... of the row, so a
// warp's loads of one 32-block step cover 512 contiguous bytes of the row. The
// activations (Q8_0 codes, scales and block sums from the act-quant kernel) are read
// after griddepcontrol.wait, the weights before it, so the weight stream overlaps the
// activation quantisation under programmatic dependent launch.
#pragma once

#include "device_common.cuh"

namespace w4a8 {

constexpr int kGemvWarps = 8;   // rows per CTA
constexpr int kGemvUnroll = 4;  // 32-block steps whose loads are in flight together

__device__ __forceinline__ uint4 ld_stream(const uint4* p) { return __ldcs(p); }

// FMT 0: Q4_0 (codes in nibbles, block scale fp16 per 32).
// FMT 1: affine (eight codes per word, bf16 scale and bias per group).
template <int MT, int FMT>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_kernel(int M, int N, int K, int group,
                                                             const int8_t* __restrict__ qx,
                                                             const float* __restrict__ dx,
                                                             const int32_t* __restrict__ sx,
                                                             const uint8_t* __restrict__ wq,
                                                             const uint16_t* __restrict__ wscale,
                                                             const uint16_t* __restrict__ wbias,
                                                             void* __restrict__ y, Epilogue epi) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = blockIdx.x * kGemvWarps + warp;
    if (n >= N) return;
    const int B = K >> 5;
    const int G = (FMT == 1) ? K / group : 0;
    const int bsh = (FMT == 1) ? group_shift(group) : 0;  // log2(blocks per group): no run-time division
    const uint4* wrow = reinterpret_cast<const uint4*>(wq + int64_t(n) * (K >> 1));
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
    bool waited = false;
    for (int b0 = 0; b0 < B; b0 += 32 * kGemvUnroll) {
        uint4 wv[kGemvUnroll];
        float ws[kGemvUnroll], wb[kGemvUnroll];
#pragma unroll
        for (int u = 0; u < kGemvUnroll; ++u) {
            const int b = b0 + u * 32 + lane;
            wv[u] = make_uint4(0u, 0u, 0u, 0u);
            ws[u] = 0.0f;
            wb[u] = 0.0f;
            if (b < B) {
                wv[u] = ld_stream(wrow + b);
                if (FMT == 0) {
                    ws[u] = __half2float(__ushort_as_half(wscale[int64_t(n) * B + b]));
                } else {
                    const int g = b >> bsh;
                    ws[u] = __bfloat162float(__ushort_as_bfloat16(wscale[int64_t(n) * G + g]));
                    wb[u] = __bfloat162float(__ushort_as_bfloat16(wbias[int64_t(n) * G + g]));
                }
            }
        }
        if (!waited) {
            pdl_wait_primary();
            waited = true;
        }
#pragma unroll
        for (int u = 0; u < kGemvUnroll; ++u) {
            const int b = b0 + u * 32 + lane;
            if (b >= B) continue;
            const uint32_t w[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
            uint32_t lo[4], hi[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                lo[i] = w[i] & 0x0F0F0F0Fu;         // Q4_0: elements 4i..4i+3; affine: 8i, 8i+2, 8i+4, 8i+6
                hi[i] = (w[i] >> 4) & 0x0F0F0F0Fu;  // Q4_0: elements 16+4i..;  affine: 8i+1, 8i+3, 8i+5, 8i+7
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m < M) {
                    const int4* a = reinterpret_cast<const int4*>(qx + int64_t(m) * K + int64_t(b) * 32);
                    const int4 a0 = a[0], a1 = a[1];
                    const int aw[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                    int dot = 0;
                    if (FMT == 0) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            dot = __dp4a(int(lo[i]), aw[i], dot);
                            dot = __dp4a(int(hi[i]), aw[4 + i], dot);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int ev = int(__byte_perm(aw[2 * i], aw[2 * i + 1], 0x6420));
                            const int od = int(__byte_perm(aw[2 * i], aw[2 * i + 1], 0x7531));
                            dot = __dp4a(int(lo[i]), ev, dot);
                            dot = __dp4a(int(hi[i]), od, dot);
                        }
                    }
                    const int S = sx[int64_t(m) * B + b];
                    const float dxv = dx[int64_t(m) * B + b];
                    if (FMT == 0) {
                        const int D = dot - 8 * S;  // sum (q - 8) * q_x
                        acc[m] = fmaf(__fmul_rn(ws[u], dxv), float(D), acc[m]);
                    } else {
                        const float t = fmaf(ws[u], float(dot), __fmul_rn(wb[u], float(S)));
                        acc[m] = fmaf(dxv, t, acc[m]);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        float v = acc[m];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0 && m < M) epi_store(y, int64_t(m) * N + n, n, v, epi);
    }
}

}  // namespace w4a8

namespace w4a8 {

// ------------------------------------------------------------------ persistent GEMV
// One 512-thread CTA per SM. Warp w of the grid takes rows w, w+W, w+2W, ... (W = all
// warps); a work item is 128 consecutive blocks of one row (lane l: blocks l, l+32,
// l+64, l+96 of the item). The weight loads of the first three items are issued before
// anything else, and every later item is loaded three items ahead, so each SM keeps
// ~48-96 KB of weights in flight. The activation (Q8_0 codes, scales, block sums) lives
// in shared memory for the whole kernel: either quantised here from x (XMODE 1 = f32 x,
// 2 = bf16 x; the same arithmetic as quant_act_rowmajor_kernel) or copied from a
// prepared workspace after griddepcontrol.wait (XMODE 0).
// Shared layout of the codes: row m, half h (bytes 0-15 / 16-31 of a block), block b at
// m*K + h*K/2 + 16b, so the 16-byte loads of consecutive lanes are consecutive.
constexpr int kGemv2Warps = 16;
constexpr int kGemv2Threads = kGemv2Warps * 32;
constexpr int kGemv2ItemBlocks = 128;

__host__ __device__ constexpr size_t gemv2_smem_bytes(int MT, int K) {
    return ((size_t(MT) * K + 15) & ~size_t(15)) + size_t(MT) * (K / 32) * 8;
}

template <int MT, int FMT, int XMODE>
__global__ void __launch_bounds__(kGemv2Threads, 1)
    gemv2_kernel(int M, int N, int K, int group, const void* __restrict__ x, const int8_t* __restrict__ qx,
                 const float* __restrict__ dx, const int32_t* __restrict__ sx, const uint8_t* __restrict__ wq,
                 const uint16_t* __restrict__ wscale, const uint16_t* __restrict__ wbias, void* __restrict__ y,
                 Epilogue epi) {
    extern __shared__ __align__(16) uint8_t g2_smem[];
    const int B = K >> 5;
    int8_t* qs_ = reinterpret_cast<int8_t*>(g2_smem);
    float* dxs = reinterpret_cast<float*>(g2_smem + ((size_t(MT) * K + 15) & ~size_t(15)));
    int32_t* sxs = reinterpret_cast<int32_t*>(dxs + MT * B);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int W = gridDim.x * kGemv2Warps;
    const int gw = blockIdx.x * kGemv2Warps + warp;
    const int C = (B + kGemv2ItemBlocks - 1) / kGemv2ItemBlocks;
    const int rows_w = (gw < N) ? (N - 1 - gw) / W + 1 : 0;
    const int T = rows_w * C;
    const int G = (FMT == 1) ? K / group : 0;
    const int bsh = (FMT == 1) ? group_shift(group) : 0;  // log2(blocks per group): no run-time division

    struct Item {
        uint4 w[4];
        float s[4], b[4];
    };
    auto load_item = [&](int t, Item& it) {
        const int n = gw + (t / C) * W;
        const int c = t - (t / C) * C;
        const uint4* wrow = reinterpret_cast<const uint4*>(wq + int64_t(n) * (K >> 1));
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int b = c * kGemv2ItemBlocks + u * 32 + lane;
            it.w[u] = make_uint4(0u, 0u, 0u, 0u);
            it.s[u] = 0.0f;
            it.b[u] = 0.0f;
            if (b < B) {
                it.w[u] = ld_stream(wrow + b);
                if (FMT == 0) {
                    it.s[u] = __half2float(__ushort_as_half(wscale[int64_t(n) * B + b]));
                } else {
                    it.s[u] = __bfloat162float(__ushort_as_bfloat16(wscale[int64_t(n) * G + (b >> bsh)]));
                    it.b[u] = __bfloat162float(__ushort_as_bfloat16(wbias[int64_t(n) * G + (b >> bsh)]));
                }
            }
        }
    };

    Item i0, i1, i2;
    if (0 < T) load_item(0, i0);
    if (1 < T) load_item(1, i1);
    if (2 < T) load_item(2, i2);
    // A dependent launch may start its own weight prefetch now; it still waits for this
    // grid to complete before it reads anything this grid writes.
    pdl_launch_dependents();
    // x (or its prepared quantisation) may be written by the preceding kernel.
    pdl_wait_primary();

    // ---- activation into shared memory
    if (XMODE == 0) {
        const int pieces = M * B * 2;  // 16-byte pieces of the codes
        for (int p = threadIdx.x; p < pieces; p += kGemv2Threads) {
            const int m = p / (2 * B), rem = p - m * 2 * B, b = rem >> 1, h = rem & 1;
            const uint4 v = *reinterpret_cast<const uint4*>(qx + int64_t(m) * K + b * 32 + h * 16);
            *reinterpret_cast<uint4*>(qs_ + m * K + h * (K >> 1) + b * 16) = v;
        }
        for (int i = threadIdx.x; i < M * B; i += kGemv2Threads) {
            dxs[i] = dx[i];
            sxs[i] = sx[i];
        }
    } else {
        const int nblk = M * B;
        const int sub = threadIdx.x & 7;
        for (int base = 0; base < nblk; base += kGemv2Threads / 8) {
            const int blk = base + (threadIdx.x >> 3);
            const bool valid = blk < nblk;
            float v[4] = {0.f, 0.f, 0.f, 0.f};
            if (valid) load4<XMODE == 2>(x, int64_t(blk) * 32 + sub * 4, v);
            float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
            amax = warp_max8(amax);
            const float d = __fdiv_rn(amax, 127.0f);
            const float id = (d != 0.0f) ? __frcp_rn(d) : 0.0f;
            int s = 0;
            uint32_t packed = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                int qi = static_cast<int>(roundf(__fmul_rn(v[i], id)));
                qi = max(-127, min(127, qi));
                s += qi;
                packed |= (uint32_t(qi) & 0xFFu) << (8 * i);
            }
            s = warp_sum8(s);
            if (valid) {
                const int m = blk / B, b = blk - m * B;
                *reinterpret_cast<uint32_t*>(qs_ + m * K + (sub >> 2) * (K >> 1) + b * 16 + (sub & 3) * 4) = packed;
                if (sub == 0) {
                    dxs[blk] = d;
                    sxs[blk] = s;
                }
            }
        }
    }
    __syncthreads();

    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.0f;

    auto process = [&](int t, const Item& it) {
        const int n = gw + (t / C) * W;
        const int c = t - (t / C) * C;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int b = c * kGemv2ItemBlocks + u * 32 + lane;
            if (b < B) {
                const uint32_t w[4] = {it.w[u].x, it.w[u].y, it.w[u].z, it.w[u].w};
                uint32_t lo[4], hi[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    lo[i] = w[i] & 0x0F0F0F0Fu;
                    hi[i] = (w[i] >> 4) & 0x0F0F0F0Fu;
                }
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m < M) {
                        const int4 a0 = *reinterpret_cast<const int4*>(qs_ + m * K + b * 16);
                        const int4 a1 = *reinterpret_cast<const int4*>(qs_ + m * K + (K >> 1) + b * 16);
                        const int aw[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                        int dot = 0;
                        if (FMT == 0) {
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                dot = __dp4a(int(lo[i]), aw[i], dot);
                                dot = __dp4a(int(hi[i]), aw[4 + i], dot);
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                dot = __dp4a(int(lo[i]), int(__byte_perm(aw[2 * i], aw[2 * i + 1], 0x6420)), dot);
                                dot = __dp4a(int(hi[i]), int(__byte_perm(aw[2 * i], aw[2 * i + 1], 0x7531)), dot);
                            }
                        }
                        const int S = sxs[m * B + b];
                        const float dxv = dxs[m * B + b];
                        if (FMT == 0) {
                            acc[m] = fmaf(__fmul_rn(it.s[u], dxv), float(dot - 8 * S), acc[m]);
                        } else {
                            acc[m] = fmaf(dxv, fmaf(it.s[u], float(dot), __fmul_rn(it.b[u], float(S))), acc[m]);
                        }
                    }
                }
            }
        }
        if (c == C - 1) {  // row complete: reduce over the warp and store
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                float v = acc[m];
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                if (lane == 0 && m < M) epi_store(y, int64_t(m) * N + n, n, v, epi);
                acc[m] = 0.0f;
            }
        }
    };

    for (int t = 0; t < T; t += 3) {
        process(t, i0);
        if (t + 3 < T) load_item(t + 3, i0);
        if (t + 1 < T) {
            process(t + 1, i1);
            if (t + 4 < T) load_item(t + 4, i1);
        }
        if (t + 2 < T) {
            process(t + 2, i2);
            if (t + 5 < T) load_item(t + 5, i2);
        }
    }
}

}  // namespace w4a8

namespace w4a8 {

// ------------------------------------------------------------------ GEMV, 6- and 8-bit affine codes
// Same scheme as gemv_kernel (one warp per weight row, lane l takes blocks l, l+32, ...;
// weights before griddepcontrol.wait, activations after it) for codes of BITS = 6 or 8
// bits in a little-endian bit stream (24 or 32 bytes per 32-block). The block dot runs
// on dp4a with the codes widened to one byte each: 8-bit codes as q - 128 (q ^ 0x80 read
// as a signed byte), so D = dot + 128 * sum(q_x); 6-bit codes (0..63) as they are.
template <int MT, int BITS>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_wide_kernel(int M, int N, int K, int group,
                                                                  const int8_t* __restrict__ qx,
                                                                  const float* __restrict__ dx,
                                                                  const int32_t* __restrict__ sx,
                                                                  const uint8_t* __restrict__ wq,
                                                                  const uint16_t* __restrict__ wscale,
                                                                  const uint16_t* __restrict__ wbias,
                                                                  void* __restrict__ y, Epilogue epi) {
    static_assert(BITS == 6 || BITS == 8, "code width");
    constexpr int WORDS = BITS;  // 32-bit words per block (4 * BITS bytes)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = blockIdx.x * kGemvWarps + warp;
    if (n >= N) return;
    const int B = K >> 5;
    const int bsh = group_shift(group);
    const int G = B >> bsh;
    const uint8_t* wrow = wq + int64_t(n) * (int64_t(K) * BITS / 8);
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
    bool waited = false;
    for (int b0 = 0; b0 < B; b0 += 32 * kGemvUnroll) {
        uint32_t wv[kGemvUnroll][WORDS];
        float ws[kGemvUnroll], wb[kGemvUnroll];
#pragma unroll
        for (int u = 0; u < kGemvUnroll; ++u) {
            const int b = b0 + u * 32 + lane;
#pragma unroll
            for (int i = 0; i < WORDS; ++i) wv[u][i] = 0u;
            ws[u] = 0.0f;
            wb[u] = 0.0f;
            if (b < B) {
                if (BITS == 8) {
                    const uint4* p = reinterpret_cast<const uint4*>(wrow + int64_t(b) * 32);
                    const uint4 v0 = ld_stream(p), v1 = ld_stream(p + 1);
                    wv[u][0] = v0.x; wv[u][1] = v0.y; wv[u][2] = v0.z; wv[u][3] = v0.w;
                    wv[u][4] = v1.x; wv[u][5] = v1.y; wv[u][6] = v1.z; wv[u][7] = v1.w;
                } else {
                    const uint2* p = reinterpret_cast<const uint2*>(wrow + int64_t(b) * 24);
#pragma unroll
                    for (int i = 0; i < 3; ++i) {
                        const uint2 v = __ldcs(p + i);
                        wv[u][2 * i] = v.x;
                        wv[u][2 * i + 1] = v.y;
                    }
                }
                const int g = b >> bsh;
                ws[u] = __bfloat162float(__ushort_as_bfloat16(wscale[int64_t(n) * G + g]));
                wb[u] = __bfloat162float(__ushort_as_bfloat16(wbias[int64_t(n) * G + g]));
            }
        }
        if (!waited) {
            pdl_wait_primary();
            waited = true;
        }
#pragma unroll
        for (int u = 0; u < kGemvUnroll; ++u) {
            const int b = b0 + u * 32 + lane;
            if (b >= B) continue;
            uint32_t c[8];  // codes 4i..4i+3 as bytes
            if (BITS == 8) {
#pragma unroll
                for (int i = 0; i < 8; ++i) c[i] = wv[u][i] ^ 0x80808080u;
            } else {
                // 24-bit groups of four codes at bit 24i of the block's 192-bit stream
                uint32_t v[8];
                v[0] = wv[u][0];
                v[1] = __funnelshift_r(wv[u][0], wv[u][1], 24);
                v[2] = __funnelshift_r(wv[u][1], wv[u][2], 16);
                v[3] = wv[u][2] >> 8;
                v[4] = wv[u][3];
                v[5] = __funnelshift_r(wv[u][3], wv[u][4], 24);
                v[6] = __funnelshift_r(wv[u][4], wv[u][5], 16);
                v[7] = wv[u][5] >> 8;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    c[i] = (v[i] & 0x3Fu) | ((v[i] << 2) & 0x3F00u) | ((v[i] << 4) & 0x3F0000u) |
                           ((v[i] << 6) & 0x3F000000u);
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m < M) {
                    const int4* a = reinterpret_cast<const int4*>(qx + int64_t(m) * K + int64_t(b) * 32);
                    const int4 a0 = a[0], a1 = a[1];
                    const int aw[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                    int dot = 0;
#pragma unroll
                    for (int i = 0; i < 8; ++i) dot = __dp4a(int(c[i]), aw[i], dot);
                    const int S = sx[int64_t(m) * B + b];
                    const float dxv = dx[int64_t(m) * B + b];
                    const int D = (BITS == 8) ? dot + 128 * S : dot;  // sum q * q_x
                    const float t = fmaf(ws[u], float(D), __fmul_rn(wb[u], float(S)));
                    acc[m] = fmaf(dxv, t, acc[m]);
                }
            }
        }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        float v = acc[m];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0 && m < M) epi_store(y, int64_t(m) * N + n, n, v, epi);
    }
}

}  // namespace w4a8
