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
                                                             float* __restrict__ y) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = blockIdx.x * kGemvWarps + warp;
    if (n >= N) return;
    const int B = K >> 5;
    const int G = (FMT == 1) ? K / group : 0;
    const int bpg = (FMT == 1) ? (group >> 5) : 1;
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
                    const int g = b / bpg;
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
        if (lane == 0 && m < M) y[int64_t(m) * N + n] = v;
    }
}

}  // namespace w4a8
