// Quantisation kernels: Q8_0 activations (row-major, and the tensor-core operand
// layout the tcgen05 GEMM consumes), Q4_0 weight pack, affine 4-bit weight pack.
//
// Every floating-point step is written with explicit round-to-nearest intrinsics so
// that no multiply-add is contracted and the results are the ones the definitions give:
//   Q8_0  (tract PR #2432, "Pipeline": activation -> int8 per block):
//         d = amax/127 (f32), q = clamp(round_half_away(x * (1/d)), -127, 127).
//   Q4_0  (tract PR #2432, "The kernel": per-32-block weight scale):
//         d = mx/-8 for the first element of largest magnitude mx,
//         q = min(15, trunc(x * (1/d) + 8.5)), scale stored as fp16(d).
//   affine (MLX PR #4802, mode="affine"): s = bf16((max-min)/15), b = bf16(min),
//         q = clamp(round_half_away((w - b)/s), 0, 15).
#pragma once

#include "device_common.cuh"

namespace w4a8 {

// Tensor-core operand geometry shared by the activation kernel and the GEMM: the
// token tile (tokens per GEMM tile) is 16, 32, 64 or 128.
namespace tcgeo {
__host__ __device__ constexpr int tok_block_bytes(int tt) { return tt * 64; }  // one 32-wide block, fp16
}  // namespace tcgeo

// ------------------------------------------------------------------ Q8_0, row-major
// One aligned group of 8 lanes quantises one 32-element block; lane s of the group
// holds elements 4s..4s+3. Blocks are numbered row-major (block = m*K/32 + b), which is
// also the element order of x, so block i covers x[32i .. 32i+31].
template <bool BF16>
__global__ void __launch_bounds__(256) quant_act_rowmajor_kernel(const void* __restrict__ x, int64_t nblocks,
                                                                 int8_t* __restrict__ qx, float* __restrict__ dx,
                                                                 int32_t* __restrict__ sx) {
    pdl_launch_dependents();
    const int64_t blk = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 3;
    const int sub = threadIdx.x & 7;
    const bool valid = blk < nblocks;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (valid) load4<BF16>(x, blk * 32 + sub * 4, v);
    float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
    amax = warp_max8(amax);
    const float d = __fdiv_rn(amax, 127.0f);
    const float id = (d != 0.0f) ? __frcp_rn(d) : 0.0f;
    int q[4];
    int s = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int qi = static_cast<int>(roundf(__fmul_rn(v[i], id)));
        qi = max(-127, min(127, qi));
        q[i] = qi;
        s += qi;
    }
    s = warp_sum8(s);
    if (valid) {
        const uint32_t packed = (uint32_t(q[0]) & 0xFFu) | ((uint32_t(q[1]) & 0xFFu) << 8) |
                                ((uint32_t(q[2]) & 0xFFu) << 16) | ((uint32_t(q[3]) & 0xFFu) << 24);
        *reinterpret_cast<uint32_t*>(qx + blk * 32 + sub * 4) = packed;
        if (sub == 0) {
            dx[blk] = d;
            if (sx) sx[blk] = s;
        }
    }
}

// ------------------------------------------------------------------ Q8_0, MMA operand
// Same quantisation, written as the token operand of the tcgen05 GEMM.
//
// Layout (per token tile t of `tt` rows and block b): a contiguous chunk of tt x 32
// fp16 at chunk index t*B + b. Inside a chunk, token row r and 16-byte segment c
// (c = 0..3) sit at byte (r/8)*512 + c*128 + (r%8)*16: the K-major, no-swizzle
// arrangement of 8-row x 16-byte core matrices (K-adjacent core matrices 128 B apart,
// 8-row groups 512 B apart).
//
// The 8 fp16 slots of segment c hold the block's codes q (exact small integers) in the
// order in which the GEMM's weight expansion produces them (a permutation of K within
// the block, applied identically to both operands, so every block dot is unchanged):
//   FMT 0 (Q4_0):   4c, 4c+2, 4c+1, 4c+3, 16+4c, 16+4c+2, 16+4c+1, 16+4c+3
//   FMT 1 (affine): 8c, 8c+4, 8c+2, 8c+6, 8c+1, 8c+5, 8c+3, 8c+7
//   FMT 2 (affine 6- and 8-bit codes): 8c, 8c+1, ..., 8c+7
// The block scale d goes to `dxs[chunk*tt + r]` (f32). Rows past M are zero (codes and
// scale). For FMT 1 and 2 it also writes, per token and weight group g, Z = the f32 sum over
// the group's blocks of d*sum(q) (the factor of the bias term), at zb[(t*G + g)*tt + r],
// and, when `sums` is given (128-token tiles), per token and block the 16-byte token
// column of the CTA-pair GEMM's bias MMA at sums[chunk*tt + r].
template <bool BF16, int FMT>
__global__ void __launch_bounds__(256) quant_act_tc_kernel(const void* __restrict__ x, int M, int K, int tt,
                                                           int64_t nblocks, __half* __restrict__ tok,
                                                           float* __restrict__ dxs, float* __restrict__ zb,
                                                           int group, uint4* __restrict__ sums) {
    pdl_launch_dependents();
    const int B = K >> 5;
    const int64_t blk = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 3;
    const int sub = threadIdx.x & 7;
    const bool valid = blk < nblocks;
    const int64_t m = valid ? blk / B : 0;
    const int b = valid ? int(blk - m * B) : 0;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (valid && m < M) load4<BF16>(x, m * K + int64_t(b) * 32 + sub * 4, v);
    float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
    amax = warp_max8(amax);
    const float d = __fdiv_rn(amax, 127.0f);
    const float id = (d != 0.0f) ? __frcp_rn(d) : 0.0f;
    int q[4];
    int s = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int qi = static_cast<int>(roundf(__fmul_rn(v[i], id)));
        qi = max(-127, min(127, qi));
        q[i] = qi;
        s += qi;
    }
    s = warp_sum8(s);
    // Exchange codes with the partner lane that holds the other half of the segment.
    const uint32_t mine = (uint32_t(q[0]) & 0xFFu) | ((uint32_t(q[1]) & 0xFFu) << 8) |
                          ((uint32_t(q[2]) & 0xFFu) << 16) | ((uint32_t(q[3]) & 0xFFu) << 24);
    const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, FMT == 0 ? 4 : 1);
    static_assert(FMT >= 0 && FMT <= 2, "token operand order");
    auto code = [](uint32_t w, int i) { return int(int8_t((w >> (8 * i)) & 0xFFu)); };
    const int64_t t = m / tt;
    const int r = int(m - t * tt);
    const int64_t chunk = t * B + b;
    const bool writer = (FMT == 0) ? (sub < 4) : ((sub & 1) == 0);
    if (valid && writer) {
        const int c = (FMT == 0) ? sub : (sub >> 1);
        int e[8];
        if (FMT == 0) {  // own = elements 4c..4c+3, other = 16+4c..16+4c+3
            e[0] = code(mine, 0); e[1] = code(mine, 2); e[2] = code(mine, 1); e[3] = code(mine, 3);
            e[4] = code(other, 0); e[5] = code(other, 2); e[6] = code(other, 1); e[7] = code(other, 3);
        } else if (FMT == 1) {  // own = elements 8c..8c+3, other = 8c+4..8c+7
            e[0] = code(mine, 0); e[1] = code(other, 0); e[2] = code(mine, 2); e[3] = code(other, 2);
            e[4] = code(mine, 1); e[5] = code(other, 1); e[6] = code(mine, 3); e[7] = code(other, 3);
        } else {                // element order
            e[0] = code(mine, 0); e[1] = code(mine, 1); e[2] = code(mine, 2); e[3] = code(mine, 3);
            e[4] = code(other, 0); e[5] = code(other, 1); e[6] = code(other, 2); e[7] = code(other, 3);
        }
        uint32_t h[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t lo = __half_as_ushort(__int2half_rn(e[2 * i]));
            const uint32_t hi = __half_as_ushort(__int2half_rn(e[2 * i + 1]));
            h[i] = lo | (hi << 16);
        }
        char* dst = reinterpret_cast<char*>(tok) + chunk * tcgeo::tok_block_bytes(tt) + (r >> 3) * 512 + c * 128 +
                    (r & 7) * 16;
        *reinterpret_cast<uint4*>(dst) = make_uint4(h[0], h[1], h[2], h[3]);
    }
    if (valid && sub == 0) dxs[chunk * tt + r] = d;
    if (FMT >= 1 && sums) {
        // The block's two 16-element code sums S1 (lanes 0-3) and S2 (lanes 4-7), |S| <= 2032,
        // exact in fp16 as are S/2^11: the token column [S1, S2, S1/2^11, S2/2^11, 0, 0, 0, 0]
        // of the bias MMA of the CTA-pair GEMM (its weight column: b + 8s in two parts).
        int h = q[0] + q[1] + q[2] + q[3];
        h += __shfl_xor_sync(0xffffffffu, h, 1);
        h += __shfl_xor_sync(0xffffffffu, h, 2);
        const int h2 = __shfl_xor_sync(0xffffffffu, h, 4);
        if (valid && sub == 0) {
            const uint32_t p = uint32_t(__half_as_ushort(__int2half_rn(h))) |
                               (uint32_t(__half_as_ushort(__int2half_rn(h2))) << 16);
            const uint32_t ps = uint32_t(__half_as_ushort(__float2half_rn(float(h) * 0x1p-11f))) |
                                (uint32_t(__half_as_ushort(__float2half_rn(float(h2) * 0x1p-11f))) << 16);
            sums[chunk * tt + r] = make_uint4(p, ps, 0u, 0u);
        }
    }
    if (FMT >= 1) {
        // Blocks of one weight group are adjacent 8-lane groups of this warp (the warp's
        // four blocks start at a multiple of 4 and B is a multiple of group/32).
        float z = __fmul_rn(d, float(s));
        if (group >= 64) z = __fadd_rn(z, __shfl_xor_sync(0xffffffffu, z, 8));
        if (group == 128) z = __fadd_rn(z, __shfl_xor_sync(0xffffffffu, z, 16));
        const int gsh = group_shift(group);  // log2(blocks per group)
        if (valid && sub == 0 && (b & ((1 << gsh) - 1)) == 0) {
            const int G = K >> (gsh + 5);
            zb[(t * G + (b >> gsh)) * tt + r] = z;
        }
    }
}

// The same quantisation into the Q4_0 operand (FMT 0) with four lanes per block: lane c
// loads the eight elements of its 16-byte segment (4c..4c+3 and 16+4c..16+4c+3, two
// 16-byte loads for f32 x) and writes that segment, so no codes pass between lanes.
// Same layout, rounding and padding as quant_act_tc_kernel<BF16, 0>.
template <bool BF16>
__global__ void __launch_bounds__(256) quant_act_tc4_kernel(const void* __restrict__ x, int M, int K, int tt,
                                                            int64_t nblocks, __half* __restrict__ tok,
                                                            float* __restrict__ dxs) {
    pdl_launch_dependents();
    const int B = K >> 5;
    const int64_t blk = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 2;
    const int c = threadIdx.x & 3;
    const bool valid = blk < nblocks;
    const int64_t m = valid ? blk / B : 0;
    const int b = valid ? int(blk - m * B) : 0;
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (valid && m < M) {
        float a[4], h[4];
        load4<BF16>(x, m * K + int64_t(b) * 32 + c * 4, a);
        load4<BF16>(x, m * K + int64_t(b) * 32 + 16 + c * 4, h);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[i] = a[i];
            v[4 + i] = h[i];
        }
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const float d = __fdiv_rn(amax, 127.0f);
    const float id = (d != 0.0f) ? __frcp_rn(d) : 0.0f;
    int q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = max(-127, min(127, static_cast<int>(roundf(__fmul_rn(v[i], id)))));
    if (valid) {
        const int64_t t = m / tt;
        const int r = int(m - t * tt);
        const int64_t chunk = t * B + b;
        // slot order of segment c: 4c, 4c+2, 4c+1, 4c+3, 16+4c, 16+4c+2, 16+4c+1, 16+4c+3
        const int e[8] = {q[0], q[2], q[1], q[3], q[4], q[6], q[5], q[7]};
        uint32_t hw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            hw[i] = uint32_t(__half_as_ushort(__int2half_rn(e[2 * i]))) |
                    (uint32_t(__half_as_ushort(__int2half_rn(e[2 * i + 1]))) << 16);
        char* dst = reinterpret_cast<char*>(tok) + chunk * tcgeo::tok_block_bytes(tt) + (r >> 3) * 512 + c * 128 +
                    (r & 7) * 16;
        *reinterpret_cast<uint4*>(dst) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        if (c == 0) dxs[chunk * tt + r] = d;
    }
}

// ------------------------------------------------------------------ Q4_0 pack
// 8 lanes per block; blocks numbered row-major, so block i is W[32i .. 32i+31] and its
// 16 code bytes are qs[16i .. 16i+15].
template <bool BF16>
__global__ void __launch_bounds__(256) pack_q4_0_kernel(const void* __restrict__ w, int64_t nblocks,
                                                        uint8_t* __restrict__ qs, uint16_t* __restrict__ dq) {
    const int64_t blk = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 3;
    const int sub = threadIdx.x & 7;
    const bool valid = blk < nblocks;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (valid) load4<BF16>(w, blk * 32 + sub * 4, v);
    // first element of largest magnitude: reduce (|x| descending, index ascending)
    float a = 0.0f, mx = 0.0f;
    int idx = 32;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (fabsf(v[i]) > a) { a = fabsf(v[i]); mx = v[i]; idx = sub * 4 + i; }
    }
#pragma unroll
    for (int off = 4; off >= 1; off >>= 1) {
        const float oa = __shfl_xor_sync(0xffffffffu, a, off);
        const float om = __shfl_xor_sync(0xffffffffu, mx, off);
        const int oi = __shfl_xor_sync(0xffffffffu, idx, off);
        if (oa > a || (oa == a && oi < idx)) { a = oa; mx = om; idx = oi; }
    }
    const float d = __fdiv_rn(mx, -8.0f);
    const float id = (d != 0.0f) ? __frcp_rn(d) : 0.0f;
    uint32_t mine = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int qi = __float2int_rz(__fadd_rn(__fmul_rn(v[i], id), 8.5f));
        qi = max(0, min(15, qi));
        mine |= uint32_t(qi) << (8 * i);
    }
    const uint32_t hi = __shfl_xor_sync(0xffffffffu, mine, 4);
    if (valid && sub < 4) *reinterpret_cast<uint32_t*>(qs + blk * 16 + sub * 4) = mine | (hi << 4);
    if (valid && sub == 0) dq[blk] = __half_as_ushort(__float2half_rn(d));
}

// ------------------------------------------------------------------ affine pack
// group/4 lanes per group (8 for 32, 16 for 64, 32 for 128); groups numbered row-major.
// min and max keep the first occurrence among equal values (so signed zeros resolve
// the way a sequential scan does). BITS-bit codes (4, 6 or 8) of a row form a
// little-endian bit stream: element k at bits [BITS*k, BITS*k + BITS) of the row's bytes.
template <bool BF16, int BITS>
__global__ void __launch_bounds__(256) pack_affine_kernel(const void* __restrict__ w, int64_t ngroups, int group,
                                                          uint8_t* __restrict__ q, uint16_t* __restrict__ scale,
                                                          uint16_t* __restrict__ bias) {
    constexpr int QMAX = (1 << BITS) - 1;
    const int L = group >> 2;  // lanes per group (power of two)
    const int64_t gt = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t grp = gt / L;
    const int sub = int(gt - grp * L);
    const bool valid = grp < ngroups;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (valid) load4<BF16>(w, grp * group + sub * 4, v);
    float mn = v[0], mx = v[0];
    int imn = sub * 4, imx = sub * 4;
#pragma unroll
    for (int i = 1; i < 4; ++i) {
        if (v[i] < mn) { mn = v[i]; imn = sub * 4 + i; }
        if (v[i] > mx) { mx = v[i]; imx = sub * 4 + i; }
    }
    for (int off = L >> 1; off >= 1; off >>= 1) {
        const float omn = __shfl_xor_sync(0xffffffffu, mn, off);
        const int oimn = __shfl_xor_sync(0xffffffffu, imn, off);
        const float omx = __shfl_xor_sync(0xffffffffu, mx, off);
        const int oimx = __shfl_xor_sync(0xffffffffu, imx, off);
        if (omn < mn || (omn == mn && oimn < imn)) { mn = omn; imn = oimn; }
        if (omx > mx || (omx == mx && oimx < imx)) { mx = omx; imx = oimx; }
    }
    const float range = __fsub_rn(mx, mn);
    const __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(range, float(QMAX)));
    const __nv_bfloat16 bb = __float2bfloat16_rn(mn);
    const float sf = __bfloat162float(sb), bf = __bfloat162float(bb);
    uint32_t mine = 0;  // this lane's 4 codes, BITS bits each
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int qi = 0;
        if (sf != 0.0f) {
            qi = static_cast<int>(roundf(__fdiv_rn(__fsub_rn(v[i], bf), sf)));
            qi = max(0, min(QMAX, qi));
        }
        mine |= uint32_t(qi) << (BITS * i);
    }
    uint8_t* qg = q + grp * (group * BITS / 8);  // the group's first byte
    if (BITS == 4) {
        const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
        if (valid && (sub & 1) == 0) reinterpret_cast<uint32_t*>(qg)[sub >> 1] = mine | (other << 16);
    } else if (BITS == 8) {
        if (valid) reinterpret_cast<uint32_t*>(qg)[sub] = mine;
    } else {  // 24 bits per lane: 3 bytes
        if (valid) {
            qg[sub * 3] = uint8_t(mine);
            qg[sub * 3 + 1] = uint8_t(mine >> 8);
            qg[sub * 3 + 2] = uint8_t(mine >> 16);
        }
    }
    if (valid && sub == 0) {
        scale[grp] = __bfloat16_as_ushort(sb);
        bias[grp] = __bfloat16_as_ushort(bb);
    }
}

}  // namespace w4a8
