// Tensor-core path: tcgen05 GEMM with the weight block scale folded into the weight
// operand and the activation block scale applied per block in the epilogue.
//
// y[m][n] = sum_b  d_x[m][b] * P[m][n][b],   P = d_w[n][b] * D[m][n][b],
// D = the exact 32-wide integer block dot. The block dot must stay exact and each block
// must be rescaled separately (tract PR #2432, "The kernel": Q4_0's per-32-block scales
// force a per-block rescale, one multiply per block over accumulator lanes that each own
// one output). Here the tensor core produces P directly, exactly up to the f32 rounding
// of its accumulator, and the epilogue does one f32 FMA per (output, block):
//
// Weight operand (fp16, one K-major core-matrix tile per block):
//   Q4_0:   d_w = d_hi + d_lo, d_hi = d_w with the three lowest significand bits cleared
//           (8 significant bits), d_lo = the rest (3 bits). The slots hold d_hi*(q-8) and
//           d_lo*(q-8): an 8-bit times a 3-bit magnitude (|q-8| <= 8) fits the 11-bit fp16
//           significand, so both parts are exact; they are formed by one fused multiply-add
//           whose addend 24*d_hi must fit fp16, so |d_hi| <= 2720 (larger, infinite or nan
//           scales set W4A8_ERR_RANGE in the device status word). Four kind::f16
//           MMAs (hi and lo parts, two K = 16 halves each) accumulate d_w*D in one TMEM
//           tile: the hi half-sums are exact, the lo parts add at most two f32 roundings.
//   affine: s*(q-8) with s the bf16 group scale (8 significant bits): exact in fp16 for
//           2^-17 <= |s| <= 2720 (or s = 0; others set W4A8_ERR_RANGE). Two MMAs per block
//           give s*sum (q-8)*q_x; the epilogue adds (b + 8s)*Z per group, where
//           Z[m][g] = sum over the group's blocks of d_x*sum(q_x) (MLX PR #4802, mode
//           "affine": scale and bias applied on the original codes, rewritten with the
//           codes centred at 8 so that the scaled codes stay exact in fp16).
// Token operand: the Q8_0 codes as fp16 (exact), written by quant_act_tc_kernel in the
// same K permutation as the weight expansion.
//
// Two orientations of the same MMA (K-major operands, so A and B just swap roles):
//   TOKL = true  (large M): TMEM lane = token (128 per tile), TMEM column = weight row
//                (MN per tile). d_x is a per-thread scalar: the epilogue is acc += d_x * P.
//   TOKL = false (small M): TMEM lane = weight row (128 per tile), TMEM column = token
//                (MN = 16..128 per tile, so few MMA rows are padding); d_x comes from a
//                broadcast shared-memory load per 4 tokens.
// Warp roles: EPI_WARPS epilogue warps (warp w reads TMEM lane quarter w%4, column chunk
// w/4 of CW columns, accumulates in f32 registers); PROD_WARPS producer warps (one weight
// row per thread: reads the stage's packed codes and scales, nibble -> scaled fp16
// expansion, store in the core-matrix layout); one MMA-issue warp (also allocates TMEM);
// one copy warp (2-D TMA boxes of the packed weights; token operand, d_x and Z via plain
// cp.async.bulk, each CTA fetching its own data). The
// MMA and copy warps run their loops warp-uniformly with one elected lane issuing. Every
// wait is bounded and taken by each warp on its own (all lanes probe, a vote keeps the
// warp converged), so no role is held in lockstep by its slowest warp; the epilogue
// releases a pipeline stage as soon as it has read the stage's scales. On a timeout all
// roles stop, outstanding copies and MMAs are drained, TMEM is freed and the kernel
// returns.
#pragma once

#include <cuda.h>  // CUtensorMap (the type only; maps are encoded by the host code)

#include "device_common.cuh"
#include "quant.cuh"

namespace w4a8 {

// Bit set in the device status word when a weight scale is outside the range in which
// the tensor-core path's fp16 weight operand is exact.
constexpr unsigned kDevErrRange = 2u;

namespace tc {

constexpr int CTRL_BYTES = 1024;
constexpr uint32_t LBO = 128, SBO = 512;  // core-matrix strides: along K, along rows
constexpr int SMEM_LIMIT = 232448;

__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int align_up(int v, int a) { return (v + a - 1) / a * a; }

// Geometry of one instantiation. FMT: 0 = Q4_0, 1 = affine. MN: the MMA's N (weight
// rows per tile when TOKL, tokens per tile otherwise); the MMA's M is always 128.
template <int FMT, bool TOKL, int MN>
struct Geo {
    static constexpr int TT = TOKL ? 128 : MN;   // tokens per tile
    static constexpr int NW = TOKL ? MN : 128;   // weight rows per tile
    static constexpr int WP = (FMT == 0) ? 2 : 1;  // weight operand parts (hi, lo)
    static constexpr int W_PART = NW * 64;       // bytes of one part of one block
    static constexpr int W_BLK = W_PART * WP;
    static constexpr int T_BLK = TT * 64;
    static constexpr int DX_BLK = TT * 4;
    static constexpr int PER_BLK = W_BLK + T_BLK;
    // Quant blocks per pipeline stage (one tcgen05.commit covers a stage).
    static constexpr int S = PER_BLK <= 12288 ? 4 : (PER_BLK <= 24576 ? 2 : 1);
    static constexpr int OFF_T = S * W_BLK;
    static constexpr int OFF_DX = OFF_T + S * T_BLK;
    static constexpr int OFF_C = align_up(OFF_DX + S * DX_BLK, 128);           // affine: b + 8s per row
    static constexpr int OFF_Z = OFF_C + (FMT == 1 ? S * NW * 4 : 0);          // affine: Z per token
    // Packed weights as fetched by TMA: per block of the stage a [NW rows][16 B] box of
    // codes; the scales (and affine biases) of the 8 blocks (groups) around the stage as a
    // [NW rows][8 x 16 bit] box each.
    static constexpr int OFF_RAW = align_up(OFF_Z + (FMT == 1 ? S * TT * 4 : 0), 128);
    static constexpr int OFF_RSC = OFF_RAW + S * NW * 16;
    static constexpr int OFF_RBI = OFF_RSC + NW * 16;
    static constexpr int STAGE_BYTES = align_up(OFF_RBI + (FMT == 1 ? NW * 16 : 0), 1024);
    static constexpr int NS = cmin(8, (SMEM_LIMIT - CTRL_BYTES - 1024) / STAGE_BYTES);
    static constexpr int SMEM_BYTES = NS * STAGE_BYTES + CTRL_BYTES + 1024;
    static constexpr int NBUF = cmin(16, 512 / MN);  // TMEM accumulator tiles (one per block)
    static constexpr int NG = NBUF / S;              // TMEM groups: stage st uses group st % NG
    static constexpr int TMEM_COLS = NBUF * MN;
    static constexpr int CW = cmin(MN, 64);  // columns per epilogue warp
    static constexpr int EPI_WARPS = 4 * MN / CW;
    static constexpr int PROD_WARPS = NW / 32;
    static constexpr int PROD_WARP0 = EPI_WARPS;
    static constexpr int MMA_WARP = PROD_WARP0 + PROD_WARPS;
    static constexpr int COPY_WARP = MMA_WARP + 1;
    static constexpr int NUM_THREADS = (COPY_WARP + 1) * 32;
    // Registers per thread at this size: each SM sub-partition holds ceil(warps/4) warps
    // of the CTA in 16384 registers. Below 160 the epilogue reads its columns in halves
    // so that the accumulators and one half of the tile fit.
    static constexpr int REG_CAP = 16384 / (((NUM_THREADS / 32) + 3) / 4 * 32) / 8 * 8;
    static constexpr int LD_COLS = (REG_CAP < 160 && CW == 64) ? 32 : CW;
    static constexpr uint32_t IDESC = idesc_f16_f32(128, MN);
    static_assert(MN == 16 || MN == 32 || MN == 64 || MN == 128, "MMA N");
    static_assert(!TOKL || MN >= 64, "token-lane tiles cover 64 or 128 weight rows");
    static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM allocation");
    static_assert(NS >= 2, "pipeline depth");
    static_assert(NG >= 2 && NBUF % S == 0, "TMEM groups");
    static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory");
    static_assert(OFF_T % 128 == 0 && OFF_DX % 16 == 0 && OFF_Z % 16 == 0, "operand alignment");
};

constexpr int MAX_NS = 8, MAX_NG = 8;
struct Ctrl {
    unsigned long long raw[MAX_NS];     // TMA of the packed weights (1 arrival + bytes)
    unsigned long long full[MAX_NS];    // producer threads (one arrival per weight row) + bulk copies (1 + bytes)
    unsigned long long empty[MAX_NS];   // one arrival per epilogue warp (after the stage's MMAs completed
                                        // and the warp read the stage's scales)
    unsigned long long tfull[MAX_NG];   // MMA commit, once per stage
    unsigned long long tempty[MAX_NG];  // one arrival per epilogue warp
    unsigned long long drain;             // final MMA drain
    uint32_t tmem_base;
    uint32_t abort;
};
static_assert(sizeof(Ctrl) <= CTRL_BYTES, "control block");


// One 32-bit word of packed codes as four fp16x2 words holding 8 + q/2: each nibble is
// moved to mantissa bits 6..9 under the exponent of 8.0 (0x4800). Slot order (both
// operands use it): Q4_0 word i = bytes 4i..4i+3 of a block gives elements 4i, 4i+2 |
// 4i+1, 4i+3 | 16+4i, 16+4i+2 | 16+4i+1, 16+4i+3; affine word t (element 8t+e at bits
// 4e) gives 8t, 8t+4 | 8t+2, 8t+6 | 8t+1, 8t+5 | 8t+3, 8t+7.
__device__ __forceinline__ void codes_raw(uint32_t w, uint32_t (&r)[4]) {
    constexpr uint32_t M = 0x03C003C0u, E = 0x48004800u;
    r[0] = ((w << 6) & M) | E;
    r[1] = ((w >> 2) & M) | E;
    r[2] = ((w << 2) & M) | E;
    r[3] = ((w >> 6) & M) | E;
}
// (8 + q/2) * (2d) - 24d = (q - 8) * d in one fused multiply-add per pair. With d of at
// most 8 significant bits (d_hi, d_lo, or a bf16 scale) the addend 24d and the result
// (q - 8)*d are representable in fp16, so the single rounding leaves them exact.
__device__ __forceinline__ uint32_t scaled_codes(uint32_t raw, uint32_t d2x2, uint32_t m24d2) {
    __half2 r = __hfma2(*reinterpret_cast<const __half2*>(&raw), *reinterpret_cast<const __half2*>(&d2x2),
                        *reinterpret_cast<const __half2*>(&m24d2));
    return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t pair_of(__half h) { return uint32_t(__half_as_ushort(h)) * 0x10001u; }

// Global load written as volatile asm so that the compiler issues it where it stands in
// the program (stages ahead of its use) instead of sinking it to the first use.
__device__ __forceinline__ uint16_t ld_nc_u16(const void* p) {
    uint16_t v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// Loads CW TMEM columns of this warp's lane quarter into registers (and waits for them).
__device__ __forceinline__ void tmem_load_cols(uint32_t taddr, uint32_t (&r)[64]) {
    tmem_ld_32x32_x64(taddr, r);
    tmem_wait_ld64(r);
}
__device__ __forceinline__ void tmem_load_cols(uint32_t taddr, uint32_t (&r)[32]) {
    tmem_ld_32x32(taddr, r);
    tmem_wait_ld(r);
}
__device__ __forceinline__ void tmem_load_cols(uint32_t taddr, uint32_t (&r)[16]) {
    tmem_ld_32x32_x16(taddr, r);
    tmem_wait_ld16(r);
}

template <int FMT, bool TOKL, int MN>
__global__ void __launch_bounds__(Geo<FMT, TOKL, MN>::NUM_THREADS, 1)
    gemm_tc_kernel(int M, int N, int K, int group, const __half* __restrict__ tok, const float* __restrict__ dxs,
                   const float* __restrict__ zb, const uint8_t* __restrict__ wq,
                   const uint16_t* __restrict__ wscale, const uint16_t* __restrict__ wbias,
                   void* __restrict__ y, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CUtensorMap tm_b, int sc_tma,
                   int bsplit, float* __restrict__ ypart, Epilogue epi) {
    using Gm = Geo<FMT, TOKL, MN>;
    constexpr int S = Gm::S, NS = Gm::NS, NG = Gm::NG, TT = Gm::TT, NW = Gm::NW, CW = Gm::CW;
    constexpr int W_PART = Gm::W_PART, W_BLK = Gm::W_BLK, T_BLK = Gm::T_BLK, DX_BLK = Gm::DX_BLK;
    constexpr int OFF_T = Gm::OFF_T, OFF_DX = Gm::OFF_DX, OFF_C = Gm::OFF_C, OFF_Z = Gm::OFF_Z;
    constexpr int OFF_RAW = Gm::OFF_RAW, OFF_RSC = Gm::OFF_RSC, OFF_RBI = Gm::OFF_RBI;
    constexpr int STAGE_BYTES = Gm::STAGE_BYTES, EPI_WARPS = Gm::EPI_WARPS, PROD_WARP0 = Gm::PROD_WARP0;
    constexpr int LD_COLS = Gm::LD_COLS;
    constexpr int PROD_THREADS = Gm::PROD_WARPS * 32;
    constexpr int MMA_WARP = Gm::MMA_WARP, COPY_WARP = Gm::COPY_WARP;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + NS * STAGE_BYTES);
    volatile uint32_t* abort = &ctrl->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = K >> 5;
    // Split of K over blockIdx.z: this CTA contracts blocks [kb0, kb0 + Bl) (bsplit is a
    // multiple of 8) and, when K is split, writes its partial sums to ypart[z] for the
    // reduction kernel instead of y.
    const int kb0 = blockIdx.z * bsplit;
    const int Bl = min(B, kb0 + bsplit) - kb0;
    const int nstages = (Bl + S - 1) / S;
    // Split of K: partial sums (f32, no epilogue) to ypart[z] for the reduction kernel.
    const bool split = gridDim.z > 1;
    float* __restrict__ yp = split ? ypart + size_t(blockIdx.z) * size_t(M) * size_t(N) : nullptr;
    const int n0 = blockIdx.x * NW;
    const int t = blockIdx.y;
    // Blocks per affine group (2 or 4: group 64 or 128) as a shift: division and modulo by
    // a run-time divisor cost hundreds of cycles on the copy and producer paths.
    const int bsh = (FMT == 1) ? group_shift(group) : 0;
    const int bpm = (1 << bsh) - 1;  // block index & bpm == bpm: last block of its group
    const int G = (FMT == 1) ? K / group : 0;

    auto stage_ptr = [&](int slot) { return smem + slot * STAGE_BYTES; };
    auto bar = [](unsigned long long* p) { return smem_addr(p); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar(&ctrl->raw[s]), 1);
            mbar_init(bar(&ctrl->full[s]), PROD_THREADS + 1);
            mbar_init(bar(&ctrl->empty[s]), EPI_WARPS);
        }
        for (int j = 0; j < NG; ++j) {
            mbar_init(bar(&ctrl->tfull[j]), 1);
            mbar_init(bar(&ctrl->tempty[j]), EPI_WARPS);
        }
        mbar_init(bar(&ctrl->drain), 1);
        ctrl->abort = 0;
        mbar_init_fence();
    }
    if (warp == MMA_WARP) {
        tmem_alloc(smem_addr(&ctrl->tmem_base), Gm::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctrl->tmem_base;
    // Dependent launches may begin their prologue; they wait for this grid's completion
    // before reading its output.
    pdl_launch_dependents();

    if (warp >= PROD_WARP0 && warp < MMA_WARP) {
        // ------------------------------------------------------------ producer
        const int p = threadIdx.x - PROD_WARP0 * 32;  // weight row within the tile
        const int n = n0 + p;
        const bool row_ok = n < N;
        bool range_bad = false;
        // Scales of the stages st, st+1, st+2 when they are not fetched by TMA (their row
        // pitch is not a multiple of 16 bytes): plain loads two stages ahead.
        uint16_t sA[S], sB[S], sC[S], bA[S], bB[S], bC[S];
        auto load_sc = [&](int st, uint16_t (&sv)[S], uint16_t (&bv)[S]) {
#pragma unroll
            for (int k = 0; k < S; ++k) {
                const int b = kb0 + st * S + k;
                sv[k] = 0;
                bv[k] = 0;
                if (!sc_tma && row_ok && st * S + k < Bl) {
                    if (FMT == 0) {
                        sv[k] = ld_nc_u16(wscale + int64_t(n) * B + b);
                    } else {
                        sv[k] = ld_nc_u16(wscale + int64_t(n) * G + (b >> bsh));
                        bv[k] = ld_nc_u16(wbias + int64_t(n) * G + (b >> bsh));
                    }
                }
            }
        };
        load_sc(0, sA, bA);
        load_sc(1, sB, bB);
        load_sc(2, sC, bC);
        for (int st = 0; st < nstages; ++st) {
            const int slot = st % NS;
            // The packed weights of this stage are in shared memory (the copy warp took the
            // slot from the epilogue before fetching them).
            if (!bounded_wait_warp(bar(&ctrl->raw[slot]), (st / NS) & 1, abort)) break;
            uint8_t* sp = stage_ptr(slot);
            const int sb0 = kb0 + st * S;  // first block of the stage
            const int e0 = (FMT == 0) ? sb0 & ~7 : (sb0 >> bsh) & ~7;  // first scale of the TMA box
#pragma unroll
            for (int k = 0; k < S; ++k) {
                const int b = sb0 + k;
                uint4 wv = make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);  // codes 8: zero
                uint32_t sb = 0, bb = 0;
                if (st * S + k < Bl) {
                    wv = *reinterpret_cast<const uint4*>(sp + OFF_RAW + k * NW * 16 + p * 16);
                    if (sc_tma) {
                        const int e = (FMT == 0) ? b : b >> bsh;
                        sb = reinterpret_cast<const uint16_t*>(sp + OFF_RSC + p * 16)[e - e0];
                        if (FMT == 1) bb = reinterpret_cast<const uint16_t*>(sp + OFF_RBI + p * 16)[e - e0];
                    } else {
                        sb = sA[k];
                        bb = bA[k];
                    }
                }
                const uint32_t w[4] = {wv.x, wv.y, wv.z, wv.w};
                uint8_t* dst = sp + k * W_BLK + (p >> 3) * 512 + (p & 7) * 16;
                if (FMT == 0) {
                    range_bad |= (sb & 0x7FF8u) > 0x6950u;  // d_hi > 2720 (24 d_hi > 65504), inf or nan
                    const __half dh = __ushort_as_half(uint16_t(sb & 0xFFF8u));
                    const __half dl = __hsub(__ushort_as_half(uint16_t(sb)), dh);  // exact
                    const uint32_t h2 = pair_of(__hmul(dh, __float2half(2.0f)));
                    const uint32_t h24 = pair_of(__hmul(dh, __float2half(-24.0f)));
                    const uint32_t l2 = pair_of(__hmul(dl, __float2half(2.0f)));
                    const uint32_t l24 = pair_of(__hmul(dl, __float2half(-24.0f)));
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t r[4];
                        codes_raw(w[c], r);
                        *reinterpret_cast<uint4*>(dst + c * 128) =
                            make_uint4(scaled_codes(r[0], h2, h24), scaled_codes(r[1], h2, h24),
                                       scaled_codes(r[2], h2, h24), scaled_codes(r[3], h2, h24));
                        *reinterpret_cast<uint4*>(dst + W_PART + c * 128) =
                            make_uint4(scaled_codes(r[0], l2, l24), scaled_codes(r[1], l2, l24),
                                       scaled_codes(r[2], l2, l24), scaled_codes(r[3], l2, l24));
                    }
                } else {
                    const float sf = __bfloat162float(__ushort_as_bfloat16(uint16_t(sb)));
                    const float af = fabsf(sf);
                    range_bad |= !(af <= 2720.0f) || (af != 0.0f && af < 7.62939453125e-06f);  // 2^-17
                    const __half sh = __float2half_rn(sf);  // exact in range
                    const uint32_t s2 = pair_of(__hmul(sh, __float2half(2.0f)));
                    const uint32_t s24 = pair_of(__hmul(sh, __float2half(-24.0f)));
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t r[4];
                        codes_raw(w[c], r);
                        *reinterpret_cast<uint4*>(dst + c * 128) =
                            make_uint4(scaled_codes(r[0], s2, s24), scaled_codes(r[1], s2, s24),
                                       scaled_codes(r[2], s2, s24), scaled_codes(r[3], s2, s24));
                    }
                    if ((b & bpm) == bpm) {  // last block of a group: its bias factor b + 8s
                        const float bf = __bfloat162float(__ushort_as_bfloat16(uint16_t(bb)));
                        reinterpret_cast<float*>(sp + OFF_C)[k * NW + p] = __fadd_rn(bf, __fmul_rn(8.0f, sf));
                    }
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(bar(&ctrl->full[slot]));
            if (!sc_tma) {
#pragma unroll
                for (int k = 0; k < S; ++k) {
                    sA[k] = sB[k];
                    sB[k] = sC[k];
                    bA[k] = bB[k];
                    bB[k] = bC[k];
                }
                load_sc(st + 3, sC, bC);
            }
        }
        if (range_bad) atomicOr(&g_device_status, kDevErrRange);
    } else if (warp == COPY_WARP) {
        // ------------------------------------------------------------ bulk copies
        // The whole warp runs the loop (uniform control flow); one elected lane issues.
        const bool leader = elect_one();
        pdl_wait_primary();  // the token operands are written by the preceding kernel
        int issued = 0;
        for (int st = 0; st < nstages; ++st) {
            const int slot = st % NS;
            if (!bounded_wait_warp(bar(&ctrl->empty[slot]), ((st / NS) & 1) ^ 1, abort)) break;
            const int b0 = kb0 + st * S;
            const int nb = min(S, kb0 + Bl - b0);
            if (leader) {
                int nz = 0;  // affine: group ends in this stage (each brings its Z row)
                if (FMT == 1)
                    for (int k = 0; k < nb; ++k) nz += ((b0 + k) & bpm) == bpm;
                uint8_t* sp = stage_ptr(slot);
                // packed weights of the stage (codes, and scales when their pitch allows TMA)
                const uint32_t rb = bar(&ctrl->raw[slot]);
                const int e0 = (FMT == 0) ? b0 & ~7 : (b0 >> bsh) & ~7;
                mbar_arrive_expect_tx(rb, uint32_t(nb * NW * 16 + (sc_tma ? NW * 16 * (FMT == 1 ? 2 : 1) : 0)));
                for (int k = 0; k < nb; ++k)
                    tma_load_2d<1>(smem_addr(sp + OFF_RAW + k * NW * 16), &tm_q, (b0 + k) * 16, n0, rb);
                if (sc_tma) {
                    tma_load_2d<2>(smem_addr(sp + OFF_RSC), &tm_s, e0, n0, rb);
                    if (FMT == 1) tma_load_2d<2>(smem_addr(sp + OFF_RBI), &tm_b, e0, n0, rb);
                }
                const uint32_t fb = bar(&ctrl->full[slot]);
                mbar_arrive_expect_tx(fb, uint32_t(nb * (T_BLK + DX_BLK) + nz * TT * 4));
                bulk_g2s(smem_addr(sp + OFF_T), reinterpret_cast<const uint8_t*>(tok) + (int64_t(t) * B + b0) * T_BLK,
                         uint32_t(nb * T_BLK), fb);
                bulk_g2s(smem_addr(sp + OFF_DX), dxs + (int64_t(t) * B + b0) * TT, uint32_t(nb * DX_BLK), fb);
                if (FMT == 1) {
                    for (int k = 0; k < nb; ++k)
                        if (((b0 + k) & bpm) == bpm)
                            bulk_g2s(smem_addr(sp + OFF_Z + k * TT * 4), zb + (int64_t(t) * G + ((b0 + k) >> bsh)) * TT,
                                     TT * 4, fb);
                }
            }
            __syncwarp();
            issued = st + 1;
        }
        // Let every copy this warp issued land before the CTA can exit. On the normal path
        // the stage barriers complete (the MMA warp has consumed every stage). After an
        // abort the producer may never arrive, so each wait is capped at 200 us, far longer
        // than a few-KB copy takes to land.
        for (int st = max(0, issued - NS); st < issued; ++st) {
            drain_wait_warp(bar(&ctrl->raw[st % NS]), (st / NS) & 1, 200000ull);
            drain_wait_warp(bar(&ctrl->full[st % NS]), (st / NS) & 1, 200000ull);
        }
    } else if (warp == MMA_WARP) {
        // ------------------------------------------------------------ MMA issue
        // Uniform loop over the warp; the elected lane issues every MMA and commit (a
        // commit tracks the MMAs of the thread that issues it).
        const bool leader = elect_one();
        const uint32_t smem0 = smem_addr(smem);
        for (int st = 0; st < nstages; ++st) {
            const int slot = st % NS, g = st % NG;
            if (!bounded_wait_warp(bar(&ctrl->full[slot]), (st / NS) & 1, abort)) break;
            if (!bounded_wait_warp(bar(&ctrl->tempty[g]), ((st / NG) & 1) ^ 1, abort)) break;
            tc_fence_after();
            if (leader) {
                // Straight-line issue of all S blocks: a branch between two MMAs lets the
                // issue stall until the earlier one completes. In a short last stage the
                // blocks past the end fill TMEM tiles that the epilogue never reads.
#pragma unroll
                for (int k = 0; k < S; ++k) {
                    const uint32_t w_addr = smem0 + uint32_t(slot * STAGE_BYTES + k * W_BLK);
                    const uint32_t t_addr = smem0 + uint32_t(slot * STAGE_BYTES + OFF_T + k * T_BLK);
                    const uint32_t d = tmem_base + uint32_t((g * S + k) * MN);
#pragma unroll
                    for (int part = 0; part < Gm::WP; ++part) {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint64_t wd = smem_desc_kmajor(w_addr + part * W_PART + h * 256, LBO, SBO);
                            const uint64_t td = smem_desc_kmajor(t_addr + h * 256, LBO, SBO);
                            if (TOKL)
                                tc_mma_f16(d, td, wd, Gm::IDESC, (part | h) != 0);
                            else
                                tc_mma_f16(d, wd, td, Gm::IDESC, (part | h) != 0);
                        }
                    }
                }
                tc_commit(bar(&ctrl->tfull[g]));  // the stage's accumulators are complete and its operands read
            }
            __syncwarp();
        }
        // Wait until every MMA (and the barrier arrivals their commits trigger) is done
        // before TMEM and shared memory are released.
        uint32_t local_abort = 0;
        if (leader) tc_commit(bar(&ctrl->drain));
        __syncwarp();
        bounded_wait_warp(bar(&ctrl->drain), 0, &local_abort);
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;             // TMEM lane quarter
        const int c0 = (warp >> 2) * CW;    // first TMEM column of this warp
        const int r = q * 32 + lane;        // this thread's TMEM lane: token (TOKL) or weight row
        // f32 accumulators, one per column. Scalar FMAs: the packed f32x2 form does the same
        // work on the FMA pipe and would need its operands re-paired after each tensor-
        // memory load, which costs more issue slots than it saves.
        float acc[CW];
#pragma unroll
        for (int j = 0; j < CW; ++j) acc[j] = 0.0f;
        const uint32_t lane_base = tmem_base + (uint32_t(q * 32) << 16);
        for (int st = 0; st < nstages; ++st) {
            const int slot = st % NS, g = st % NG;
            const int nb = min(S, Bl - st * S);
            if (!bounded_wait_warp(bar(&ctrl->tfull[g]), (st / NG) & 1, abort)) break;
            tc_fence_after();
            const uint8_t* sp = stage_ptr(slot);
            bool released = false;
#pragma unroll
            for (int k = 0; k < S; ++k) {
                if (k >= nb) break;
                const int i = kb0 + st * S + k;
                const bool last = (k == nb - 1);
                const float* dxk = reinterpret_cast<const float*>(sp + OFF_DX) + k * TT;
                const bool group_end = (FMT == 1) && ((i & bpm) == bpm);
                const float dxr = TOKL ? dxk[r] : 0.0f;
#pragma unroll
                for (int h0 = 0; h0 < CW; h0 += LD_COLS) {
                    uint32_t pr[LD_COLS];
                    tmem_load_cols(lane_base + uint32_t((g * S + k) * MN + c0 + h0), pr);
                    if (last && h0 + LD_COLS == CW) {  // the group's tiles are all in registers: free it
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(&ctrl->tempty[g]));
                    }
                    if (TOKL) {
#pragma unroll
                        for (int j = 0; j < LD_COLS; ++j) acc[h0 + j] = fmaf(__uint_as_float(pr[j]), dxr, acc[h0 + j]);
                    } else {
#pragma unroll
                        for (int j = 0; j < LD_COLS; j += 4) {
                            const float4 dv = *reinterpret_cast<const float4*>(dxk + c0 + h0 + j);
                            acc[h0 + j] = fmaf(__uint_as_float(pr[j]), dv.x, acc[h0 + j]);
                            acc[h0 + j + 1] = fmaf(__uint_as_float(pr[j + 1]), dv.y, acc[h0 + j + 1]);
                            acc[h0 + j + 2] = fmaf(__uint_as_float(pr[j + 2]), dv.z, acc[h0 + j + 2]);
                            acc[h0 + j + 3] = fmaf(__uint_as_float(pr[j + 3]), dv.w, acc[h0 + j + 3]);
                        }
                    }
                }
                if (group_end) {  // last block of a group: add (b + 8s) * Z
                    const float* cs = reinterpret_cast<const float*>(sp + OFF_C) + k * NW;
                    const float* zs = reinterpret_cast<const float*>(sp + OFF_Z) + k * TT;
                    if (TOKL) {
                        const float z = zs[r];
#pragma unroll
                        for (int j = 0; j < CW; j += 4) {
                            const float4 cv = *reinterpret_cast<const float4*>(cs + c0 + j);
                            acc[j] = fmaf(cv.x, z, acc[j]);
                            acc[j + 1] = fmaf(cv.y, z, acc[j + 1]);
                            acc[j + 2] = fmaf(cv.z, z, acc[j + 2]);
                            acc[j + 3] = fmaf(cv.w, z, acc[j + 3]);
                        }
                    } else {
                        const float c = cs[r];
#pragma unroll
                        for (int j = 0; j < CW; j += 4) {
                            const float4 zv = *reinterpret_cast<const float4*>(zs + c0 + j);
                            acc[j] = fmaf(zv.x, c, acc[j]);
                            acc[j + 1] = fmaf(zv.y, c, acc[j + 1]);
                            acc[j + 2] = fmaf(zv.z, c, acc[j + 2]);
                            acc[j + 3] = fmaf(zv.w, c, acc[j + 3]);
                        }
                    }
                }
            }
            if (!released) {  // the values read from the stage were consumed above
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(&ctrl->empty[slot]));
            }
        }
        if (!*abort) {
            if (TOKL) {
                const int m = t * TT + r;
                const int nb = n0 + c0;
                if (m < M) {
                    const int64_t row = int64_t(m) * N;
                    // Plain f32 stores for split partials and calls without an epilogue; the
                    // epilogue's per-element work only when one is given.
                    float* yf = split ? yp : ((epi.bias || epi.out_bf16) ? nullptr : reinterpret_cast<float*>(y));
                    if (yf) {
                        if ((N & 3) == 0 && nb + CW <= N) {
#pragma unroll
                            for (int j = 0; j < CW; j += 4)
                                *reinterpret_cast<float4*>(yf + row + nb + j) = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
                        } else {
#pragma unroll
                            for (int j = 0; j < CW; ++j)
                                if (nb + j < N) yf[row + nb + j] = acc[j];
                        }
                    } else if ((N & 3) == 0 && nb + CW <= N) {
#pragma unroll
                        for (int j = 0; j < CW; j += 4)
                            epi_store4(y, row + nb + j, nb + j, acc[j], acc[j + 1], acc[j + 2], acc[j + 3], epi);
                    } else {
#pragma unroll
                        for (int j = 0; j < CW; ++j)
                            if (nb + j < N) epi_store(y, row + nb + j, nb + j, acc[j], epi);
                    }
                }
            } else {
                const int n = n0 + r;
                float* yf = split ? yp : ((epi.bias || epi.out_bf16) ? nullptr : reinterpret_cast<float*>(y));
                if (n < N && yf) {
#pragma unroll
                    for (int j = 0; j < CW; ++j) {
                        const int m = t * TT + c0 + j;
                        if (m < M) yf[int64_t(m) * N + n] = acc[j];
                    }
                } else if (n < N) {
#pragma unroll
                    for (int j = 0; j < CW; ++j) {
                        const int m = t * TT + c0 + j;
                        if (m < M) epi_store(y, int64_t(m) * N + n, n, acc[j], epi);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Gm::TMEM_COLS);
    }
}

// Sum of the K-split partial outputs in split order: y = part[0] + part[1] + ... (the
// same order on every call, so results do not depend on scheduling). n4 = M*N/4.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float4* __restrict__ part, int ks, int64_t n4,
                                                             int N, void* __restrict__ y, Epilogue epi) {
    pdl_wait_primary();  // the partials are written by the preceding GEMM
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += int64_t(gridDim.x) * blockDim.x) {
        // splits in order, in groups of 16 whose sums are added in order (at most 15 + ks/16
        // roundings in any output's chain)
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int z0 = 0; z0 < ks; z0 += 16) {
            float4 g = part[int64_t(z0) * n4 + i];
            for (int z = z0 + 1; z < ks && z < z0 + 16; ++z) {
                const float4 b = part[int64_t(z) * n4 + i];
                g.x = __fadd_rn(g.x, b.x);
                g.y = __fadd_rn(g.y, b.y);
                g.z = __fadd_rn(g.z, b.z);
                g.w = __fadd_rn(g.w, b.w);
            }
            if (z0 == 0) {
                a = g;
            } else {
                a.x = __fadd_rn(a.x, g.x);
                a.y = __fadd_rn(a.y, g.y);
                a.z = __fadd_rn(a.z, g.z);
                a.w = __fadd_rn(a.w, g.w);
            }
        }
        if (!epi.bias && !epi.out_bf16) {
            reinterpret_cast<float4*>(y)[i] = a;
        } else if ((N & 3) == 0) {  // the four outputs lie in one row
            epi_store4(y, 4 * i, int((4 * i) % N), a.x, a.y, a.z, a.w, epi);
        } else {
            const float v[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) epi_store(y, 4 * i + j, int((4 * i + j) % N), v[j], epi);
        }
    }
}

// The same reduction element by element, for M * N not a multiple of 4 (partial z of
// output i at part[z * n + i]).
__global__ void __launch_bounds__(256) splitk_reduce_scalar_kernel(const float* __restrict__ part, int ks, int64_t n,
                                                                    int N, void* __restrict__ y, Epilogue epi) {
    pdl_wait_primary();  // the partials are written by the preceding GEMM
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
        float a = 0.0f;
        for (int z0 = 0; z0 < ks; z0 += 16) {  // in groups of 16, as splitk_reduce_kernel
            float g = part[int64_t(z0) * n + i];
            for (int z = z0 + 1; z < ks && z < z0 + 16; ++z) g = __fadd_rn(g, part[int64_t(z) * n + i]);
            a = (z0 == 0) ? g : __fadd_rn(a, g);
        }
        epi_store(y, i, int(i % N), a, epi);
    }
}

}  // namespace tc
}  // namespace w4a8
