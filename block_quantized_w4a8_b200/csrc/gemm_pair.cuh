// Tensor-core path on CTA pairs (cta_group::2) for token tiles on the TMEM lanes.
//
// Same arithmetic as the token-lane instantiation of gemm_tc_kernel (exact fp16 weight
// operand with the weight scale folded in, one f32 FMA per output and block for the
// activation scale; tract PR #2432, "The kernel": a separate rescale per 32-block), but
// two CTAs of a cluster share each weight tile: the pair's MMA is 256 tokens x 128 weight
// rows, the even CTA holding tokens 0..127 of the pair and weight rows 0..63, the odd CTA
// tokens 128..255 and weight rows 64..127. Each CTA therefore expands and stores only half
// of the weight rows for the same MMA work, which halves the shared-memory stores that
// bound the single-CTA kernel (the expanded operand is 128 B per row and block), while the
// epilogue is unchanged: each CTA's tensor memory holds its 128 tokens x all 128 rows.
//
// Affine weights: the group bias term (b + 8s) * sum(q_x) goes through the tensor core as
// one more K = 16 MMA per block into the block's accumulator, ahead of the per-block
// activation scale: the token operand carries the block's two 16-element code sums
// [S1, S2, S1/2^11, S2/2^11] (exact fp16, written by the quantisation kernel), the weight
// operand the row's C = b + 8s as [C_hi, C_hi, C_lo, C_lo] with C_hi = fp16(C) and
// C_lo = fp16((C - C_hi) * 2^11), so that C_hi + C_lo / 2^11 carries 22 bits of C. The
// second 8-element K chunk of both operands is a zero region of shared memory. The
// epilogue is then the same single FMA per output and block as for Q4_0.
//
// Affine 6- and 8-bit codes (FMT 3 and 2) read their codes as a little-endian bit stream
// (one TMA box of both blocks of a stage per row) and widen each code q to the fp16 value
// 1024 + q with one byte permute per pair. The group scale s is split into two exact
// parts s_hi + s_lo (its top 4 and low 4 significant bits for 8-bit codes, 5 and 3 for
// 6-bit) and each part gives (1024 + q) * s_part - (1024 + c) * s_part = (q - c) * s_part
// (c = 128 or 32) in one fused multiply-add, rounded once to an exactly representable
// value, so the weight operand has two parts as for Q4_0. The bias column holds
// C = b + c*s. Exact for s = 0 or 2^-17 <= |s| <= 32.
//
// Roles per CTA (448 threads): 8 epilogue warps, 4 producer warps (one thread per (row of
// the CTA's half, block of the stage), two stages at a time), one MMA warp, one bulk-copy
// warp. Only the even
// CTA's MMA warp issues MMAs; the odd CTA's MMA warp forwards its stage-ready signal to the
// even CTA (one remote arrive per stage). The even CTA's MMA warp waits for its own stage,
// the forwarded one and both CTAs' epilogues (TMEM groups), issues the stage's MMAs and
// one commit that arrives on both CTAs' barriers. All waits are bounded as in the
// single-CTA kernel; both CTAs meet at a cluster barrier before the pair's tensor memory
// is freed, so neither exits while the other or the tensor core may still touch it.
#pragma once

#include "gemm_tc.cuh"

namespace w4a8 {
namespace tc {

template <int FMT>
struct PairGeo {
    static constexpr int TT = 128;                  // tokens per CTA (256 per pair)
    static constexpr int NWT = 128;                 // weight rows per pair tile (the MMA's N)
    static constexpr int NWH = NWT / 2;             // weight rows each CTA expands and stages
    static constexpr int MN = NWT;                  // TMEM columns per accumulator tile
    static constexpr bool AFF = FMT >= 1;           // affine: group scale and bias, bias MMA
    static constexpr bool WIDE = FMT >= 2;          // 8-bit (FMT 2) or 6-bit (FMT 3) codes
    static constexpr int BITS = (FMT == 2) ? 8 : (FMT == 3 ? 6 : 4);
    static constexpr int BPB = 4 * BITS;            // code bytes per row and block
    static constexpr int WORDS = BPB / 4;
    static constexpr int WP = (FMT == 1) ? 1 : 2;   // weight operand parts (hi, lo)
    static constexpr int W_PART = NWH * 64;
    static constexpr int W_BLK = W_PART * WP;
    static constexpr int T_BLK = TT * 64;
    static constexpr int DX_BLK = TT * 4;
    static constexpr int S = 2;                     // quant blocks per stage (one commit)
    static constexpr int OFF_T = S * W_BLK;
    static constexpr int OFF_DX = OFF_T + S * T_BLK;
    static constexpr int OFF_XT = align_up(OFF_DX + S * DX_BLK, 128);           // affine: token code sums
    static constexpr int OFF_XW = OFF_XT + (AFF ? S * TT * 16 : 0);             // affine: C parts, own half
    static constexpr int OFF_RAW = align_up(OFF_XW + (AFF ? S * NWH * 16 : 0), 128);  // codes, own half
    static constexpr int OFF_RSC = OFF_RAW + S * NWH * BPB;                     // scales, all 128 rows
    static constexpr int OFF_RBI = OFF_RSC + NWT * 16;                          // affine biases
    static constexpr int STAGE_BYTES = align_up(OFF_RBI + (AFF ? NWT * 16 : 0), 1024);
    static constexpr int ZERO_BYTES = AFF ? TT * 16 : 0;  // zero K chunk of the bias MMA
    static constexpr int NS = cmin(8, (SMEM_LIMIT - CTRL_BYTES - ZERO_BYTES - 1024) / STAGE_BYTES);
    static constexpr int OFF_ZERO = NS * STAGE_BYTES + CTRL_BYTES;
    static constexpr int SMEM_BYTES = OFF_ZERO + ZERO_BYTES + 1024;
    static constexpr int NBUF = 512 / MN;           // accumulator tiles (one per block)
    static constexpr int NG = NBUF / S;             // TMEM groups: stage st uses group st % NG
    static constexpr int TMEM_COLS = 512;
    static constexpr int CW = 64;                   // columns per epilogue warp
    static constexpr int EPI_WARPS = 4 * MN / CW;
    static constexpr int PROD_WARPS = NWH * S / 32;
    static constexpr int PROD_WARP0 = EPI_WARPS;
    static constexpr int MMA_WARP = PROD_WARP0 + PROD_WARPS;
    static constexpr int COPY_WARP = MMA_WARP + 1;
    static constexpr int NUM_THREADS = (COPY_WARP + 1) * 32;
    static constexpr int LD_COLS = 32;              // TMEM columns per load (registers: 64 accumulators + 32)
    static constexpr uint32_t IDESC = idesc_f16_f32(256, NWT);
    static_assert(NS >= 3 && NS <= 8, "pipeline depth");
    static_assert(NG == 2 && NBUF % S == 0, "TMEM groups");
    static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory");
    static_assert(OFF_T % 128 == 0 && OFF_DX % 16 == 0 && OFF_XT % 128 == 0 && OFF_RSC % 16 == 0, "alignment");
};

struct PairCtrl {
    unsigned long long raw[MAX_NS];     // TMA of the packed weights (1 arrival + bytes)
    unsigned long long full[MAX_NS];    // producer warps + bulk copies (1 arrival + bytes)
    unsigned long long empty[MAX_NS];   // one arrival per epilogue warp of this CTA
    unsigned long long pfull[MAX_NS];   // even CTA: the odd CTA's stage is ready (1 remote arrival)
    unsigned long long tfull[MAX_NG];   // pair commit, once per stage, on both CTAs
    unsigned long long tempty[MAX_NG];  // even CTA: one arrival per epilogue warp of both CTAs
    unsigned long long drain;           // final pair commit, on both CTAs
    uint32_t tmem_base;
    uint32_t abort;
};
static_assert(sizeof(PairCtrl) <= CTRL_BYTES, "control block");

// Grid: x = token tile (pairs of consecutive tiles form a cluster), y = 128-row weight
// tile, z = split of K. The scale (and affine bias) tensor maps have boxes of 128 rows x 8
// entries, the code map boxes of 64 rows x 16 bytes; both require the rows' pitch to be a
// multiple of 16 bytes, which the host checks before choosing this kernel.
template <int FMT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairGeo<FMT>::NUM_THREADS, 1)
    gemm_pair_kernel(int M, int N, int K, int group, const __half* __restrict__ tok, const float* __restrict__ dxs,
                     const uint4* __restrict__ xsum, void* __restrict__ y, const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CUtensorMap tm_b, int bsplit,
                     float* __restrict__ ypart, Epilogue epi) {
    using Gm = PairGeo<FMT>;
    constexpr int S = Gm::S, NS = Gm::NS, NG = Gm::NG, TT = Gm::TT, NWT = Gm::NWT, NWH = Gm::NWH;
    constexpr int MN = Gm::MN, CW = Gm::CW, W_PART = Gm::W_PART, W_BLK = Gm::W_BLK, T_BLK = Gm::T_BLK;
    constexpr int DX_BLK = Gm::DX_BLK, OFF_T = Gm::OFF_T, OFF_DX = Gm::OFF_DX, OFF_XT = Gm::OFF_XT;
    constexpr int OFF_XW = Gm::OFF_XW, OFF_RAW = Gm::OFF_RAW, OFF_RSC = Gm::OFF_RSC, OFF_RBI = Gm::OFF_RBI;
    constexpr int STAGE_BYTES = Gm::STAGE_BYTES, EPI_WARPS = Gm::EPI_WARPS, PROD_WARP0 = Gm::PROD_WARP0;
    constexpr int PROD_WARPS = Gm::PROD_WARPS, MMA_WARP = Gm::MMA_WARP, COPY_WARP = Gm::COPY_WARP;
    constexpr int LD_COLS = Gm::LD_COLS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    PairCtrl* ctrl = reinterpret_cast<PairCtrl*>(smem + NS * STAGE_BYTES);
    volatile uint32_t* abort = &ctrl->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0: even CTA (issues the MMAs), 1: odd CTA
    const int B = K >> 5;
    const int kb0 = blockIdx.z * bsplit;  // this pair contracts blocks [kb0, kb0 + Bl)
    const int Bl = min(B, kb0 + bsplit) - kb0;
    const int nstages = (Bl + S - 1) / S;
    // Split of K: partial sums (f32, no epilogue) to ypart[z] for the reduction kernel.
    const bool split = gridDim.z > 1;
    float* __restrict__ yp = split ? ypart + size_t(blockIdx.z) * size_t(M) * size_t(N) : nullptr;
    const int t = blockIdx.x;                // token tile
    const int n0 = blockIdx.y * NWT;         // the pair's weight rows
    const int nh0 = n0 + int(rank) * NWH;    // the rows this CTA stages
    // Blocks per affine group (2 or 4: group 64 or 128) as a shift: division and modulo by
    // a run-time divisor cost hundreds of cycles on the copy and producer paths.
    const int bsh = Gm::AFF ? group_shift(group) : 0;

    auto stage_ptr = [&](int slot) { return smem + slot * STAGE_BYTES; };
    auto bar = [](unsigned long long* p) { return smem_addr(p); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar(&ctrl->raw[s]), 1);
            mbar_init(bar(&ctrl->full[s]), PROD_WARPS + 1);
            mbar_init(bar(&ctrl->empty[s]), EPI_WARPS);
            mbar_init(bar(&ctrl->pfull[s]), 1);
        }
        for (int j = 0; j < NG; ++j) {
            mbar_init(bar(&ctrl->tfull[j]), 1);
            mbar_init(bar(&ctrl->tempty[j]), 2 * EPI_WARPS);
        }
        mbar_init(bar(&ctrl->drain), 1);
        ctrl->abort = 0;
        mbar_init_fence();
    }
    if (Gm::AFF && threadIdx.x < Gm::ZERO_BYTES / 16) {
        reinterpret_cast<uint4*>(smem + Gm::OFF_ZERO)[threadIdx.x] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();  // read by the tensor core
    }
    if (warp == MMA_WARP) {
        tmem_alloc_pair(smem_addr(&ctrl->tmem_base), Gm::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised, tensor memory allocated
    tc_fence_after();
    const uint32_t tmem_base = ctrl->tmem_base;
    pdl_launch_dependents();

    if (warp >= PROD_WARP0 && warp < MMA_WARP) {
        // ------------------------------------------------------------ producer
        // Two stages per iteration: their loads, expansions and stores interleave, and one
        // proxy fence covers both (a single row-block per thread leaves the warp waiting on
        // one dependent chain at a time).
        const int tid = threadIdx.x - PROD_WARP0 * 32;
        const int p = tid % NWH;   // weight row within this CTA's half
        const int kq = tid / NWH;  // block of the stage this thread expands
        bool range_bad = false;
        // The packed codes and scale of this thread's (row, block) task, read from the stage
        // before any expanded value is stored (the stores of one stage could alias the next
        // stage's loads, so the loads of both stages are issued first).
        struct Raw {
            uint32_t w[Gm::WORDS];  // the codes of this row and block
            uint32_t sb;
            uint32_t bb;  // affine: the group's bias
        };
        auto load_raw = [&](int st) {
            Raw rw;
#pragma unroll
            for (int i = 0; i < Gm::WORDS; ++i) rw.w[i] = 0u;
            rw.sb = 0u;
            rw.bb = 0u;
            const uint8_t* sp = stage_ptr(st % NS);
            const int sb0 = kb0 + st * S;
            const int e0 = (FMT == 0) ? sb0 & ~7 : ((sb0 >> bsh)) & ~7;  // first scale of the TMA box
            if (st * S + kq < Bl) {
                const int b = sb0 + kq;
                const int e = (FMT == 0) ? b : (b >> bsh);
                if (Gm::BITS == 4) {  // one 16-byte box row per block
                    const uint4 v = *reinterpret_cast<const uint4*>(sp + OFF_RAW + kq * NWH * 16 + p * 16);
                    rw.w[0] = v.x; rw.w[1] = v.y; rw.w[2] = v.z; rw.w[3] = v.w;
                } else if (Gm::BITS == 8) {  // one box of both blocks: row p at p * 64
                    const uint4* v = reinterpret_cast<const uint4*>(sp + OFF_RAW + p * (S * 32) + kq * 32);
                    const uint4 a = v[0], c = v[1];
                    rw.w[0] = a.x; rw.w[1] = a.y; rw.w[2] = a.z; rw.w[3] = a.w;
                    rw.w[4] = c.x; rw.w[5] = c.y; rw.w[6] = c.z; rw.w[7] = c.w;
                } else {  // 6-bit: row p at p * 48, 24 bytes per block
                    const uint2* v = reinterpret_cast<const uint2*>(sp + OFF_RAW + p * (S * 24) + kq * 24);
#pragma unroll
                    for (int i = 0; i < 3; ++i) {
                        const uint2 a = v[i];
                        rw.w[2 * i] = a.x;
                        rw.w[2 * i + 1] = a.y;
                    }
                }
                rw.sb = reinterpret_cast<const uint16_t*>(sp + OFF_RSC + (int(rank) * NWH + p) * 16)[e - e0];
                if (Gm::AFF) rw.bb = reinterpret_cast<const uint16_t*>(sp + OFF_RBI + (int(rank) * NWH + p) * 16)[e - e0];
            }
            return rw;
        };
        auto expand = [&](int st, const Raw& rw) {
            uint8_t* sp = stage_ptr(st % NS);
            if (st * S + kq < Bl) {
                const uint32_t sb = rw.sb;
                const uint32_t* w = rw.w;
                uint8_t* dst = sp + kq * W_BLK + (p >> 3) * 512 + (p & 7) * 16;
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
                } else if (Gm::WIDE) {
                    const float sf = __bfloat162float(__ushort_as_bfloat16(uint16_t(sb)));
                    const float af = fabsf(sf);
                    range_bad |= !(af <= 32.0f) || (af != 0.0f && af < 7.62939453125e-06f);  // 2^-17
                    // s = s_hi + s_lo: the top 4 (8-bit) or 5 (6-bit) significant bits of the
                    // bf16 scale, and the rest (exact in f32 and in fp16 within the range)
                    const uint16_t hib = uint16_t(sb) & uint16_t(Gm::BITS == 8 ? 0xFFF0u : 0xFFF8u);
                    const float shf = __bfloat162float(__ushort_as_bfloat16(hib));
                    const __half sh = __float2half_rn(shf);
                    const __half sl = __float2half_rn(__fsub_rn(sf, shf));
                    const __half off = __float2half(Gm::BITS == 8 ? -1152.0f : -1056.0f);  // -(1024 + c)
                    const uint32_t h1 = pair_of(sh), hA = pair_of(__hmul(sh, off));
                    const uint32_t l1 = pair_of(sl), lA = pair_of(__hmul(sl, off));
                    uint32_t cb[8];  // codes 4i..4i+3 as bytes
                    if (Gm::BITS == 8) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) cb[i] = w[i];
                    } else {
                        uint32_t v[8];  // 24-bit groups of four codes at bit 24i
                        v[0] = w[0];
                        v[1] = __funnelshift_r(w[0], w[1], 24);
                        v[2] = __funnelshift_r(w[1], w[2], 16);
                        v[3] = w[2] >> 8;
                        v[4] = w[3];
                        v[5] = __funnelshift_r(w[3], w[4], 24);
                        v[6] = __funnelshift_r(w[4], w[5], 16);
                        v[7] = w[5] >> 8;
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            cb[i] = (v[i] & 0x3Fu) | ((v[i] << 2) & 0x3F00u) | ((v[i] << 4) & 0x3F0000u) |
                                    ((v[i] << 6) & 0x3F000000u);
                    }
#pragma unroll
                    for (int c = 0; c < 4; ++c) {  // segment c: codes 8c..8c+7 as fp16 1024 + q
                        const uint32_t r[4] = {__byte_perm(cb[2 * c], 0x64646464u, 0x4140),
                                               __byte_perm(cb[2 * c], 0x64646464u, 0x4342),
                                               __byte_perm(cb[2 * c + 1], 0x64646464u, 0x4140),
                                               __byte_perm(cb[2 * c + 1], 0x64646464u, 0x4342)};
                        *reinterpret_cast<uint4*>(dst + c * 128) =
                            make_uint4(scaled_codes(r[0], h1, hA), scaled_codes(r[1], h1, hA),
                                       scaled_codes(r[2], h1, hA), scaled_codes(r[3], h1, hA));
                        *reinterpret_cast<uint4*>(dst + W_PART + c * 128) =
                            make_uint4(scaled_codes(r[0], l1, lA), scaled_codes(r[1], l1, lA),
                                       scaled_codes(r[2], l1, lA), scaled_codes(r[3], l1, lA));
                    }
                    const float bf = __bfloat162float(__ushort_as_bfloat16(uint16_t(rw.bb)));
                    const float cf = __fadd_rn(bf, __fmul_rn(Gm::BITS == 8 ? 128.0f : 32.0f, sf));  // b + c*s
                    range_bad |= !(fabsf(cf) <= 65504.0f);
                    const __half ch = __float2half_rn(cf);
                    const __half cl = __float2half_rn(__fmul_rn(__fsub_rn(cf, __half2float(ch)), 2048.0f));
                    *reinterpret_cast<uint4*>(sp + OFF_XW + kq * NWH * 16 + p * 16) =
                        make_uint4(pair_of(ch), pair_of(cl), 0u, 0u);
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
                    // The bias MMA's weight column for this row and block: C = b + 8s in two
                    // fp16 parts (C - C_hi is exact in f32; the scaled low part stays normal
                    // down to |C| = 2^-14).
                    const float bf = __bfloat162float(__ushort_as_bfloat16(uint16_t(rw.bb)));
                    const float cf = __fadd_rn(bf, __fmul_rn(8.0f, sf));
                    range_bad |= !(fabsf(cf) <= 65504.0f);
                    const __half ch = __float2half_rn(cf);
                    const __half cl = __float2half_rn(__fmul_rn(__fsub_rn(cf, __half2float(ch)), 2048.0f));
                    *reinterpret_cast<uint4*>(sp + OFF_XW + kq * NWH * 16 + p * 16) =
                        make_uint4(pair_of(ch), pair_of(cl), 0u, 0u);
                }
            }
        };
        for (int st = 0; st < nstages; st += 2) {
            const bool two = st + 1 < nstages;  // warp-uniform
            if (!bounded_wait_warp(bar(&ctrl->raw[st % NS]), (st / NS) & 1, abort)) break;
            if (two && !bounded_wait_warp(bar(&ctrl->raw[(st + 1) % NS]), ((st + 1) / NS) & 1, abort)) break;
            const Raw r0 = load_raw(st);
            const Raw r1 = load_raw(two ? st + 1 : nstages);  // past the end: zeros
            expand(st, r0);
            if (two) expand(st + 1, r1);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(&ctrl->full[st % NS]));
                if (two) mbar_arrive(bar(&ctrl->full[(st + 1) % NS]));
            }
        }
        if (range_bad) atomicOr(&g_device_status, kDevErrRange);
    } else if (warp == COPY_WARP) {
        // ------------------------------------------------------------ bulk copies
        const bool leader = elect_one();
        pdl_wait_primary();  // the token operands are written by the preceding kernel
        int issued = 0;
        for (int st = 0; st < nstages; ++st) {
            const int slot = st % NS;
            if (!bounded_wait_warp(bar(&ctrl->empty[slot]), ((st / NS) & 1) ^ 1, abort)) break;
            const int b0 = kb0 + st * S;
            const int nb = min(S, kb0 + Bl - b0);
            if (leader) {
                uint8_t* sp = stage_ptr(slot);
                const uint32_t rb = bar(&ctrl->raw[slot]);
                const int e0 = (FMT == 0) ? b0 & ~7 : ((b0 >> bsh)) & ~7;
                if (Gm::BITS == 4) {  // a box of 16 bytes x 64 rows per block
                    mbar_arrive_expect_tx(rb, uint32_t(nb * NWH * 16 + NWT * 16 * (Gm::AFF ? 2 : 1)));
                    for (int k = 0; k < nb; ++k)
                        tma_load_2d<1>(smem_addr(sp + OFF_RAW + k * NWH * 16), &tm_q, (b0 + k) * 16, nh0, rb);
                } else {  // one box of both blocks (b0 is even: its byte offset is a multiple of 16)
                    mbar_arrive_expect_tx(rb, uint32_t(S * Gm::BPB * NWH + NWT * 16 * 2));
                    tma_load_2d<1>(smem_addr(sp + OFF_RAW), &tm_q, b0 * Gm::BPB, nh0, rb);
                }
                tma_load_2d<2>(smem_addr(sp + OFF_RSC), &tm_s, e0, n0, rb);
                if (Gm::AFF) tma_load_2d<2>(smem_addr(sp + OFF_RBI), &tm_b, e0, n0, rb);
                const uint32_t fb = bar(&ctrl->full[slot]);
                mbar_arrive_expect_tx(fb, uint32_t(nb * (T_BLK + DX_BLK + (Gm::AFF ? TT * 16 : 0))));
                bulk_g2s(smem_addr(sp + OFF_T), reinterpret_cast<const uint8_t*>(tok) + (int64_t(t) * B + b0) * T_BLK,
                         uint32_t(nb * T_BLK), fb);
                bulk_g2s(smem_addr(sp + OFF_DX), dxs + (int64_t(t) * B + b0) * TT, uint32_t(nb * DX_BLK), fb);
                if (Gm::AFF)
                    bulk_g2s(smem_addr(sp + OFF_XT), xsum + (int64_t(t) * B + b0) * TT, uint32_t(nb * TT * 16), fb);
            }
            __syncwarp();
            issued = st + 1;
        }
        // Let every copy this warp issued land before the CTA can exit (capped waits, as in
        // the single-CTA kernel).
        for (int st = max(0, issued - NS); st < issued; ++st) {
            drain_wait_warp(bar(&ctrl->raw[st % NS]), (st / NS) & 1, 200000ull);
            drain_wait_warp(bar(&ctrl->full[st % NS]), (st / NS) & 1, 200000ull);
        }
    } else if (warp == MMA_WARP) {
        const bool leader = elect_one();
        uint32_t local_abort = 0;
        if (rank == 0) {
            // -------------------------------------------------------- MMA issue (even CTA)
            const uint32_t smem0 = smem_addr(smem);
            const uint32_t zero_addr = smem0 + uint32_t(Gm::OFF_ZERO);
            for (int st = 0; st < nstages; ++st) {
                const int slot = st % NS, g = st % NG;
                if (!bounded_wait_warp(bar(&ctrl->full[slot]), (st / NS) & 1, abort)) break;
                if (!bounded_wait_warp<true>(bar(&ctrl->pfull[slot]), (st / NS) & 1, abort)) break;
                if (!bounded_wait_warp<true>(bar(&ctrl->tempty[g]), ((st / NG) & 1) ^ 1, abort)) break;
                tc_fence_after();
                if (leader) {
                    // Straight-line issue of all S blocks (blocks past the end of a short
                    // last stage fill TMEM tiles that the epilogue never reads).
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
                                tc_mma_f16_pair(d, td, wd, Gm::IDESC, (part | h) != 0);
                            }
                        }
                        if (Gm::AFF) {  // the group bias term; K chunk 1 of both operands is the zero region
                            const uint32_t xt = smem0 + uint32_t(slot * STAGE_BYTES + OFF_XT + k * TT * 16);
                            const uint32_t xw = smem0 + uint32_t(slot * STAGE_BYTES + OFF_XW + k * NWH * 16);
                            tc_mma_f16_pair(d, smem_desc_kmajor(xt, zero_addr - xt, 128),
                                            smem_desc_kmajor(xw, zero_addr - xw, 128), Gm::IDESC, true);
                        }
                    }
                    tc_commit_pair(bar(&ctrl->tfull[g]), 3);
                }
                __syncwarp();
            }
            if (leader) tc_commit_pair(bar(&ctrl->drain), 3);
        } else {
            // -------------------------------------------------------- stage relay (odd CTA)
            const uint32_t pfull0 = mapa_shared(bar(&ctrl->pfull[0]), 0);
            for (int st = 0; st < nstages; ++st) {
                const int slot = st % NS;
                if (!bounded_wait_warp(bar(&ctrl->full[slot]), (st / NS) & 1, abort)) break;
                if (leader) mbar_arrive_remote(pfull0 + uint32_t(slot) * 8u);
                __syncwarp();
            }
        }
        // Both CTAs: every MMA of the pair (and the arrivals of its commits) is done before
        // the tensor memory and the shared memory are released.
        __syncwarp();
        bounded_wait_warp(bar(&ctrl->drain), 0, &local_abort);
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;           // TMEM lane quarter
        const int c0 = (warp >> 2) * CW;  // first TMEM column of this warp
        const int r = q * 32 + lane;      // this thread's TMEM lane: token within the tile
        const uint32_t tempty0 = (rank == 0) ? bar(&ctrl->tempty[0]) : mapa_shared(bar(&ctrl->tempty[0]), 0);
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
            // Only d_x is read from the stage: read it, then hand the stage back to the copy
            // warp (the stage's MMAs are complete).
            float dxv[S];
#pragma unroll
            for (int k = 0; k < S; ++k) dxv[k] = reinterpret_cast<const float*>(sp + OFF_DX)[k * TT + r];
            {
                const float dep = dxv[0] + dxv[S - 1];  // one warp instruction: waits for the loads
                __syncwarp();
                if (lane == 0) mbar_arrive_after(bar(&ctrl->empty[slot]), dep);
            }
#pragma unroll
            for (int k = 0; k < S; ++k) {
                if (k >= nb) break;
                const bool last = (k == nb - 1);
                const float dxr = dxv[k];
#pragma unroll
                for (int h0 = 0; h0 < CW; h0 += LD_COLS) {
                    uint32_t pr[LD_COLS];
                    tmem_load_cols(lane_base + uint32_t((g * S + k) * MN + c0 + h0), pr);
                    if (last && h0 + LD_COLS == CW) {  // the group's tiles are all read: free it
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            if (rank == 0)
                                mbar_arrive(tempty0 + uint32_t(g) * 8u);
                            else
                                mbar_arrive_remote(tempty0 + uint32_t(g) * 8u);
                        }
                    }
#pragma unroll
                    for (int j = 0; j < LD_COLS; ++j) acc[h0 + j] = fmaf(__uint_as_float(pr[j]), dxr, acc[h0 + j]);
                }
            }
        }
        if (!*abort) {
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
        }
    }

    tc_fence_before();
    cluster_sync();  // neither CTA frees the pair's tensor memory or exits while the other may use it
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, Gm::TMEM_COLS);
    }
}

}  // namespace tc
}  // namespace w4a8
