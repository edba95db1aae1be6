// Large-M path: tcgen05 tensor-core GEMM with per-block rescaling.
//
// y[m][n] = sum_b  s_w[n][b] * d_x[m][b] * D[m][n][b],  D = exact 32-wide block dot.
// The block dot must stay exact and each block must be rescaled separately (tract PR
// #2432, "The kernel": Q4_0's per-32-block scales force a per-block rescale; there it
// is one vector multiply per block over accumulator lanes that each hold one output).
// Here every block gets its own tensor-memory accumulator: TMEM lane = weight row,
// TMEM column = token, so each epilogue thread owns one output row and needs no
// cross-lane reduction.
//
// Per block the tensor core produces two 128 x 128 tiles in TMEM:
//   P = 16 * D      two kind::f16 MMAs on fp16 operands that hold small integers (weight
//                   codes q-8 or 16(q-8), affine q or 16q; activation codes 16q_x or q_x,
//                   see quant_act_tc_kernel): every product and block sum is an exact
//                   integer below 2^20, so P is exact.
//   S = s_w (x) d_x/16   one kind::tf32 MMA with K = 8: the weight side holds
//                   (s_w, s_w, s_w, .) per row, the activation side (a, b, c, 0) with
//                   a + b + c = d_x/16 exactly, the second K-chunk of both points at a
//                   zero region. So S = s_w * d_x / 16 up to the accumulator's rounding.
// The epilogue then does acc += P * S per element: one FMA, no per-column scale traffic
// through shared memory (the outer product of the scales comes from the tensor core).
//
// CTA tile: 128 weight rows x TT tokens (TT = 32, 64 or 128); one pipeline stage = 2
// quant blocks (K = 64), 4-7 stages; 512/(2 TT) block buffers in TMEM, each a P tile and
// an S tile. Warp roles (E = TT/8 epilogue warps):
//   warps 0..E-1   epilogue: warp w reads TMEM lanes 32(w%4).. (its hardware lane
//                  quarter) and token columns 32(w/4)..+31 of P and S, accumulates in f32
//   warps E..E+3   producer: load packed 4-bit codes (16 B per row-block, two stages
//                  ahead), expand to fp16 in the MMA's K-major core-matrix layout, store
//                  the row's scale operand (and the affine bias) per block
//   warp E+4       TMEM allocation + single-thread MMA issue
//   warp E+5       one thread issuing the bulk copies of the token operand, its scale
//                  operand and (affine) the per-group bias factor
// Every wait is bounded (bounded_wait); within the epilogue and the producer one thread
// polls and the other warps block on a named barrier. On a timeout all roles stop,
// outstanding copies and MMAs are drained, TMEM is freed and the kernel returns.
#pragma once

#include "device_common.cuh"
#include "quant.cuh"

namespace w4a8 {
namespace tc {

constexpr int BN = 128;                   // weight rows per CTA (MMA M, TMEM lanes)
constexpr int S = 2;                      // quant blocks per stage
constexpr int A_BLK = BN * 64;            // fp16 weight operand bytes per block
constexpr int AS_BLK = BN * 16;           // tf32 scale operand, first K-chunk, weight side
constexpr int ZERO_BYTES = 128 * 16;      // second K-chunk of both scale operands
constexpr int CTRL_BYTES = 512;
constexpr int TMEM_COLS = 512;
constexpr int EPI_COLS = 32;              // token columns per epilogue warp
constexpr uint32_t LBO = 128, SBO = 512;  // fp16 operands: core-matrix strides (K, M/N)
constexpr uint32_t SBO_S = 128;           // tf32 scale operands: 8-row groups 128 B apart

// Geometry for a token tile of TT tokens (32, 64 or 128): TMEM holds NBUF block buffers
// of a P tile (TT columns) and an S tile (TT columns); TT/8 epilogue warps cover the
// 128 x TT tile 32 columns each; the shared-memory ring is as deep as fits.
template <int TT>
struct Geo {
    static constexpr int NBUF = TMEM_COLS / (2 * TT);
    static constexpr int B_BLK = tcgeo::tok_block_bytes(TT);
    static constexpr int BS_BLK = TT * 16;
    static constexpr int OFF_B = S * A_BLK;
    static constexpr int OFF_AS = OFF_B + S * B_BLK;
    static constexpr int OFF_BS = OFF_AS + S * AS_BLK;
    static constexpr int OFF_Z = OFF_BS + S * BS_BLK;
    static constexpr int STAGE_BYTES = OFF_Z + TT * 4;  // + one group's bias factor (affine)
    static constexpr int NS = (TT == 128) ? 4 : (TT == 64) ? 6 : 7;
    static constexpr int SMEM_BYTES = NS * STAGE_BYTES + ZERO_BYTES + CTRL_BYTES + 1024;
    static constexpr int P_COL0 = 0, S_COL0 = NBUF * TT;
    static constexpr int EPI_WARPS = TT / 8;
    static constexpr int PROD_WARP0 = EPI_WARPS;
    static constexpr int MMA_WARP = EPI_WARPS + 4;
    static constexpr int COPY_WARP = EPI_WARPS + 5;
    static constexpr int NUM_THREADS = (EPI_WARPS + 6) * 32;
    static constexpr uint32_t IDESC_P = idesc_f16_f32(BN, TT);
    // kind::tf32: D f32, A and B tf32 (format 2), K-major, M x N
    static constexpr uint32_t IDESC_S =
        (1u << 4) | (2u << 7) | (2u << 10) | (uint32_t(TT >> 3) << 17) | (uint32_t(BN >> 4) << 24);
    static_assert(STAGE_BYTES % 16 == 0, "stage alignment");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert(EPI_WARPS * EPI_COLS == 4 * TT, "epilogue covers the tile");
    static_assert(NBUF * 2 * TT == TMEM_COLS, "tmem columns");
};

constexpr int MAX_NS = 8, MAX_NBUF = 8;
struct Ctrl {
    unsigned long long full_a[MAX_NS];    // producer threads (128 arrivals)
    unsigned long long full_b[MAX_NS];    // bulk copies (1 arrival + bytes)
    unsigned long long empty[MAX_NS];     // MMA commit + one arrival per epilogue warp
    unsigned long long tfull[MAX_NBUF];   // MMA commit
    unsigned long long tempty[MAX_NBUF];  // one arrival per epilogue warp
    unsigned long long drain;         // final MMA drain
    uint32_t tmem_base;
    uint32_t abort;
};
static_assert(sizeof(Ctrl) <= CTRL_BYTES, "control block");

// Expand one 32-bit word of packed codes into four fp16x2 words (8 K-slots).
// Q4_0 word = bytes 4i..4i+3 of a block: low nibbles elements 4i..4i+3, high nibbles
// 16+4i..; affine word = elements 8t..8t+7 at bits 4e. Output slot order (both
// operands use it): low nibbles of bytes 0,2 | of bytes 1,3 | high nibbles of bytes
// 0,2 | of bytes 1,3. Low-nibble slots hold the code, high-nibble slots 16*code; the
// Q4_0 codes are shifted by -8 (-128 for the x16 slots). 0x6400 is fp16 1024, so
// (0x6400 | v) is 1024 + v exactly and one packed subtract removes the offset.
template <int FMT>
__device__ __forceinline__ uint4 expand_word(uint32_t w) {
    const uint32_t ea = (w & 0x000F000Fu) | 0x64006400u;
    const uint32_t eb = ((w >> 8) & 0x000F000Fu) | 0x64006400u;
    const uint32_t ec = (w & 0x00F000F0u) | 0x64006400u;
    const uint32_t ed = ((w >> 8) & 0x00F000F0u) | 0x64006400u;
    const uint32_t off_lo = (FMT == 0) ? 0x64086408u : 0x64006400u;  // 1032 : 1024
    const uint32_t off_hi = (FMT == 0) ? 0x64806480u : 0x64006400u;  // 1152 : 1024
    auto sub = [](uint32_t a, uint32_t b) {
        __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
        return *reinterpret_cast<uint32_t*>(&r);
    };
    return make_uint4(sub(ea, off_lo), sub(eb, off_lo), sub(ec, off_hi), sub(ed, off_hi));
}

// tf32 MMA: D[tmem] (+)= A[smem] * B[smem]^T, both K-major, f32 accumulator.
__device__ __forceinline__ void tc_mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Codes and scales of one stage of one weight row, held in registers until stored.
struct RowStage {
    uint4 w[S];
    float s[S], b[S];
};

template <int FMT, int TT>
__global__ void __launch_bounds__(Geo<TT>::NUM_THREADS, 1)
    gemm_tc_kernel(int M, int N, int K, int group, const __half* __restrict__ tok, const float4* __restrict__ bs,
                   const float* __restrict__ zb, const uint8_t* __restrict__ wq,
                   const uint16_t* __restrict__ wscale, const uint16_t* __restrict__ wbias,
                   float* __restrict__ y) {
    using Gm = Geo<TT>;
    constexpr int NS = Gm::NS, NBUF = Gm::NBUF, B_BLK = Gm::B_BLK, BS_BLK = Gm::BS_BLK;
    constexpr int OFF_B = Gm::OFF_B, OFF_AS = Gm::OFF_AS, OFF_BS = Gm::OFF_BS, OFF_Z = Gm::OFF_Z;
    constexpr int STAGE_BYTES = Gm::STAGE_BYTES, P_COL0 = Gm::P_COL0, S_COL0 = Gm::S_COL0;
    constexpr int EPI_WARPS = Gm::EPI_WARPS, PROD_WARP0 = Gm::PROD_WARP0, MMA_WARP = Gm::MMA_WARP;
    constexpr int COPY_WARP = Gm::COPY_WARP, NUM_THREADS = Gm::NUM_THREADS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* zero = smem + NS * STAGE_BYTES;
    Ctrl* ctrl = reinterpret_cast<Ctrl*>(zero + ZERO_BYTES);
    volatile uint32_t* abort = &ctrl->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = K >> 5;
    const int nstages = (B + S - 1) / S;
    const int n0 = blockIdx.x * BN;
    const int t = blockIdx.y;
    const int bpg = (FMT == 1) ? (group >> 5) : 1;  // blocks per affine group
    const int G = (FMT == 1) ? K / group : 0;

    auto stage_ptr = [&](int slot) { return smem + slot * STAGE_BYTES; };
    auto bar = [](unsigned long long* p) { return smem_addr(p); };

    for (int i = threadIdx.x; i < ZERO_BYTES / 16; i += NUM_THREADS)
        reinterpret_cast<uint4*>(zero)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar(&ctrl->full_a[s]), 128);
            mbar_init(bar(&ctrl->full_b[s]), 1);
            mbar_init(bar(&ctrl->empty[s]), 1 + EPI_WARPS);
        }
        for (int j = 0; j < NBUF; ++j) {
            mbar_init(bar(&ctrl->tfull[j]), 1);
            mbar_init(bar(&ctrl->tempty[j]), EPI_WARPS);
        }
        mbar_init(bar(&ctrl->drain), 1);
        ctrl->abort = 0;
        mbar_init_fence();
    }
    if (warp == MMA_WARP) {
        tmem_alloc(smem_addr(&ctrl->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    fence_proxy_async_smem();  // the zero region is read by the tensor core
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctrl->tmem_base;
    // Dependent launches may begin their prologue; they wait for this grid's completion
    // before reading its output.
    pdl_launch_dependents();

    if (warp >= PROD_WARP0 && warp < PROD_WARP0 + 4) {
        // ------------------------------------------------------------ producer
        const int p = threadIdx.x - PROD_WARP0 * 32;
        const int n = n0 + p;
        const bool row_ok = n < N;
        const uint4* wrow = reinterpret_cast<const uint4*>(wq + int64_t(row_ok ? n : 0) * (K >> 1));
        auto load = [&](int st, RowStage& rs) {
#pragma unroll
            for (int k = 0; k < S; ++k) {
                const int b = st * S + k;
                rs.w[k] = make_uint4(0u, 0u, 0u, 0u);
                rs.s[k] = 0.0f;
                rs.b[k] = 0.0f;
                if (row_ok && b < B) {
                    rs.w[k] = __ldg(wrow + b);
                    if (FMT == 0) {
                        rs.s[k] = __half2float(__ushort_as_half(wscale[int64_t(n) * B + b]));
                    } else {
                        rs.s[k] = __bfloat162float(__ushort_as_bfloat16(wscale[int64_t(n) * G + b / bpg]));
                        rs.b[k] = __bfloat162float(__ushort_as_bfloat16(wbias[int64_t(n) * G + b / bpg]));
                    }
                }
            }
        };
        // Store one stage into shared memory; false if the wait gave up.
        auto produce = [&](int st, const RowStage& rs) {
            const int slot = st % NS;
            if (!bounded_wait_group(bar(&ctrl->empty[slot]), ((st / NS) & 1) ^ 1, abort, p == 0, 2, 128)) return false;
            uint8_t* sp = stage_ptr(slot);
#pragma unroll
            for (int k = 0; k < S; ++k) {
                const uint32_t w[4] = {rs.w[k].x, rs.w[k].y, rs.w[k].z, rs.w[k].w};
                uint8_t* arow = sp + k * A_BLK + (p >> 3) * 512 + (p & 7) * 16;
#pragma unroll
                for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(arow + c * 128) = expand_word<FMT>(w[c]);
                // scale operand (s, s, s, bias): the fourth slot meets a zero on the token
                // side, so it only carries the affine bias to the epilogue
                reinterpret_cast<float4*>(sp + OFF_AS + k * AS_BLK)[p] = make_float4(rs.s[k], rs.s[k], rs.s[k], rs.b[k]);
            }
            fence_proxy_async_smem();
            mbar_arrive(bar(&ctrl->full_a[slot]));
            return true;
        };
        RowStage r0, r1, r2;  // stages st, st+1, st+2 in flight
        load(0, r0);
        if (1 < nstages) load(1, r1);
        for (int st = 0; st < nstages; st += 3) {
            if (st + 2 < nstages) load(st + 2, r2);
            if (!produce(st, r0)) break;
            if (st + 1 >= nstages) break;
            if (st + 3 < nstages) load(st + 3, r0);
            if (!produce(st + 1, r1)) break;
            if (st + 2 >= nstages) break;
            if (st + 4 < nstages) load(st + 4, r1);
            if (!produce(st + 2, r2)) break;
        }
    } else if (warp >= MMA_WARP) {
        if (warp == COPY_WARP && lane == 0) {
            // -------------------------------------------------------- bulk copies
            pdl_wait_primary();  // the token operands are written by the preceding kernel
            int issued = 0;
            for (int st = 0; st < nstages; ++st) {
                const int slot = st % NS;
                if (!bounded_wait(bar(&ctrl->empty[slot]), ((st / NS) & 1) ^ 1, abort)) break;
                const int b0 = st * S;
                const int nb = min(S, B - b0);
                // affine: the bias factor of the group whose last block is in this stage
                const bool zlast = (FMT == 1) && (((b0 + nb) % bpg) == 0);
                const uint32_t bytes_tok = nb * B_BLK, bytes_bs = nb * BS_BLK;
                const uint32_t bytes_z = zlast ? TT * 4 : 0;
                const uint32_t fb = bar(&ctrl->full_b[slot]);
                uint8_t* sp = stage_ptr(slot);
                mbar_arrive_expect_tx(fb, bytes_tok + bytes_bs + bytes_z);
                bulk_g2s(smem_addr(sp + OFF_B), reinterpret_cast<const uint8_t*>(tok) + (int64_t(t) * B + b0) * B_BLK,
                         bytes_tok, fb);
                bulk_g2s(smem_addr(sp + OFF_BS), bs + (int64_t(t) * B + b0) * TT, bytes_bs, fb);
                if (zlast) bulk_g2s(smem_addr(sp + OFF_Z), zb + (int64_t(t) * G + (b0 + nb - 1) / bpg) * TT, bytes_z, fb);
                issued = st + 1;
            }
            // Let every copy this thread issued land before the CTA can exit (on the
            // normal path they have, or soon will; after an abort some may not be consumed).
            uint32_t local_abort = 0;
            for (int st = max(0, issued - NS); st < issued; ++st)
                bounded_wait(bar(&ctrl->full_b[st % NS]), (st / NS) & 1, &local_abort);
        } else if (warp == MMA_WARP && lane == 0) {
            // -------------------------------------------------------- MMA issue
            const uint32_t zero_addr = smem_addr(zero);
            for (int i = 0; i < B; ++i) {
                const int st = i / S, k = i - st * S, slot = st % NS;
                const uint32_t par = (st / NS) & 1;
                if (k == 0) {
                    if (!bounded_wait(bar(&ctrl->full_a[slot]), par, abort)) break;
                    if (!bounded_wait(bar(&ctrl->full_b[slot]), par, abort)) break;
                }
                const int buf = i % NBUF;
                if (!bounded_wait(bar(&ctrl->tempty[buf]), ((i / NBUF) & 1) ^ 1, abort)) break;
                tc_fence_after();
                uint8_t* sp = stage_ptr(slot);
                const uint32_t a_addr = smem_addr(sp + k * A_BLK);
                const uint32_t b_addr = smem_addr(sp + OFF_B + k * B_BLK);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    tc_mma_f16(tmem_base + uint32_t(P_COL0 + buf * TT), smem_desc_kmajor(a_addr + h * 256, LBO, SBO),
                               smem_desc_kmajor(b_addr + h * 256, LBO, SBO), Gm::IDESC_P, h);
                }
                const uint32_t as_addr = smem_addr(sp + OFF_AS + k * AS_BLK);
                const uint32_t bs_addr = smem_addr(sp + OFF_BS + k * BS_BLK);
                tc_mma_tf32(tmem_base + uint32_t(S_COL0 + buf * TT),
                            smem_desc_kmajor(as_addr, zero_addr - as_addr, SBO_S),
                            smem_desc_kmajor(bs_addr, zero_addr - bs_addr, SBO_S), Gm::IDESC_S, 0);
                tc_commit(bar(&ctrl->tfull[buf]));
                if (k == S - 1 || i == B - 1) tc_commit(bar(&ctrl->empty[slot]));
            }
            // Wait until every MMA (and the barrier arrivals their commits trigger) is done
            // before TMEM and shared memory are released.
            uint32_t local_abort = 0;
            tc_commit(bar(&ctrl->drain));
            bounded_wait(bar(&ctrl->drain), 0, &local_abort);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                    // lane quarter: weight rows 32q..32q+31
        const int c0 = (warp >> 2) * EPI_COLS;     // token columns c0..c0+31
        const int p = q * 32 + lane;               // this thread's weight row within the tile
        unsigned long long acc[EPI_COLS / 2];      // f32 pairs
#pragma unroll
        for (int j = 0; j < EPI_COLS / 2; ++j) acc[j] = 0ull;
        const uint32_t lane_base = tmem_base + (uint32_t(q * 32) << 16);
        for (int i = 0; i < B; ++i) {
            const int st = i / S, k = i - st * S, slot = st % NS;
            const int buf = i % NBUF;
            if (!bounded_wait_group(bar(&ctrl->tfull[buf]), (i / NBUF) & 1, abort, threadIdx.x == 0, 1,
                                    EPI_WARPS * 32))
                break;
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < EPI_COLS / 16; ++h) {
                uint32_t pr[16], sr[16];
                tmem_ld_32x32_x16(lane_base + uint32_t(P_COL0 + buf * TT + c0 + 16 * h), pr);
                tmem_ld_32x32_x16(lane_base + uint32_t(S_COL0 + buf * TT + c0 + 16 * h), sr);
                tmem_wait_ld16x2(pr, sr);
                if (h == EPI_COLS / 16 - 1) {  // TMEM buffer free: every value is in registers
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(&ctrl->tempty[buf]));
                }
#pragma unroll
                for (int j = 0; j < 16; j += 2) fma2_pp(acc[8 * h + j / 2], pr[j], pr[j + 1], sr[j], sr[j + 1]);
            }
            if (FMT == 1 && ((i + 1) % bpg) == 0) {  // last block of a group: add bias * Z
                const uint8_t* sp = stage_ptr(slot);
                const float bsc = reinterpret_cast<const float4*>(sp + OFF_AS + k * AS_BLK)[p].w;
                const unsigned long long b2 = pack2(bsc, bsc);
                const float* zs = reinterpret_cast<const float*>(sp + OFF_Z) + c0;
#pragma unroll
                for (int j = 0; j < EPI_COLS; j += 4) {
                    const float4 zv = *reinterpret_cast<const float4*>(zs + j);
                    fma2_bias(acc[j / 2], zv.x, zv.y, b2);
                    fma2_bias(acc[j / 2 + 1], zv.z, zv.w, b2);
                }
            }
            __syncwarp();
            if (lane == 0 && (k == S - 1 || i == B - 1)) mbar_arrive(bar(&ctrl->empty[slot]));
        }
        const int n = n0 + p;
        if (n < N && !*abort) {
#pragma unroll
            for (int j = 0; j < EPI_COLS; j += 2) {
                float a, b;
                unpack2(acc[j / 2], a, b);
                const int m = t * TT + c0 + j;
                if (m < M) y[int64_t(m) * N + n] = a;
                if (m + 1 < M) y[int64_t(m + 1) * N + n] = b;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace tc
}  // namespace w4a8
