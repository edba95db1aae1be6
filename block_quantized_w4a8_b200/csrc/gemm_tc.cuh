// Large-M path: tcgen05 tensor-core GEMM with per-block rescaling.
//
// y[m][n] = sum_b  s_w[n][b] * d_x[m][b] * D[m][n][b],  D = exact 32-wide block dot.
// The block dot must stay exact and each block must be rescaled separately (tract PR
// #2432, "The kernel": Q4_0's per-32-block scales force a per-block rescale; there it
// is one vector multiply per block over accumulator lanes that each hold one output).
// Here every block gets its own tensor-memory accumulator: TMEM lane = weight row,
// TMEM column = token, so each epilogue thread owns one output row and rescales its
// columns with a per-thread (weight) and a per-column (activation) scale, with no
// cross-lane reduction.
//
// Operands are fp16 holding small integers, so the MMA (kind::f16, f32 accumulate) is
// exact: weight codes (q-8 or 16(q-8); affine q or 16q) times activation codes (16q_x or
// q_x, see quant_act_tc_kernel), every product an integer below 2^15 and every block
// sum below 2^20. The block dot comes out of TMEM as 16*D in f32 with no conversion.
//
// CTA tile: 128 weight rows x 128 tokens; one pipeline stage = 4 quant blocks (K=128),
// 3 stages; 4 TMEM accumulator buffers of 128 columns (the whole 512-column TMEM).
// Warp roles (448 threads):
//   WG0, WG1 (warps 0-7)  epilogue: warp w reads TMEM lanes 32(w%4).. (its hardware lane
//                         quarter) and token columns 64(w/4)..+63 of each block's
//                         accumulator (16x256b loads: each thread 4 rows x 16 columns),
//                         scales them and accumulates in f32 registers
//   WG2 (warps 8-11)      producer: load packed 4-bit codes (16 B per row-block, two
//                         stages ahead), expand to fp16 in the MMA's K-major core-matrix
//                         layout, store the per-row scales
//   warp 12               TMEM allocation + single-thread MMA issue
//   warp 13               one thread issuing the bulk copies of the token operand and
//                         its scales
// The kernel runs one CTA per SM with 128 registers per thread.
// Every wait is bounded (bounded_wait); on a timeout all roles stop, outstanding copies
// and MMAs are drained, TMEM is freed and the kernel returns.
#pragma once

#include "device_common.cuh"
#include "quant.cuh"

namespace w4a8 {
namespace tc {

constexpr int BN = 128;                   // weight rows per CTA (MMA M, TMEM lanes)
constexpr int TT = tcgeo::kTokTile;       // tokens per CTA (MMA N)
constexpr int S = 4;                      // quant blocks per stage
constexpr int NS = 3;                     // stages in the ring
constexpr int NACC = 4;                   // TMEM accumulator buffers
constexpr int A_BLK = BN * 64;            // fp16 weight operand bytes per block
constexpr int B_BLK = tcgeo::kTokBlockBytes;
constexpr int OFF_B = S * A_BLK;
constexpr int OFF_DX = OFF_B + S * B_BLK;
constexpr int OFF_WS = OFF_DX + S * TT * 4;
constexpr int OFF_WB = OFF_WS + S * BN * 4;
constexpr int OFF_Z = OFF_WB + S * BN * 4;
constexpr int STAGE_BYTES = OFF_Z + S * TT * 4;
constexpr int CTRL_BYTES = 256;
constexpr int SMEM_BYTES = NS * STAGE_BYTES + CTRL_BYTES + 1024;  // + alignment slack
constexpr int TMEM_COLS = NACC * TT;
constexpr int EPI_WARPS = 8;
constexpr int EPI_COLS = TT / (EPI_WARPS / 4);   // token columns per epilogue warp (64)
constexpr int PROD_WARP0 = 8;
constexpr int MMA_WARP = 12;
constexpr int COPY_WARP = 13;
constexpr int NUM_THREADS = 448;
constexpr int MAX_REGS = 128;
constexpr uint32_t IDESC = idesc_f16_f32(BN, TT);
constexpr uint32_t LBO = 128, SBO = 512;  // core-matrix strides (K, M/N)

static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
static_assert(SMEM_BYTES <= 232448, "shared memory");
static_assert(TMEM_COLS == 512, "tmem allocation must be a power of two >= 32");
static_assert(EPI_COLS == 64, "epilogue loads 64 columns per warp");
static_assert(NUM_THREADS * MAX_REGS <= 65536, "register file");

struct Ctrl {
    unsigned long long full_a[NS];    // producer threads (128 arrivals)
    unsigned long long full_b[NS];    // bulk copies (1 arrival + bytes)
    unsigned long long empty[NS];     // MMA commit + one arrival per epilogue warp
    unsigned long long tfull[NACC];   // MMA commit
    unsigned long long tempty[NACC];  // one arrival per epilogue warp
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

// Codes and scales of one stage of one weight row, held in registers until stored.
struct RowStage {
    uint4 w[S];
    float s[S], b[S];
};

template <int FMT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_tc_kernel(int M, int N, int K, int group, const __half* __restrict__ tok, const float* __restrict__ dx16,
                   const float* __restrict__ zb, const uint8_t* __restrict__ wq,
                   const uint16_t* __restrict__ wscale, const uint16_t* __restrict__ wbias,
                   float* __restrict__ y) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + NS * STAGE_BYTES);
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

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar(&ctrl->full_a[s]), 128);
            mbar_init(bar(&ctrl->full_b[s]), 1);
            mbar_init(bar(&ctrl->empty[s]), 1 + EPI_WARPS);
        }
        for (int j = 0; j < NACC; ++j) {
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
            if (!bounded_wait_warp(bar(&ctrl->empty[slot]), ((st / NS) & 1) ^ 1, abort)) return false;
            uint8_t* sp = stage_ptr(slot);
#pragma unroll
            for (int k = 0; k < S; ++k) {
                const uint32_t w[4] = {rs.w[k].x, rs.w[k].y, rs.w[k].z, rs.w[k].w};
                uint8_t* arow = sp + k * A_BLK + (p >> 3) * 512 + (p & 7) * 16;
#pragma unroll
                for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(arow + c * 128) = expand_word<FMT>(w[c]);
                reinterpret_cast<float*>(sp + OFF_WS)[k * BN + p] = rs.s[k];
                if (FMT == 1) reinterpret_cast<float*>(sp + OFF_WB)[k * BN + p] = rs.b[k];
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
            pdl_wait_primary();  // the token operand is written by the preceding kernel
            int issued = 0;
            for (int st = 0; st < nstages; ++st) {
                const int slot = st % NS;
                if (!bounded_wait(bar(&ctrl->empty[slot]), ((st / NS) & 1) ^ 1, abort)) break;
                const int b0 = st * S;
                const int nb = min(S, B - b0);
                const uint32_t bytes_tok = nb * B_BLK, bytes_dx = nb * TT * 4;
                const uint32_t bytes_z = (FMT == 1) ? (nb / bpg) * TT * 4 : 0;
                const uint32_t fb = bar(&ctrl->full_b[slot]);
                uint8_t* sp = stage_ptr(slot);
                mbar_arrive_expect_tx(fb, bytes_tok + bytes_dx + bytes_z);
                bulk_g2s(smem_addr(sp + OFF_B), reinterpret_cast<const uint8_t*>(tok) + (int64_t(t) * B + b0) * B_BLK,
                         bytes_tok, fb);
                bulk_g2s(smem_addr(sp + OFF_DX), dx16 + (int64_t(t) * B + b0) * TT, bytes_dx, fb);
                if (FMT == 1) bulk_g2s(smem_addr(sp + OFF_Z), zb + (int64_t(t) * G + b0 / bpg) * TT, bytes_z, fb);
                issued = st + 1;
            }
            // Let every copy this thread issued land before the CTA can exit (on the
            // normal path they have, or soon will; after an abort some may not be consumed).
            uint32_t local_abort = 0;
            for (int st = max(0, issued - NS); st < issued; ++st)
                bounded_wait(bar(&ctrl->full_b[st % NS]), (st / NS) & 1, &local_abort);
        } else if (warp == MMA_WARP && lane == 0) {
            // -------------------------------------------------------- MMA issue
            for (int i = 0; i < B; ++i) {
                const int st = i / S, k = i - st * S, slot = st % NS;
                const uint32_t par = (st / NS) & 1;
                if (k == 0) {
                    if (!bounded_wait(bar(&ctrl->full_a[slot]), par, abort)) break;
                    if (!bounded_wait(bar(&ctrl->full_b[slot]), par, abort)) break;
                }
                const int buf = i % NACC;
                if (!bounded_wait(bar(&ctrl->tempty[buf]), ((i / NACC) & 1) ^ 1, abort)) break;
                tc_fence_after();
                const uint32_t a_addr = smem_addr(stage_ptr(slot) + k * A_BLK);
                const uint32_t b_addr = smem_addr(stage_ptr(slot) + OFF_B + k * B_BLK);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    tc_mma_f16(tmem_base + uint32_t(buf * TT), smem_desc_kmajor(a_addr + h * 256, LBO, SBO),
                               smem_desc_kmajor(b_addr + h * 256, LBO, SBO), IDESC, h);
                }
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
        // Warp w covers TMEM lanes 32q..32q+31 (q = w%4, its hardware lane quarter) and
        // token columns c0..c0+63 (c0 = 64*(w/4)). It reads them as 2 row halves x 2
        // column groups with tcgen05.ld.16x256b.x4, so thread t owns weight rows
        // 32q + t/4 + {0, 8, 16, 24} and token columns c0 + 8j + 2(t%4) + {0, 1}
        // (j = 0..7): 4 row scales and 8 column-scale pairs per block instead of one
        // broadcast column scale per accumulator.
        const int q = warp & 3;
        const int c0 = (warp >> 2) * EPI_COLS;
        const int tr = lane >> 2, tc = (lane & 3) * 2;
        unsigned long long acc[4][8];  // [row 0..3][column pair j]
#pragma unroll
        for (int r_ = 0; r_ < 4; ++r_)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[r_][j] = 0ull;
        const uint32_t lane_base = tmem_base + (uint32_t(q * 32) << 16);
        for (int i = 0; i < B; ++i) {
            const int st = i / S, k = i - st * S, slot = st % NS;
            const int buf = i % NACC;
            if (!bounded_wait_warp(bar(&ctrl->tfull[buf]), (i / NACC) & 1, abort)) break;
            tc_fence_after();
            const uint8_t* sp = stage_ptr(slot);
            const float* dxs = reinterpret_cast<const float*>(sp + OFF_DX) + k * TT + c0 + tc;
            const float* wss = reinterpret_cast<const float*>(sp + OFF_WS) + k * BN + q * 32 + tr;
            // Four chunks per block, chunk c = (column group g = c/2, row half h = c%2);
            // the TMEM load of chunk c+1 is issued before chunk c is scaled, so only the
            // first load of a block is exposed.
            const uint32_t tbase = lane_base + uint32_t(buf * TT + c0);
            auto chunk_addr = [&](int c) { return tbase + (uint32_t(16 * (c & 1)) << 16) + uint32_t(32 * (c >> 1)); };
            unsigned long long dx2[4];
            auto load_dx = [&](int g) {
#pragma unroll
                for (int jj = 0; jj < 4; ++jj)
                    dx2[jj] = *reinterpret_cast<const unsigned long long*>(dxs + 8 * (4 * g + jj));
            };
            auto scale_chunk = [&](int c, const uint32_t (&r)[16]) {
                const int g = c >> 1, h = c & 1;
                const float wa = wss[16 * h], wb = wss[16 * h + 8];
                const unsigned long long wa2 = pack2(wa, wa), wb2 = pack2(wb, wb);
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int j = 4 * g + jj;
                    fma2(acc[2 * h][j], r[4 * jj], r[4 * jj + 1], mul2(dx2[jj], wa2));
                    fma2(acc[2 * h + 1][j], r[4 * jj + 2], r[4 * jj + 3], mul2(dx2[jj], wb2));
                }
            };
            uint32_t ra[16], rb[16];
            load_dx(0);
            tmem_ld_16x256_x4(chunk_addr(0), ra);
            tmem_wait_ld16(ra);
            tmem_ld_16x256_x4(chunk_addr(1), rb);
            scale_chunk(0, ra);
            tmem_wait_ld16(rb);
            tmem_ld_16x256_x4(chunk_addr(2), ra);
            scale_chunk(1, rb);
            tmem_wait_ld16(ra);
            tmem_ld_16x256_x4(chunk_addr(3), rb);
            load_dx(1);
            scale_chunk(2, ra);
            tmem_wait_ld16(rb);
            tc_fence_before();  // TMEM buffer free: every value of the block is in registers
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(&ctrl->tempty[buf]));
            scale_chunk(3, rb);
            if (FMT == 1 && ((i + 1) % bpg) == 0) {  // last block of a group: add bias * Z
                const float* bss = reinterpret_cast<const float*>(sp + OFF_WB) + k * BN + q * 32 + tr;
                const float* zs = reinterpret_cast<const float*>(sp + OFF_Z) + (k / bpg) * TT + c0 + tc;
#pragma unroll
                for (int r_ = 0; r_ < 4; ++r_) {
                    const float bv = bss[8 * r_];
                    const unsigned long long b2 = pack2(bv, bv);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float2 z = *reinterpret_cast<const float2*>(zs + 8 * j);
                        fma2_bias(acc[r_][j], z.x, z.y, b2);
                    }
                }
            }
            __syncwarp();
            if (lane == 0 && (k == S - 1 || i == B - 1)) mbar_arrive(bar(&ctrl->empty[slot]));
        }
        if (!*abort) {
#pragma unroll
            for (int r_ = 0; r_ < 4; ++r_) {
                const int n = n0 + q * 32 + tr + 8 * r_;
                if (n < N) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        float a, b;
                        unpack2(acc[r_][j], a, b);
                        const int m = t * TT + c0 + 8 * j + tc;
                        if (m < M) y[int64_t(m) * N + n] = a;
                        if (m + 1 < M) y[int64_t(m + 1) * N + n] = b;
                    }
                }
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
