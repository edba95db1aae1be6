// Tensor-core path for small M on int8 MMAs: tcgen05.mma kind::i8, one K = 32 MMA per
// quant block, the exact int32 block dot in tensor memory, the per-block rescale in f32
// (tract PR #2432, "The kernel": Q4_0's per-32-block scales force a rescale per block; MLX
// PR #4802: int8 x int8 MMAs on the original codes).
//
// Orientation: the 128 weight rows of a tile are the MMA's M (TMEM lanes), the tile's MN =
// 16, 32 or 64 tokens its N (TMEM columns), so at small M almost no MMA row is padding.
//
// Weight operand: Q4_0 codes as signed bytes 16*(q - 8): the high nibble in place
// ((w & 0xF0F0F0F0) ^ 0x80808080: (q ^ 8) << 4, which as a two's complement byte is
// 16*(q - 8)) and the low nibble moved up the same way -- three logic operations per four
// bytes, no arithmetic. Byte j of a block's 16 code bytes holds element j (low nibble)
// and element j + 16 (high nibble), so the expanded row is elements 0..31 in order.
// Token operand: the Q8_0 codes in element order (quant_act_i8_kernel). The MMA gives
// D16 = 16 * sum (q - 8) q_x exactly (|D16| <= 520192 < 2^22). For 16 and 32 tokens the MMA
// accumulates onto tensor-memory words preset to the bits of the float 1.5 * 2^23
// (0x4B400000): the floats in [2^23, 2^24) are the integers, so each word then is the float
// 1.5 * 2^23 + D16 exactly, with no conversion instruction; for 64 tokens the MMA writes
// D16 and the epilogue adds the same bits with an integer add after the load. The epilogue forms round(D16 * d_w / 16) with one FMA
// (F * w - 1.5 * 2^23 * w; the addend is exact, w having at most 12 significant bits) and
// adds its product with d_x with a second: two roundings per block, and unlike the fp16
// path no range limit on the weight scales.
//
// Pipelines: a ring of raw code boxes (one 2-D TMA box of 128 rows x 128 bytes -- 8 blocks
// of codes -- per stage, 128-byte swizzled so that the producers' 16-byte reads down a
// column are conflict-free) that the copy warp keeps full from the start, before the grid
// waits on its predecessor; a ring of MMA operands -- the expanded weights in tensor memory
// (the MMA's A from TMEM: row p of the tile is lane p, written by the thread that expanded
// it, so the expansion costs no shared-memory bandwidth), the token codes in shared memory
// -- that the MMA warp itself hands back, by a tensor-core commit, once the stage's MMAs
// are done;
// and a ring of the stage's weight scales (one TMA box of 128 rows x 8 fp16) and d_x rows
// that the epilogue hands back: the epilogue reads every operand from shared memory,
// never waiting on a global load behind the weight stream. So the producers run ahead of the
// tensor core by the operand ring and the tensor core ahead of the epilogue by the TMEM
// groups, and no slot waits for a role that does not read it.
// Warp roles: epilogue warps (TMEM lane quarter x column chunk); four producer warps (one
// weight row per thread: nibbles -> bytes, stored to the row's TMEM lane); one
// MMA warp (also allocates TMEM); one copy warp for the raw code boxes; one copy warp for
// the token codes, scales and d_x (the only role that waits on the preceding grid). Every
// wait is bounded; on a timeout all roles stop, copies and MMAs are drained and TMEM is
// freed.
#pragma once

#include <cuda.h>  // CUtensorMap (the type only; maps are encoded by the host code)

#include "device_common.cuh"
#include "gemm_tc.cuh"

namespace w4a8 {
namespace i8 {

__host__ __device__ constexpr int tok_block_bytes(int tt) { return tt * 32; }  // one 32-wide block, int8

// Instruction descriptor, kind::i8: A and B signed 8-bit, D signed 32-bit, both K-major.
__host__ __device__ constexpr uint32_t idesc_i8_s32(int M, int N) {
    return (2u << 4)                          // D format s32
           | (1u << 7) | (1u << 10)           // A, B format s8
           | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}
// D (TMEM) = A (TMEM: row i in lane i, K along the columns, 4 bytes per column) x B
// (shared memory, K-major) + D if `accumulate`, one MMA of M = 128, N = MN, K = 32.
__device__ __forceinline__ void tc_mma_i8_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Core-matrix strides of a K-major operand with 32-byte rows (one block of int8): along K
// (the two 16-byte halves of a row) and along rows (groups of 8 rows).
constexpr uint32_t LBO = 128, SBO = 256;

template <int MN>
struct Geo {
    static constexpr int TT = MN;                 // tokens per tile
    static constexpr int NW = 128;                // weight rows per tile
    static constexpr int T_BLK = TT * 32;
    static constexpr int DX_BLK = TT * 4;
    static constexpr int S = 8;                   // quant blocks per stage (one code box)
    static constexpr int RAW_BYTES = NW * 128;    // one code box, 1024-aligned slots
    // operand slot: the stage's token codes in shared memory (1024-aligned) and its
    // expanded weights in tensor memory (8 columns per block)
    static constexpr int OP_BYTES = tc::align_up(S * T_BLK, 1024);
    static constexpr int NO = 4;                  // operand slots
    // epilogue slot: the stage's weight scales (NW rows x S fp16), then d_x (S x TT f32)
    static constexpr int SC_BYTES = NW * S * 2;
    static constexpr int ES_BYTES = SC_BYTES + S * DX_BLK;
    static constexpr int ND = MN == 64 ? 4 : 8;   // epilogue slots
    static constexpr int NR = tc::cmin(8, (tc::SMEM_LIMIT - 2048 - NO * OP_BYTES - ND * ES_BYTES) / RAW_BYTES);
    static constexpr int OFF_OPS = NR * RAW_BYTES;
    static constexpr int OFF_DX = OFF_OPS + NO * OP_BYTES;
    static constexpr int OFF_CTRL = tc::align_up(OFF_DX + ND * ES_BYTES, 1024);
    static constexpr int SMEM_BYTES = OFF_CTRL + 1024 + 1024;
    // TMEM: accumulators in columns [0, 256), operand slots' weights in [256, 256 + NO * 64)
    static constexpr int ACC_COLS = 256;
    static constexpr int A_COL0 = ACC_COLS;
    static constexpr int A_SLOT_COLS = S * 8;
    static constexpr int NBUF = ACC_COLS / MN;             // TMEM accumulator tiles (one per block)
    static constexpr int GS = tc::cmin(S, NBUF / 2);       // blocks per TMEM group (at least two groups)
    static constexpr int NG = tc::cmin(8, NBUF / GS);      // TMEM groups, used in turn
    static constexpr int HALVES = S / GS;                  // TMEM groups per stage
    static constexpr int TMEM_COLS = 512;
    // columns per epilogue warp: 8 warps at 16 tokens, 16 warps above (more warps per SM
    // sub-partition to cover the tensor-memory load latency)
    static constexpr int CW = MN == 64 ? 16 : 8;
    static constexpr int EPI_WARPS = 4 * MN / CW;
    // two producer warps per TMEM lane quarter, each expanding half of the stage's blocks
    static constexpr int PROD_WARPS = 2 * NW / 32;
    static constexpr int PROD_BLKS = S / 2;
    static constexpr int PROD_WARP0 = EPI_WARPS;
    static constexpr int MMA_WARP = PROD_WARP0 + PROD_WARPS;
    static constexpr int COPY_WARP = MMA_WARP + 1;
    static constexpr int OPC_WARP = COPY_WARP + 1;
    static constexpr int NUM_THREADS = (OPC_WARP + 1) * 32;
    static constexpr uint32_t IDESC = idesc_i8_s32(128, MN);
    // How the epilogue turns a tile's int32 into the float 1.5 * 2^23 + D16: by presetting
    // the tile to the bits of 1.5 * 2^23 for the MMA to accumulate onto (16 and 32 tokens),
    // or by an integer add after the load (64 tokens, where the preset stores would write
    // 256 KB of tensor memory per stage; measured 38.9 -> 34.2 us at 4096 x 14336).
    static constexpr bool PRESET = MN <= 32;
    static_assert(MN == 16 || MN == 32 || MN == 64, "MMA N");
    static_assert(NG * GS * MN <= ACC_COLS && A_COL0 + NO * A_SLOT_COLS <= TMEM_COLS, "TMEM allocation");
    static_assert(NR >= 2, "raw ring depth");
    static_assert(PROD_BLKS == 4, "a producer warp stores 32 TMEM columns per stage");
    static_assert(NG >= 2 && S % GS == 0, "TMEM groups");
    static_assert(SMEM_BYTES <= tc::SMEM_LIMIT, "shared memory");
    static_assert(OFF_DX % 16 == 0 && OP_BYTES % 1024 == 0, "operand alignment");
    static_assert(NO <= 4 && ND <= 8, "control block");
};

// The bits of the float 1.5 * 2^23: the value tensor-memory accumulators are preset to.
constexpr uint32_t kMagicBits = 0x4B400000u;
constexpr float kMagic = 12582912.0f;

// acc += round(d * w) * x lane-wise, for two accumulator words f holding the floats
// 1.5 * 2^23 + d: round(d * w) = fma(f, w, -1.5 * 2^23 * w), the addend nc = -1.5 * 2^23 * w
// exact. The product with x and the accumulation round once more.
__device__ __forceinline__ void fma2_magic(unsigned long long& acc, uint32_t f0, uint32_t f1, float x0, float x1,
                                           unsigned long long w2, unsigned long long nc2) {
    asm("{\n\t.reg .b64 ff, xx, gg;\n\t"
        "mov.b64 ff, {%1, %2};\n\t"
        "mov.b64 xx, {%3, %4};\n\t"
        "fma.rn.f32x2 gg, ff, %5, %6;\n\t"
        "fma.rn.f32x2 %0, gg, xx, %0;\n\t}\n"
        : "+l"(acc)
        : "r"(f0), "r"(f1), "f"(x0), "f"(x1), "l"(w2), "l"(nc2));
}

constexpr int MAX_NR = 8, MAX_NO = 4, MAX_ND = 8, MAX_NG = 8;
struct Ctrl {
    unsigned long long raw_full[MAX_NR];   // TMA of a code box (1 arrival + bytes)
    unsigned long long raw_empty[MAX_NR];  // one arrival per producer warp after expanding the box
    unsigned long long op_full[MAX_NO];    // one arrival per producer warp + token bulk copy (1 + bytes)
    unsigned long long op_empty[MAX_NO];   // tensor-core commit after the stage's MMAs
    unsigned long long dx_full[MAX_ND];    // scale box + d_x bulk copy (1 + bytes)
    unsigned long long dx_empty[MAX_ND];   // one arrival per epilogue warp
    unsigned long long tfull[MAX_NG];      // MMA commit, once per TMEM group use
    unsigned long long tempty[MAX_NG];     // one arrival per epilogue warp (the group's columns preset again)
    unsigned long long drain;              // final MMA drain
    uint32_t tmem_base;
    uint32_t abort;
};
static_assert(sizeof(Ctrl) <= 1024, "control block");

// Loads CW TMEM columns of this warp's lane quarter into registers (and waits for them).
__device__ __forceinline__ void tmem_cols(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7])
                 :
                 : "memory");
}
__device__ __forceinline__ void tmem_cols(uint32_t taddr, uint32_t (&r)[32]) {
    tmem_ld_32x32(taddr, r);
    tmem_wait_ld(r);
}
__device__ __forceinline__ void tmem_cols(uint32_t taddr, uint32_t (&r)[16]) {
    tmem_ld_32x32_x16(taddr, r);
    tmem_wait_ld16(r);
}

// Presets CW TMEM columns of this warp's lane quarter to kMagicBits (completion: a later
// tcgen05.wait::st).
#define W4A8_M4(v) v ", " v ", " v ", " v
#define W4A8_M8(v) W4A8_M4(v) ", " W4A8_M4(v)
template <int CW>
__device__ __forceinline__ void tmem_preset(uint32_t taddr) {
    if constexpr (CW == 8)
        asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {" W4A8_M8("%1") "};" ::"r"(taddr), "r"(kMagicBits)
                     : "memory");
    else if constexpr (CW == 16)
        asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {" W4A8_M8("%1") ", " W4A8_M8("%1") "};" ::"r"(taddr),
                     "r"(kMagicBits)
                     : "memory");
    else
        asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {" W4A8_M8("%1") ", " W4A8_M8("%1") ", " W4A8_M8(
                         "%1") ", " W4A8_M8("%1") "};" ::"r"(taddr),
                     "r"(kMagicBits)
                     : "memory");
}
#undef W4A8_M8
#undef W4A8_M4
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// Stores 32 words into 32 TMEM columns of this warp's lane quarter.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
        "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
        "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

// Q4_0 only. Launch: grid (ceil(N / 128), token tiles, splits of K), Geo<MN>::NUM_THREADS
// threads, Geo<MN>::SMEM_BYTES of dynamic shared memory; K a multiple of 256 and splits of
// K a multiple of 8 blocks (stages of 8 whole blocks, 16-byte aligned scale boxes). tm_q:
// codes as bytes [N][K/2], box 128 bytes x 128 rows, 128-byte swizzle; tm_s: scales as
// fp16 [N][K/32], box 8 x 128 rows.
template <int MN>
__global__ void __launch_bounds__(Geo<MN>::NUM_THREADS, 1)
    gemm_i8_kernel(int M, int N, int K, const int8_t* __restrict__ tok, const float* __restrict__ dxs,
                   void* __restrict__ y,
                   const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_s, int bsplit,
                   float* __restrict__ ypart, Epilogue epi) {
    using Gm = Geo<MN>;
    constexpr int S = Gm::S, NR = Gm::NR, NO = Gm::NO, ND = Gm::ND, NG = Gm::NG, GS = Gm::GS, HALVES = Gm::HALVES;
    constexpr int TT = Gm::TT, NW = Gm::NW, CW = Gm::CW;
    constexpr int T_BLK = Gm::T_BLK, DX_BLK = Gm::DX_BLK;
    constexpr int OFF_DX = Gm::OFF_DX;
    constexpr int RAW_BYTES = Gm::RAW_BYTES, OP_BYTES = Gm::OP_BYTES, OFF_OPS = Gm::OFF_OPS;
    constexpr int EPI_WARPS = Gm::EPI_WARPS, PROD_WARP0 = Gm::PROD_WARP0;
    constexpr int MMA_WARP = Gm::MMA_WARP, COPY_WARP = Gm::COPY_WARP, OPC_WARP = Gm::OPC_WARP;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + Gm::OFF_CTRL);
    volatile uint32_t* abort = &ctrl->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = K >> 5;
    // Split of K over blockIdx.z: this CTA contracts blocks [kb0, kb0 + Bl) (bsplit is a
    // multiple of 8) and, when K is split, writes its partial sums to ypart[z].
    const int kb0 = blockIdx.z * bsplit;
    const int Bl = min(B, kb0 + bsplit) - kb0;
    const int nstages = Bl / S;  // Bl is a multiple of 8
    const bool split = gridDim.z > 1;
    float* __restrict__ yp = split ? ypart + size_t(blockIdx.z) * size_t(M) * size_t(N) : nullptr;
    const int n0 = blockIdx.x * NW;
    const int t = blockIdx.y;

    auto raw_ptr = [&](int slot) { return smem + slot * RAW_BYTES; };
    auto op_ptr = [&](int slot) { return smem + OFF_OPS + slot * OP_BYTES; };
    auto es_ptr = [&](int slot) { return smem + OFF_DX + slot * Gm::ES_BYTES; };
    auto bar = [](unsigned long long* p) { return smem_addr(p); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < NR; ++s) {
            mbar_init(bar(&ctrl->raw_full[s]), 1);
            mbar_init(bar(&ctrl->raw_empty[s]), Gm::PROD_WARPS);
        }
        for (int s = 0; s < NO; ++s) {
            mbar_init(bar(&ctrl->op_full[s]), Gm::PROD_WARPS + 1);
            mbar_init(bar(&ctrl->op_empty[s]), 1);
        }
        for (int s = 0; s < ND; ++s) {
            mbar_init(bar(&ctrl->dx_full[s]), 1);
            mbar_init(bar(&ctrl->dx_empty[s]), EPI_WARPS);
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
        // Weight row p of the tile is TMEM lane p: producer warp i writes lanes of quarter
        // i % 4 (the rows 32 (i % 4) .. + 31) for blocks 4 (i / 4) .. + 3 of each stage.
        static_assert(PROD_WARP0 % 4 == 0, "producer warp i must own TMEM lane quarter i % 4");
        const int pw = warp - PROD_WARP0;
        const int p = (pw & 3) * 32 + lane;
        const int kq = (pw >> 2) * Gm::PROD_BLKS;
        const uint32_t a_lane = tmem_base + (uint32_t(warp & 3) << 21) + uint32_t(Gm::A_COL0 + kq * 8);
        for (int st = 0; st < nstages; ++st) {
            const int rs = st % NR, os = st % NO;
            // the slot's previous MMAs are complete and the stage's code box has landed
            if (!bounded_wait2_warp(bar(&ctrl->op_empty[os]), ((st / NO) & 1) ^ 1, bar(&ctrl->raw_full[rs]),
                                    (st / NR) & 1, abort))
                break;
            tc_fence_after();
            const uint8_t* rp = raw_ptr(rs);
            // This warp's four 16-byte chunks of row p of the swizzled box first (independent
            // loads in flight together), then the expansion and one TMEM store.
            uint4 wv[Gm::PROD_BLKS];
#pragma unroll
            for (int k = 0; k < Gm::PROD_BLKS; ++k)
                wv[k] = *reinterpret_cast<const uint4*>(rp + p * 128 + (((kq + k) ^ (p & 7)) << 4));
            uint32_t v[32];
#pragma unroll
            for (int k = 0; k < Gm::PROD_BLKS; ++k) {
                const uint32_t w[4] = {wv[k].x, wv[k].y, wv[k].z, wv[k].w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    v[8 * k + c] = ((w[c] << 4) & 0xF0F0F0F0u) ^ 0x80808080u;  // 16 * (q - 8), elements 4c..4c+3
                    v[8 * k + 4 + c] = (w[c] & 0xF0F0F0F0u) ^ 0x80808080u;     // elements 16+4c..16+4c+3
                }
            }
            // block kq + k: elements 0..31 in columns 8 (kq + k) .. + 7 of the slot
            tmem_st32(a_lane + uint32_t(os * Gm::A_SLOT_COLS), v);
            // The box was read (the store above consumed every load): hand it back. The
            // expanded rows are complete in TMEM before the warp's one arrival.
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(&ctrl->raw_empty[rs]));
                mbar_arrive(bar(&ctrl->op_full[os]));
            }
        }
    } else if (warp == COPY_WARP) {
        // ------------------------------------------------------------ raw code boxes
        // Weights only: not written by the preceding kernel, so no grid wait here.
        const bool leader = elect_one();
        int issued = 0;
        for (int st = 0; st < nstages; ++st) {
            const int rs = st % NR;
            if (!bounded_wait_warp(bar(&ctrl->raw_empty[rs]), ((st / NR) & 1) ^ 1, abort)) break;
            if (leader) {
                const uint32_t rb = bar(&ctrl->raw_full[rs]);
                mbar_arrive_expect_tx(rb, uint32_t(RAW_BYTES));
                tma_load_2d<1>(smem_addr(raw_ptr(rs)), &tm_q, (kb0 + st * S) * 16, n0, rb);
            }
            __syncwarp();
            issued = st + 1;
        }
        for (int st = max(0, issued - NR); st < issued; ++st)
            drain_wait_warp(bar(&ctrl->raw_full[st % NR]), (st / NR) & 1, 200000ull);
    } else if (warp == OPC_WARP) {
        // ------------------------------------------------------------ token codes, scales, d_x
        const bool leader = elect_one();
        if (leader) pdl_wait_primary();  // the token codes and d_x are written by the preceding kernel
        __syncwarp();
        int issued_op = 0, issued_es = 0;
        for (int st = 0; st < nstages; ++st) {
            const int os = st % NO, ds = st % ND;
            const int b0 = kb0 + st * S;
            if (!bounded_wait_warp(bar(&ctrl->op_empty[os]), ((st / NO) & 1) ^ 1, abort)) break;
            // (checked build: the stage's token codes and d_x lie within the operands of
            // gridDim.y token tiles)
            if (leader && in_range((int64_t(t) * B + b0) * T_BLK, S * T_BLK, int64_t(gridDim.y) * B * T_BLK)) {
                const uint32_t fb = bar(&ctrl->op_full[os]);
                mbar_arrive_expect_tx(fb, uint32_t(S * T_BLK));
                bulk_g2s(smem_addr(op_ptr(os)),
                         reinterpret_cast<const uint8_t*>(tok) + (int64_t(t) * B + b0) * T_BLK, uint32_t(S * T_BLK), fb);
            }
            issued_op = st + 1;
            if (!bounded_wait_warp(bar(&ctrl->dx_empty[ds]), ((st / ND) & 1) ^ 1, abort)) break;
            if (leader && in_range((int64_t(t) * B + b0) * TT, S * TT, int64_t(gridDim.y) * B * TT)) {
                const uint32_t db = bar(&ctrl->dx_full[ds]);
                mbar_arrive_expect_tx(db, uint32_t(Gm::ES_BYTES));
                tma_load_2d<2>(smem_addr(es_ptr(ds)), &tm_s, b0, n0, db);
                bulk_g2s(smem_addr(es_ptr(ds) + Gm::SC_BYTES), dxs + (int64_t(t) * B + b0) * TT, uint32_t(S * DX_BLK),
                         db);
            }
            issued_es = st + 1;
            __syncwarp();
        }
        // Let the copies land before the CTA can exit (capped waits after an abort).
        for (int st = max(0, issued_op - NO); st < issued_op; ++st)
            drain_wait_warp(bar(&ctrl->op_full[st % NO]), (st / NO) & 1, 200000ull);
        for (int st = max(0, issued_es - ND); st < issued_es; ++st)
            drain_wait_warp(bar(&ctrl->dx_full[st % ND]), (st / ND) & 1, 200000ull);
    } else if (warp == MMA_WARP) {
        // ------------------------------------------------------------ MMA issue
        const bool leader = elect_one();
        const uint32_t smem0 = smem_addr(smem);
        int gi = 0;  // TMEM group uses so far (group gi % NG, phase (gi / NG) & 1)
        bool ok = true;
        for (int st = 0; st < nstages && ok; ++st) {
            const int os = st % NO;
            if (!bounded_wait_warp(bar(&ctrl->op_full[os]), (st / NO) & 1, abort)) break;
#pragma unroll
            for (int hf = 0; hf < HALVES; ++hf, ++gi) {
                const int g = gi % NG;
                // (with presets, phase 0 of tempty is the epilogue's first preset of the
                // columns; without, the groups start free)
                if (!bounded_wait_warp(bar(&ctrl->tempty[g]), ((gi / NG) & 1) ^ (Gm::PRESET ? 0 : 1), abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (leader) {
                    // Straight-line issue of the group's GS MMAs.
#pragma unroll
                    for (int kk = 0; kk < GS; ++kk) {
                        const int k = hf * GS + kk;
                        const uint32_t a_col = uint32_t(Gm::A_COL0 + os * Gm::A_SLOT_COLS + k * 8);
                        const uint32_t t_addr = smem0 + uint32_t(OFF_OPS + os * OP_BYTES + k * T_BLK);
                        tc_mma_i8_ta(tmem_base + uint32_t((g * GS + kk) * MN), tmem_base + a_col,
                                     smem_desc_kmajor(t_addr, LBO, SBO), Gm::IDESC, Gm::PRESET ? 1u : 0u);
                    }
                    tc_commit(bar(&ctrl->tfull[g]));  // the group's accumulators are complete
                    if (hf == HALVES - 1) tc_commit(bar(&ctrl->op_empty[os]));  // the stage's operands are read
                }
                __syncwarp();
            }
        }
        uint32_t local_abort = 0;
        if (leader) tc_commit(bar(&ctrl->drain));
        __syncwarp();
        bounded_wait_warp(bar(&ctrl->drain), 0, &local_abort);
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;           // TMEM lane quarter
        const int c0 = (warp >> 2) * CW;  // first TMEM column (token) of this warp
        const int r = q * 32 + lane;      // this thread's TMEM lane: weight row within the tile
        // f32 accumulators in pairs (packed f32x2 multiply and FMA: one issue per two outputs)
        unsigned long long acc2[CW / 2];
#pragma unroll
        for (int j = 0; j < CW / 2; ++j) acc2[j] = 0ull;
        const uint32_t lane_base = tmem_base + (uint32_t(q * 32) << 16);
        if (Gm::PRESET) {
            // Preset every accumulator column of this warp, then release the TMEM groups.
            for (int c = 0; c < NG * GS; ++c) tmem_preset<CW>(lane_base + uint32_t(c * MN + c0));
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                for (int g = 0; g < NG; ++g) mbar_arrive(bar(&ctrl->tempty[g]));
        }
        const int n = n0 + r;
        int gi = 0;
        bool ok = true;
        for (int st = 0; st < nstages && ok; ++st) {
            const int ds = st % ND;
            if (!bounded_wait_warp(bar(&ctrl->dx_full[ds]), (st / ND) & 1, abort)) break;
            const uint8_t* dp = es_ptr(ds);
            const uint4 sc = *reinterpret_cast<const uint4*>(dp + r * 16);  // this row's 8 scales (zeros past N)
            const uint32_t scw[4] = {sc.x, sc.y, sc.z, sc.w};
            float dep = 0.0f;
#pragma unroll
            for (int hf = 0; hf < HALVES; ++hf, ++gi) {
                const int g = gi % NG;
                if (!bounded_wait_warp(bar(&ctrl->tfull[g]), (gi / NG) & 1, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < GS; ++kk) {
                    const int k = hf * GS + kk;
                    // d_w / 16 (exact) of block k of the stage
                    const float ws = 0.0625f * __half2float(__ushort_as_half(
                                                   uint16_t((k & 1) ? (scw[k >> 1] >> 16) : (scw[k >> 1] & 0xFFFFu))));
                    const uint32_t ta = lane_base + uint32_t((g * GS + kk) * MN + c0);
                    const float* dxk = reinterpret_cast<const float*>(dp + Gm::SC_BYTES + k * DX_BLK) + c0;
                    const float ncw = -kMagic * ws;  // exact
                    const unsigned long long ws2 = pack2(ws, ws), nc2 = pack2(ncw, ncw);
                    // the tile's columns in chunks of at most 16 (register pressure)
                    constexpr int CH = CW < 16 ? CW : 16;
#pragma unroll
                    for (int c = 0; c < CW; c += CH) {
                        uint32_t pr[CH];
                        tmem_cols(ta + uint32_t(c), pr);
#pragma unroll
                        for (int j = 0; j < CH; j += 4) {
                            const float4 dv = *reinterpret_cast<const float4*>(dxk + c + j);  // broadcast
                            // acc += round(D16 * ws) * d_x (the words as floats 1.5 * 2^23 + D16)
                            constexpr uint32_t add = Gm::PRESET ? 0u : kMagicBits;
                            fma2_magic(acc2[(c + j) / 2], pr[j] + add, pr[j + 1] + add, dv.x, dv.y, ws2, nc2);
                            fma2_magic(acc2[(c + j) / 2 + 1], pr[j + 2] + add, pr[j + 3] + add, dv.z, dv.w, ws2,
                                       nc2);
                        }
                    }
                    if (Gm::PRESET) tmem_preset<CW>(ta);  // for the tile's next use
                    if (kk == GS - 1) {  // the group's tiles are all read (and preset): free it
                        if (Gm::PRESET) tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(&ctrl->tempty[g]));
                    }
                    dep = fmaf(dxk[0], ws, dep);  // depends on this block's scale and d_x loads
                }
            }
            if (!ok) break;
            // The stage's scales and d_x were read (the arrive waits for `dep`, which depends
            // on the last of those loads): hand the slot back.
            __syncwarp();
            if (lane == 0) mbar_arrive_after(bar(&ctrl->dx_empty[ds]), dep);
        }
        float acc[CW];
#pragma unroll
        for (int j = 0; j < CW / 2; ++j) unpack2(acc2[j], acc[2 * j], acc[2 * j + 1]);
        if (!*abort) {
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

    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Gm::TMEM_COLS);
    }
}

}  // namespace i8

// Q8_0 quantisation of x into the int8 MMA's token operand: per token tile t (tt tokens)
// and block b a chunk of tt x 32 codes in element order, K-major core matrices (token r,
// 16-byte half c at (r/8)*256 + c*128 + (r%8)*16), at tok + (t*B + b) * tt * 32; d_x at
// dxs[(t*B + b)*tt + r]. Eight threads per block (four elements each); tokens past M get
// zero codes and scales. The arithmetic is quant_act_rowmajor_kernel's.
template <bool BF16>
__global__ void __launch_bounds__(256) quant_act_i8_kernel(const void* __restrict__ x, int M, int K, int tt,
                                                           int64_t nblocks, int8_t* __restrict__ tok,
                                                           float* __restrict__ dxs) {
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
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int qi = static_cast<int>(roundf(__fmul_rn(v[i], id)));
        qi = max(-127, min(127, qi));
        packed |= (uint32_t(qi) & 0xFFu) << (8 * i);
    }
    const int64_t t = m / tt;
    const int r = int(m - t * tt);
    const int64_t chunk = t * B + b;
    if (valid) {
        char* dst = reinterpret_cast<char*>(tok) + chunk * i8::tok_block_bytes(tt) + (r >> 3) * 256 + (sub >> 2) * 128 +
                    (r & 7) * 16 + (sub & 3) * 4;
        *reinterpret_cast<uint32_t*>(dst) = packed;
        if (sub == 0) dxs[chunk * tt + r] = d;
    }
}

}  // namespace w4a8
