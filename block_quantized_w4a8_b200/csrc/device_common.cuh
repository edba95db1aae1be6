// Device-side helpers shared by the libw4a8 kernels: inline-PTX wrappers for mbarriers,
// bulk async copies, programmatic dependent launch and the tcgen05 tensor-core / tensor
// memory instructions of sm_100a, plus the bounded waits every pipeline uses.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace w4a8 {

// Bit set in the device status word when a bounded wait ran out.
constexpr unsigned kDevErrTimeout = 1u;
// Bit set by a device-side check of the checked build (W4A8_CHECKED) that failed.
constexpr unsigned kDevErrChecked = 4u;
// Upper bound on any single wait inside a kernel (ns of %globaltimer).
constexpr unsigned long long kWaitLimitNs = 1500000000ull;

// Device status word, read and cleared by w4a8_last_device_error().
__device__ unsigned int g_device_status = 0;

// Checked build (compiled with -DW4A8_CHECKED): device-side checks of the conditions a
// copy needs to be legal (alignment of TMA coordinates and bulk-copy addresses and sizes).
// A failed check records kDevErrChecked and the copy is skipped, so the waiting barrier
// runs out into the bounded-wait error path instead of the copy faulting the GPU. In the
// default build `checked` is the constant true and the checks compile away.
#ifdef W4A8_CHECKED
constexpr bool kCheckedBuild = true;
#else
constexpr bool kCheckedBuild = false;
#endif
__device__ __forceinline__ bool checked(bool ok) {
    if (kCheckedBuild && !ok) {
        atomicOr(&g_device_status, kDevErrChecked);
        return false;
    }
    return true;
}

// Checked build: the element range [off, off + len) of an operand lies within its extent
// (the copy or access is skipped and kDevErrChecked recorded otherwise).
__device__ __forceinline__ bool in_range(long long off, long long len, long long extent) {
    return checked(off >= 0 && len >= 0 && off + len <= extent);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Arrive after `dep` has been computed: passing a value derived from earlier shared-memory
// loads makes the arrive wait for those loads to return, so the buffer they read can be
// handed back before the values are used.
__device__ __forceinline__ void mbar_arrive_after(uint32_t bar, float dep) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar), "f"(dep) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// Suspend-time hint for try_wait (ns): the waiting thread sleeps in hardware until the
// phase completes or the hint runs out, instead of spinning on shared memory.
constexpr uint32_t kTryWaitHintNs = 1000000u;

// CLUSTER: acquire at cluster scope, for barriers that other CTAs of the cluster arrive on.
template <bool CLUSTER = false>
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    if (CLUSTER)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(ok)
            : "r"(bar), "r"(parity), "r"(kTryWaitHintNs)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(ok)
            : "r"(bar), "r"(parity), "r"(kTryWaitHintNs)
            : "memory");
    return ok != 0;
}
// Probe without a suspend hint: on a completed phase it returns in a fraction of the
// time of the hinted form, so every wait checks this way first.
template <bool CLUSTER = false>
__device__ __forceinline__ bool mbar_try_wait_nohint(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    if (CLUSTER)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
    return ok != 0;
}

// Wait until the phase with parity `parity` of barrier `bar` has completed. Gives up
// when `*abort` is raised by another thread or after kWaitLimitNs; in the latter case
// it records kDevErrTimeout in the device status word and raises `*abort` itself.
// Returns false when it gave up. Called by one thread.
__device__ __noinline__ bool bounded_wait_slow(uint32_t bar, uint32_t parity, volatile uint32_t* abort) {
    const unsigned long long t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 0u) {
            if (*abort) return false;
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                atomicOr(&g_device_status, kDevErrTimeout);
                *abort = 1u;
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool bounded_wait(uint32_t bar, uint32_t parity, volatile uint32_t* abort) {
    if (mbar_try_wait_nohint(bar, parity)) return true;
    return bounded_wait_slow(bar, parity, abort);
}

// Warp-wide wait: every lane probes the barrier and a vote makes the outcome uniform
// (phase completion is monotonic, so a lane that saw it keeps seeing it), so the warp
// never diverges. Same limits as bounded_wait (`limit_ns` other than kWaitLimitNs only in
// the self-test of the waits). All 32 lanes must call it.
template <bool CLUSTER = false>
__device__ __noinline__ bool bounded_wait_warp_slow(uint32_t bar, uint32_t parity, volatile uint32_t* abort,
                                                    unsigned long long limit_ns = kWaitLimitNs) {
    const unsigned long long t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (__all_sync(0xffffffffu, mbar_try_wait<CLUSTER>(bar, parity))) return true;
        if ((it & 15u) == 0u) {
            uint32_t stop = *abort;
            if (!stop && global_timer_ns() - t0 > limit_ns) stop = 2u;
            stop = __shfl_sync(0xffffffffu, stop, 0);
            if (stop) {
                if (stop == 2u && (threadIdx.x & 31u) == 0u) {
                    atomicOr(&g_device_status, kDevErrTimeout);
                    *abort = 1u;
                }
                return false;
            }
        }
    }
}
template <bool CLUSTER = false>
__device__ __forceinline__ bool bounded_wait_warp(uint32_t bar, uint32_t parity, volatile uint32_t* abort,
                                                  unsigned long long limit_ns = kWaitLimitNs) {
    if (__all_sync(0xffffffffu, mbar_try_wait_nohint<CLUSTER>(bar, parity))) return true;
    return bounded_wait_warp_slow<CLUSTER>(bar, parity, abort, limit_ns);
}

// Self-test of the bounded waits (the failure path of every pipeline): warp 0 waits with
// limit `limit_ns` on a barrier that nothing arrives at; warp 1 waits on another such
// barrier with the production limit and must stop through the abort flag that warp 0
// raises when its wait runs out. Nothing else is in flight. Bits of *outcome: 1 = warp 0
// gave up, 2 = warp 1 gave up, 4 = warp 1 stopped within 100 ms of starting. One CTA of
// 64 threads.
__global__ void __launch_bounds__(64, 1) selftest_wait_kernel(unsigned long long limit_ns, unsigned int* outcome) {
    __shared__ __align__(8) unsigned long long bars[2];
    __shared__ uint32_t abort_flag;
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bars[0]), 1);
        mbar_init(smem_addr(&bars[1]), 1);
        abort_flag = 0;
        mbar_init_fence();
    }
    __syncthreads();
    const unsigned long long t0 = global_timer_ns();
    const bool ok = bounded_wait_warp(smem_addr(&bars[warp]), 0, &abort_flag, warp == 0 ? limit_ns : kWaitLimitNs);
    const unsigned long long t1 = global_timer_ns();
    if ((threadIdx.x & 31u) == 0u) {
        unsigned int bits = ok ? 0u : (warp == 0 ? 1u : 2u);
        if (warp == 1 && !ok && t1 - t0 < 100000000ull) bits |= 4u;
        atomicOr(outcome, bits);
    }
}

// Warp-wide wait for two barriers: both probed at once on the fast path (one round trip
// when both phases are already complete), else each waited for in turn.
__device__ __forceinline__ bool bounded_wait2_warp(uint32_t bar1, uint32_t parity1, uint32_t bar2, uint32_t parity2,
                                                   volatile uint32_t* abort) {
    const bool a = mbar_try_wait_nohint(bar1, parity1);
    const bool b = mbar_try_wait_nohint(bar2, parity2);
    if (__all_sync(0xffffffffu, a && b)) return true;
    return bounded_wait_warp(bar1, parity1, abort) && bounded_wait_warp(bar2, parity2, abort);
}

// Named hardware barrier over `nthreads` threads (whole warps); waiting warps issue
// nothing until the last one arrives.
__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Warp-wide wait used only to drain asynchronous copies before a CTA exits: waits up to
// `limit_ns` and reports nothing (the caller has already recorded why it stopped).
__device__ __noinline__ void drain_wait_warp(uint32_t bar, uint32_t parity, unsigned long long limit_ns) {
    const unsigned long long t0 = global_timer_ns();
    while (!__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) {
        uint32_t stop = (global_timer_ns() - t0 > limit_ns) ? 1u : 0u;
        if (__shfl_sync(0xffffffffu, stop, 0)) return;
    }
}

// True in exactly one lane of the (converged) warp: the lowest active lane.
__device__ __forceinline__ bool elect_one() {
    uint32_t pred;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(pred));
    return pred != 0;
}

// ------------------------------------------------------------------ bulk async copy
// Global -> shared copy of `bytes` (multiple of 16, both addresses 16-byte aligned)
// that completes `bytes` transactions on mbarrier `bar`, into this CTA's shared memory only.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    if (!checked((dst & 15u) == 0 && (reinterpret_cast<uintptr_t>(src) & 15u) == 0 && (bytes & 15u) == 0)) return;
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// 2-D tiled tensor copy (TMA) global -> shared of one box of the tensor map at `tmap`
// (a __grid_constant__ kernel parameter), box origin (c0 = innermost, c1), completing its
// bytes on mbarrier `bar`, into this CTA's shared memory only. c0 times the element size must be a
// multiple of 16 bytes (ESIZE = the element size in bytes, checked in the checked
// build); parts of the box outside the tensor are filled with zeros.
template <int ESIZE>
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int c0, int c1, uint32_t bar) {
    if (!checked(((c0 * ESIZE) & 15) == 0 && (dst & 15u) == 0)) return;
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(dst),
        "l"(tmap), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ output epilogue
// What the contraction kernels store: y[m][n] = product + bias[n] (one f32 addition, the
// bias of a linear layer as in the C-Kernel-Engine Q4_K GEMM wrapper), written as f32 or
// rounded to bf16 (round to nearest even). Without a bias the product is stored as is.
struct Epilogue {
    const void* bias;  // N values, or nullptr
    int bias_bf16;     // bias elements: 0 = f32, 1 = bf16
    int out_bf16;      // y elements: 0 = f32, 1 = bf16
};
__device__ __forceinline__ float epi_value(const Epilogue& e, int n, float v) {
    if (!e.bias) return v;
    const float b = e.bias_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(e.bias)[n])
                                : reinterpret_cast<const float*>(e.bias)[n];
    return __fadd_rn(v, b);
}
// y[idx] for output column n.
__device__ __forceinline__ void epi_store(void* y, int64_t idx, int n, float v, const Epilogue& e) {
    const float r = epi_value(e, n, v);
    if (e.out_bf16)
        reinterpret_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(r);
    else
        reinterpret_cast<float*>(y)[idx] = r;
}
// y[idx .. idx+3] for columns n .. n+3 of one row (idx a multiple of 4: one 16-byte f32
// or 8-byte bf16 store).
__device__ __forceinline__ void epi_store4(void* y, int64_t idx, int n, float a, float b, float c, float d,
                                           const Epilogue& e) {
    a = epi_value(e, n, a);
    b = epi_value(e, n + 1, b);
    c = epi_value(e, n + 2, c);
    d = epi_value(e, n + 3, d);
    if (e.out_bf16) {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
        uint2 v;
        v.x = *reinterpret_cast<const uint32_t*>(&lo);
        v.y = *reinterpret_cast<const uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(y) + idx) = v;
    } else {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(y) + idx) = make_float4(a, b, c, d);
    }
}

// ------------------------------------------------------------------ PDL
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait_primary() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// The same for a CTA pair (cta_group::2): one warp of each CTA of the pair executes it,
// and the pair's tensor memory is allocated at the same columns in both CTAs.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrive once on `bar` when every tcgen05 operation this thread issued so far is done.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, both K-major, f16 inputs, f32 accumulator.
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// CTA-pair MMA, issued by one thread of the even CTA: M = 256 rows of A, 128 from each
// CTA's shared memory at the descriptor's address; B's N columns split in halves, the
// first half staged by the even CTA, the second by the odd one; each CTA's tensor memory
// receives its own 128 rows of D (all N columns).
__device__ __forceinline__ void tc_mma_f16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on the barrier at offset `bar` in each CTA of `cta_mask` when the pair MMAs
// this thread issued so far are done.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            bar),
        "h"(cta_mask)
        : "memory");
}

// ------------------------------------------------------------------ clusters
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Barrier over all threads of all CTAs of the cluster (release/acquire at cluster scope).
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Shared-memory address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
// Remote arrive with the default (CTA-scope) release: enough to signal that tensor-memory
// reads ordered before it by tcgen05.fence::before_thread_sync are done. The cluster-
// scope release costs several hundred cycles more per arrival.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t remote_bar) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(remote_bar) : "memory");
}

// Shared-memory matrix descriptor for a K-major operand without swizzle: core matrices
// of 8 rows x 16 bytes stored contiguously (128 B); `lbo` = byte distance between core
// matrices adjacent along K, `sbo` = between core matrices adjacent along M/N.
__device__ __forceinline__ uint64_t smem_desc_kmajor(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
           (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46);
}

// Instruction descriptor, kind::f16: A and B f16, D f32, both K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
    return (1u << 4)                          // D format f32
           | (0u << 7) | (0u << 10)           // A, B format f16
           | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// 32 lanes x 32 columns of 32-bit words from tensor memory; lane i of the warp gets row
// (lane base + i). The registers are valid only after tmem_wait_ld(r).
__device__ __forceinline__ void tmem_ld_32x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
// Waits for this thread's outstanding tensor-memory loads. The registers are threaded
// through the asm so that no use of them can be scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                   "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                   "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

// 32 lanes x 64 columns in one instruction (registers valid after tmem_wait_ld64).
__device__ __forceinline__ void tmem_ld_32x32_x64(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
        "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
          "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
          "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
          "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
          "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld64(uint32_t (&r)[64]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                   "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                   "+r"(r[29]), "+r"(r[30]), "+r"(r[31]), "+r"(r[32]), "+r"(r[33]), "+r"(r[34]), "+r"(r[35]),
                   "+r"(r[36]), "+r"(r[37]), "+r"(r[38]), "+r"(r[39]), "+r"(r[40]), "+r"(r[41]), "+r"(r[42]),
                   "+r"(r[43]), "+r"(r[44]), "+r"(r[45]), "+r"(r[46]), "+r"(r[47]), "+r"(r[48]), "+r"(r[49]),
                   "+r"(r[50]), "+r"(r[51]), "+r"(r[52]), "+r"(r[53]), "+r"(r[54]), "+r"(r[55]), "+r"(r[56]),
                   "+r"(r[57]), "+r"(r[58]), "+r"(r[59]), "+r"(r[60]), "+r"(r[61]), "+r"(r[62]), "+r"(r[63])
                 :
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15])
                 :
                 : "memory");
}

// 32 lanes x 16 columns (registers valid after the next tcgen05.wait::ld).
__device__ __forceinline__ void tmem_ld_32x32_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
// Two floats as one 64-bit register pair (the operand of packed f32x2 instructions) and back.
__device__ __forceinline__ unsigned long long pack2(float a, float b) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void unpack2(unsigned long long v, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}

// ------------------------------------------------------------------ misc
__device__ __forceinline__ float warp_max8(float v) {  // max over aligned groups of 8 lanes
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
    return v;
}
// log2 of the 32-blocks per affine group (groups of 32, 64 or 128): block index b lies
// in group b >> group_shift(group), without a run-time division.
__host__ __device__ __forceinline__ int group_shift(int group) { return group == 128 ? 2 : (group == 64 ? 1 : 0); }

__device__ __forceinline__ int warp_sum8(int v) {
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    return v;
}

// Four consecutive input elements (16 B of f32 or 8 B of bf16) widened to f32.
template <bool BF16>
__device__ __forceinline__ void load4(const void* base, int64_t idx, float (&v)[4]) {
    if constexpr (BF16) {
        const uint2 u = *reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(base) + idx);
        __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
        __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
        v[0] = __low2float(a); v[1] = __high2float(a); v[2] = __low2float(b); v[3] = __high2float(b);
    } else {
        const float4 f = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx);
        v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    }
}

}  // namespace w4a8
