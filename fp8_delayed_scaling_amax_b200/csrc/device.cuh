// Device-side building blocks for sm_100a: shared-memory barriers, TMA bulk-tensor loads,
// tcgen05 (5th-generation tensor core) MMA / TMEM access, fp8 conversion, and the bounded
// waits every kernel of this library uses so that a pipeline bug stalls into an error
// status instead of hanging the GPU.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cstdint>

namespace fp8dsa {

// Status codes a kernel may leave in the device status word.
enum DeviceStatus : int {
    kStatusOk = 0,
    kStatusWaitProducer = 0x101,   // GEMM producer gave up waiting for a free stage
    kStatusWaitMma = 0x102,        // GEMM MMA warp gave up waiting for operands / accumulator
    kStatusWaitEpilogue = 0x103,   // GEMM epilogue gave up waiting for an accumulator
    kStatusWaitDrain = 0x104,      // a drain wait (in-flight copies / MMAs) gave up
    kStatusWaitQuantize = 0x105,   // tiled quantize gave up waiting for an input tile
    kStatusWaitSplit = 0x106,      // split-K owner gave up waiting for its partial sums
    kStatusWaitDebug = 0x1FF,      // the deliberate stalled-wait test hook
};

// Where a kernel reports a bounded-wait expiry, and how long it may wait.
struct WaitCtl {
    int* status;                    // device status word (global memory)
    unsigned long long timeout_ns;  // upper bound of any single wait
};

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Programmatic dependent launch: let the next kernel on the stream start launching (its CTAs
// still wait in pdl_wait for this grid to finish and flush), and wait for the previous one.
// Both are no-ops when the launch carried no programmatic dependency.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void report_status(const WaitCtl& ctl, int code) {
    if (ctl.status) atomicCAS(ctl.status, 0, code);
}

// ---------------------------------------------------------------------------------------
// mbarrier (shared-memory transaction barrier)
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait for the phase with the given parity to complete.  Returns false (and raises
// `abort_flag`, and records `code` in the status word) if the wait outlives the timeout, or
// returns false at once if another role already raised `abort_flag`.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  const WaitCtl& ctl, volatile int* abort_flag,
                                                  int code) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (abort_flag != nullptr && *abort_flag) return false;
        if (global_timer_ns() - t0 > ctl.timeout_ns) {
            report_status(ctl, code);
            if (abort_flag != nullptr) *abort_flag = 1;
            return false;
        }
    }
}

// ---------------------------------------------------------------------------------------
// TMA: 3-D tiled bulk-tensor load global -> shared, completing on an mbarrier.
// (No multicast anywhere in this library.)
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_addr(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// 3-D tiled bulk-tensor store shared -> global (bulk-group completion).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* smem_src, int c0, int c1,
                                             int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(smem_addr(smem_src)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N committed bulk groups still read their shared-memory source.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until every committed bulk group has completed.
__device__ __forceinline__ void bulk_wait_group_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Order this thread's generic-proxy shared-memory writes before later async-proxy (TMA) reads.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------------------
// tcgen05: TMEM allocation, MMA issue, commit, loads and ordering fences.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(smem_result)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]; fp8 x fp8 -> fp32, one CTA, issued by one thread.
__device__ __forceinline__ void umma_f8f6f4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tc_fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Warp-collective: each lane reads 32 consecutive 32-bit columns of its TMEM lane.
__device__ __forceinline__ void tmem_load_32cols(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32"
        " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
        " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31},"
        " [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Named barrier among a subset of warps (ids 1..15; 0 is __syncthreads).
__device__ __forceinline__ void named_barrier(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Device-scope release increment / acquire load of a global counter (split-K hand-off).
__device__ __forceinline__ void counter_add_release(uint32_t* p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t counter_load_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Wait until *p >= target (device-scope acquire).  Returns false, raising `abort_flag` and
// recording `code`, if that takes longer than the timeout, or at once if `abort_flag` is
// already raised.
__device__ __forceinline__ bool counter_wait_bounded(const uint32_t* p, uint32_t target, const WaitCtl& ctl,
                                                     volatile int* abort_flag, int code) {
    if (counter_load_acquire(p) >= target) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        __nanosleep(64);
        if (counter_load_acquire(p) >= target) return true;
        if (abort_flag != nullptr && *abort_flag) return false;
        if (global_timer_ns() - t0 > ctl.timeout_ns) {
            report_status(ctl, code);
            if (abort_flag != nullptr) *abort_flag = 1;
            return false;
        }
    }
}

// ---------------------------------------------------------------------------------------
// CTA pairs (2-CTA clusters): one MMA spans both SMs' tensor cores, M = 256.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Shared::cluster address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// All threads of both CTAs: release this CTA's prior writes, wait for the peer.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on an mbarrier in another CTA of the cluster (cluster-scope release).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// As mbar_wait_bounded, with cluster-scope acquire (for barriers other CTAs arrive on).
__device__ __forceinline__ bool mbar_wait_bounded_cluster(uint64_t* bar, uint32_t parity, const WaitCtl& ctl,
                                                          volatile int* abort_flag, int code) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait_cluster(bar, parity)) return true;
        if (abort_flag != nullptr && *abort_flag) return false;
        if (global_timer_ns() - t0 > ctl.timeout_ns) {
            report_status(ctl, code);
            if (abort_flag != nullptr) *abort_flag = 1;
            return false;
        }
    }
}

// Pair TMA load: writes this CTA's shared memory and completes bytes on the mbarrier at
// `mbar_cluster_addr` (the leader CTA's barrier).  No multicast.
__device__ __forceinline__ void tma_load_3d_pair(void* smem_dst, const CUtensorMap* map, uint32_t mbar_cluster_addr,
                                                 int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_addr(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(mbar_cluster_addr), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_result, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(smem_result)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Pair MMA (M = 256 across both CTAs), issued by one thread of the leader CTA.
__device__ __forceinline__ void umma_f8f6f4_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on the barrier at this offset in every CTA of `cta_mask` once the pair MMAs this
// thread issued have completed.
__device__ __forceinline__ void umma_commit_pair_multicast(uint64_t* bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_addr(bar)),
        "h"(cta_mask)
        : "memory");
}

__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

// ---------------------------------------------------------------------------------------
// fp8 conversion: two fp32 -> two fp8 bytes (round to nearest even, saturate to finite).
// Result byte 0 = lo, byte 1 = hi.
// ---------------------------------------------------------------------------------------
template <int kFmt>
__device__ __forceinline__ uint32_t cvt_fp8x2(float lo, float hi) {
    uint16_t r;
    if constexpr (kFmt == 0)
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    else
        asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Four fp32 -> one packed word, element 0 in the lowest byte.
template <int kFmt>
__device__ __forceinline__ uint32_t cvt_fp8x4(float a, float b, float c, float d) {
    return cvt_fp8x2<kFmt>(a, b) | (cvt_fp8x2<kFmt>(c, d) << 16);
}

// One fp8 byte -> fp32 (exact), through the packed fp8x2 -> f16x2 conversion.
template <int kFmt>
__device__ __forceinline__ float fp8_to_float(uint8_t v) {
    uint32_t h2;
    const uint16_t in = v;
    if constexpr (kFmt == 0)
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    else
        asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h2) : "h"(in));
    const uint16_t lo = static_cast<uint16_t>(h2 & 0xFFFFu);
    return __half2float(__ushort_as_half(lo));
}

// Packed running maximum of |x| over two bf16 (resp. f16) lanes: each lane of the result has
// magnitude max(|acc|, |v|) (its sign is the xor of the operands' signs and carries no
// meaning); a NaN operand lane returns the other lane's value, so NaN never enters.
__device__ __forceinline__ uint32_t max_abs_bf16x2(uint32_t acc, uint32_t v) {
    uint32_t r;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(acc), "r"(v));
    return r;
}
__device__ __forceinline__ uint32_t max_abs_f16x2(uint32_t acc, uint32_t v) {
    uint32_t r;
    asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(r) : "r"(acc), "r"(v));
    return r;
}

// a = RN32(a * m), b = RN32(b * m) in one packed instruction.
__device__ __forceinline__ void mul2_rn(float& a, float& b, float m) {
    unsigned long long p, q;
    asm("mov.b64 %0, {%1, %2};" : "=l"(p) : "f"(a), "f"(b));
    asm("mov.b64 %0, {%1, %1};" : "=l"(q) : "f"(m));
    asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(p) : "l"(q));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(p));
}

// a = RN32(a + c), b = RN32(b + d) in one packed instruction.
__device__ __forceinline__ void add2_rn(float& a, float& b, float c, float d) {
    unsigned long long p, q;
    asm("mov.b64 %0, {%1, %2};" : "=l"(p) : "f"(a), "f"(b));
    asm("mov.b64 %0, {%1, %2};" : "=l"(q) : "f"(c), "f"(d));
    asm("add.rn.f32x2 %0, %0, %1;" : "+l"(p) : "l"(q));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(p));
}

// a = RN32(a * m + c), b = RN32(b * m + c) (fused, one rounding each) in one packed instruction.
__device__ __forceinline__ void fma2_rn(float& a, float& b, float m, float c) {
    unsigned long long p, q, r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(p) : "f"(a), "f"(b));
    asm("mov.b64 %0, {%1, %1};" : "=l"(q) : "f"(m));
    asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(c));
    asm("fma.rn.f32x2 %0, %0, %1, %2;" : "+l"(p) : "l"(q), "l"(r));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(p));
}

// History-ring fold done after the quantize kernel that measured the amax (one thread; the
// quantize blocks only left their maxima in the amax slot).  Ring layout [hist n | scale |
// scale_used | amax | done]: scale_used = the step the quantize used (the current scale),
// hist[idx] = amax, scale = max(RN32(RN32(peak / fp8_max) / pow2_margin), 1e-12) over the
// window, amax slot re-zeroed -- the same state the in-kernel fold leaves.
__device__ __forceinline__ void ring_fold_deferred(float* st, int n, int idx, float fp8_max, float pow2_margin) {
    const float step = __ldcg(st + n);
    const float am = __ldcg(st + n + 2);
    float peak = am;
    for (int i = 0; i < n; ++i)
        if (i != idx) peak = fmaxf(peak, __ldcg(st + i));
    st[n + 1] = step;
    st[idx] = am;
    st[n] = fmaxf(__fdiv_rn(__fdiv_rn(peak, fp8_max), pow2_margin), 1e-12f);
    st[n + 2] = 0.0f;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) {
    return __uint_as_float(b << 16);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

}  // namespace fp8dsa
