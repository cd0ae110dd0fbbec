// dsa_device.cuh -- device-side building blocks for the sm_100a kernels:
// status word, sequence lookup, bounded mbarrier waits, tcgen05 (TMEM, MMA),
// TMA and cluster (DSMEM) wrappers in inline PTX.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "dsa.h"

#define DSA_DEV __device__ __forceinline__

namespace dsa {

// ---------------------------------------------------------------------------
// Workspace status header: int32 code at byte 0, int64 detail at byte 8.
// The first error wins.
// ---------------------------------------------------------------------------
struct StatusHdr {
    int code;
    int pad;
    long long detail;
};

DSA_DEV void report(StatusHdr* st, int code, long long detail) {
    if (atomicCAS(&st->code, 0, code) == 0) atomicExch((unsigned long long*)&st->detail, (unsigned long long)detail);
}

// ---------------------------------------------------------------------------
// Sequence lookup: the sequence b holding packed query row t, binary search
// over cu_seqlens_q (batch is small).
// ---------------------------------------------------------------------------
struct SeqView {
    int batch;
    const int64_t* cu_q;
    const int64_t* cu_k;
};

struct RowInfo {
    int b;
    int64_t key_base;  // packed row of the sequence's key 0
    int64_t seqlen_k;
    int64_t pos;       // position of this query in its sequence
    bool ok;
};

DSA_DEV RowInfo row_info(const SeqView& sv, int64_t t) {
    int lo = 0, hi = sv.batch - 1;
    while (lo < hi) {  // largest b with cu_q[b] <= t
        int mid = (lo + hi + 1) >> 1;
        if (__ldg(sv.cu_q + mid) <= t) lo = mid; else hi = mid - 1;
    }
    RowInfo r;
    r.b = lo;
    int64_t q0 = __ldg(sv.cu_q + lo), q1 = __ldg(sv.cu_q + lo + 1);
    int64_t k0 = __ldg(sv.cu_k + lo), k1 = __ldg(sv.cu_k + lo + 1);
    r.key_base = k0;
    r.seqlen_k = k1 - k0;
    r.pos = (k1 - k0) - (q1 - q0) + (t - q0);
    r.ok = (t >= q0 && t < q1 && r.pos >= 0 && r.pos < r.seqlen_k);
    return r;
}

// ---------------------------------------------------------------------------
// Shared-memory addresses and mbarriers
// ---------------------------------------------------------------------------
DSA_DEV uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

DSA_DEV void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
DSA_DEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
DSA_DEV void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

DSA_DEV void mbar_arrive(uint32_t bar) {
    asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(bar) : "memory");
}
DSA_DEV void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// 16-byte asynchronous copy global -> shared (L2 only), and an arrive on `bar`
// once every cp.async of this thread issued so far has landed (the arrival
// is counted in the barrier's expected count).
DSA_DEV void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"((uint64_t)src) : "memory");
}
DSA_DEV void cp_async_arrive(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
DSA_DEV void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }" ::"r"(bar), "r"(bytes)
                 : "memory");
}
// Arrive on an mbarrier of another CTA of the cluster (cluster-space address
// from mapa).  Used to hand a buffer back to the peer that fills it: this
// thread's reads of the buffer are ordered before the arrive.
DSA_DEV void mbar_arrive_remote(uint32_t cluster_bar) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

DSA_DEV bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
// Non-blocking probe (test_wait never suspends the thread), for loops that
// poll several barriers in turn.
DSA_DEV bool mbar_probe(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
DSA_DEV bool mbar_test_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}

// Default budget of a bounded wait, in SM clock cycles (~1-2 s).  Every wait
// in these kernels is bounded: when it runs out the kernel records
// DSA_ERR_TIMEOUT, raises its CTA-wide abort flag and winds down.
constexpr long long kWaitBudget = 1ll << 31;

// Wait for the phase of `bar` with parity `parity`.  Returns false when the
// budget ran out, when *abort is raised (another role of this CTA gave up),
// or when the workspace already records a timeout (another CTA gave up), so a
// failed launch winds down in about one budget instead of one per CTA.
template <bool CLUSTER>
DSA_DEV bool mbar_wait_impl(uint32_t bar, uint32_t parity, volatile int* abort, StatusHdr* st, int where,
                            long long budget) {
    auto test = [&] { return CLUSTER ? mbar_test_cluster(bar, parity) : mbar_test(bar, parity); };
    if (test()) return true;
    const long long t0 = clock64();
    for (uint32_t it = 1;; ++it) {
        if (test()) return true;
        if (abort && *abort) return false;
        if ((it & 15) == 0) {
            const long long el = clock64() - t0;
            // the global header is only read once a wait is already long
            if (el > (1ll << 20) && st && *(volatile int*)&st->code == DSA_ERR_TIMEOUT) {
                if (abort) *abort = 1;
                return false;
            }
            if (el > budget) {
                report(st, DSA_ERR_TIMEOUT, where);
                if (abort) *abort = 1;
                return false;
            }
        }
    }
}
DSA_DEV bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort, StatusHdr* st, int where,
                       long long budget = kWaitBudget) {
    return mbar_wait_impl<false>(bar, parity, abort, st, where, budget);
}
DSA_DEV bool mbar_wait_cluster(uint32_t bar, uint32_t parity, volatile int* abort, StatusHdr* st, int where,
                               long long budget = kWaitBudget) {
    return mbar_wait_impl<true>(bar, parity, abort, st, where, budget);
}

// Warp-uniform forms: every lane polls (and so acquires), and the warp agrees
// on the outcome, so control flow never diverges on a wait.
DSA_DEV bool wait_warp(uint32_t bar, uint32_t parity, volatile int* abort, StatusHdr* st, int where) {
    const bool ok = mbar_wait(bar, parity, abort, st, where);
    return __all_sync(0xffffffffu, ok);
}
DSA_DEV bool wait_warp_cluster(uint32_t bar, uint32_t parity, volatile int* abort, StatusHdr* st, int where) {
    const bool ok = mbar_wait_cluster(bar, parity, abort, st, where);
    return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------------------
// Cluster / DSMEM
// ---------------------------------------------------------------------------
DSA_DEV uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
DSA_DEV uint32_t mapa(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}
DSA_DEV void st_cluster_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}
// Store into another CTA's shared memory and count the bytes on its
// mbarrier (complete_tx): the data is visible once that phase completes.
DSA_DEV void st_async_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint32_t remote_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(addr),
                 "r"(a), "r"(b), "r"(c), "r"(d), "r"(remote_bar)
                 : "memory");
}
DSA_DEV void st_async_b32(uint32_t addr, uint32_t a, uint32_t remote_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(addr), "r"(a),
                 "r"(remote_bar)
                 : "memory");
}
// Hint: bring the 128-byte line holding p into L2.
DSA_DEV void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"((uint64_t)p)); }
DSA_DEV void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMA: plain tiled loads and row gathers into this CTA's own shared memory
// ---------------------------------------------------------------------------
DSA_DEV void tma_prefetch_desc(const CUtensorMap* m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)m) : "memory");
}
DSA_DEV void tma_load_2d(uint32_t dst, const CUtensorMap* m, int32_t x, int32_t y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"((uint64_t)m), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
// Contiguous bytes global -> this CTA's shared memory (both 16-byte aligned,
// size a multiple of 16), counted on `bar`.
DSA_DEV void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"((uint64_t)src), "r"(bytes), "r"(bar)
                 : "memory");
}
// ---------------------------------------------------------------------------
// tcgen05: tensor memory, MMA, loads/stores
// ---------------------------------------------------------------------------
DSA_DEV void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
DSA_DEV void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory"); }
DSA_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
DSA_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
DSA_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor, K-major or MN-major, 128-byte swizzle:
// start address, leading/stride byte offsets (>>4), version 1 (sm_100),
// layout type 2 (SWIZZLE_128B).
DSA_DEV uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Shared-memory matrix descriptor, no swizzle (8-row x 16-byte core
// matrices stored as 128 contiguous bytes).  K-major: lbo = bytes between
// core matrices along K, sbo = bytes between core matrices along M/N.
DSA_DEV uint64_t sdesc_noswz(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;
    return d;
}

// Instruction descriptor, dense, fp32 accumulate.
//   kind::f16    : a/b format 1 = BF16
//   kind::f8f6f4 : a/b format 0 = E4M3
__host__ __device__ constexpr uint32_t idesc_make(uint32_t a_fmt, uint32_t b_fmt, bool b_mn_major, uint32_t M,
                                                  uint32_t N) {
    return (1u << 4)                      // D = F32
           | (a_fmt << 7) | (b_fmt << 10)  // operand formats
           | (0u << 15)                   // A K-major
           | ((b_mn_major ? 1u : 0u) << 16) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

DSA_DEV void mma_bf16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accum) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
}
DSA_DEV void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t accum) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
}
DSA_DEV void mma_fp8_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accum) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p; }" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
}
// Arrive on the mbarrier at this shared-memory offset in every CTA of
// `cta_mask` once every MMA issued so far by this thread has completed.
DSA_DEV void mma_commit_mc(uint32_t bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
        "h"(cta_mask)
        : "memory");
}
// Arrive on a CTA-local mbarrier once every MMA issued so far by this thread
// has completed.
DSA_DEV void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

DSA_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
DSA_DEV void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 consecutive 32-bit columns of this thread's lane.
DSA_DEV void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,"
        "%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
DSA_DEV void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
        "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
        "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

DSA_DEV void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
DSA_DEV void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

DSA_DEV uint32_t lane_id() { return threadIdx.x & 31; }
DSA_DEV uint32_t warp_id() { return threadIdx.x >> 5; }

DSA_DEV float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

DSA_DEV uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

}  // namespace dsa
