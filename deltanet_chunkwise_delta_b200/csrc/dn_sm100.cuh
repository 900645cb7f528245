// sm_100a primitives: mbarriers, TMA tile loads, tcgen05 MMA / TMEM, and
// shared-memory matrix descriptors, written as inline PTX.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

namespace dn {
namespace sm100 {

__device__ __forceinline__ uint32_t saddr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---- mbarrier -------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(saddr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// As above, but the thread may sleep until the phase completes (at most
// about `hint_ns`), which keeps waiting warps off the issue slots.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity,
                                                    uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(saddr(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// A CTA's abort state for its bounded waits: the flag that a wait which gave up
// raises (every other wait of the CTA then gives up at once), followed by the
// time after which a wait gives up.  Kernels keep one in shared memory and pass
// &ctl->abort to the waits below.
struct WaitCtl {
    int abort;
    int pad;
    unsigned long long limit_ns;
};
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;  // 2 s
__device__ __forceinline__ void wait_ctl_init(WaitCtl* c, unsigned long long limit_ns) {
    c->abort = 0;
    c->limit_ns = limit_ns ? limit_ns : kDefaultWaitNs;
}

// Waits for the phase with the given parity.  Gives up after `limit_ns` (0: the
// limit of the WaitCtl whose flag `abort` is), or as soon as another thread has
// raised *abort, and returns false; the caller then skips the rest of its work
// so that the CTA can drain and exit.  Drain waits pass a local flag and an
// explicit limit.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint64_t limit_ns = 0) {
    if (limit_ns == 0) limit_ns = reinterpret_cast<volatile WaitCtl*>(abort)->limit_ns;
    // spin first (the common short waits on the state chain), then sleep-wait
#pragma unroll 1
    for (int i = 0; i < 256; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
        if (*abort) return false;
        if (globaltimer() - t0 > limit_ns) {
            *abort = 1;
            return false;
        }
    }
}

// Drain wait: at most 200 ms and independent of the abort flag, for copies or
// products already issued, before the CTA exits or frees what they use.
constexpr unsigned long long kDrainWaitNs = 200000000ull;
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
    volatile int local = 0;
    mbar_wait(bar, parity, &local, kDrainWaitNs);
}

// Waits for two phases.  Both barriers are tested back to back first, so the
// common case (both complete) costs one barrier round trip instead of two.
__device__ __forceinline__ bool mbar_wait2(uint64_t* a, uint32_t pa, uint64_t* b, uint32_t pb,
                                           volatile int* abort) {
    const bool ra = mbar_try_wait(a, pa);
    const bool rb = mbar_try_wait(b, pb);
    if (ra && rb) return true;
    return (ra || mbar_wait(a, pa, abort)) && (rb || mbar_wait(b, pb, abort));
}

// ---- TMA ------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(saddr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(saddr(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(saddr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(saddr(bar)), "r"(c0), "r"(c1)
        : "memory");
}
// Tiled TMA store shared -> global of one box (bulk-group completion).  Rows
// outside the tensor are not written.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* src, int c0, int c1, int c2,
                                             int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(saddr(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
// Plain bulk copy shared -> global (16-byte aligned, size a multiple of 16), in the
// current bulk group.
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(saddr(src)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until the shared-memory sources of every committed bulk group have been read.
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Waits until every committed bulk group has completed (its writes are performed).
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Plain bulk copy global -> shared (16-byte aligned, size a multiple of 16),
// completing on `bar` with its byte count.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            saddr(dst)),
        "l"(src), "r"(bytes), "r"(saddr(bar))
        : "memory");
}
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- tcgen05 ----------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     saddr(dst)),
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
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem], kind::f16 (bf16 in, fp32 accumulate).
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem], kind::f16.  A (M = 128 lanes) in tensor memory:
// lane m holds row m, column c the pair (A[m][2c] low half, A[m][2c+1] high half),
// so the k-step j of an MMA starts 8 columns after step j - 1.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrives (once) on `bar` when every MMA issued so far by this thread is complete.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            saddr(bar))
        : "memory");
}
// Waits until every tensor-core product this thread has issued is complete: a
// commit to `bar` (a barrier of count 1 used for nothing else, phase 0) and a
// drain wait on it.  Issuers call it once before the CTA frees its tensor
// memory, so that no product in flight writes freed columns or reads shared
// memory after the CTA has left, also when a bounded wait gave up.
__device__ __forceinline__ void umma_drain(uint64_t* bar) {
    umma_commit(bar);
    mbar_drain(bar, 0);
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn,
                                                  bool a_neg = false) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_neg ? 1u : 0u) << 13) |
           ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor, 128-byte swizzle (tile bases 1024-aligned).
//   K-major:  sbo = byte stride between 8-row groups, lbo unused (16).
//   MN-major: lbo = byte stride between 64-element atoms along M/N,
//             sbo = byte stride between 8-row groups along K.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

#define DN_R8(b) "=r"(r[b + 0]), "=r"(r[b + 1]), "=r"(r[b + 2]), "=r"(r[b + 3]), "=r"(r[b + 4]), \
                 "=r"(r[b + 5]), "=r"(r[b + 6]), "=r"(r[b + 7])
#define DN_I8(b) "r"(r[b + 0]), "r"(r[b + 1]), "r"(r[b + 2]), "r"(r[b + 3]), "r"(r[b + 4]), \
                 "r"(r[b + 5]), "r"(r[b + 6]), "r"(r[b + 7])

// 32 consecutive 32-bit TMEM columns of this thread's lane; waits for completion.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
        "tcgen05.wait::ld.sync.aligned;\n"
        : DN_R8(0), DN_R8(8), DN_R8(16), DN_R8(24)
        : "r"(taddr)
        : "memory");
}

// 64 consecutive columns, one wait.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
        "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n"
        "tcgen05.wait::ld.sync.aligned;\n"
        : DN_R8(0), DN_R8(8), DN_R8(16), DN_R8(24), DN_R8(32), DN_R8(40), DN_R8(48), DN_R8(56)
        : "r"(taddr)
        : "memory");
}

// 16 lanes x 8 columns starting at taddr (lane, column), in the mma fragment
// layout: thread t receives rows t/4 and t/4 + 8, columns 2 (t % 4) and + 1:
//   r[0] (t/4, 2(t%4)), r[1] (t/4, 2(t%4)+1), r[2] (t/4+8, 2(t%4)), r[3] (t/4+8, 2(t%4)+1).
// Does not wait: follow with tmem_wait_ld() before using the registers.
__device__ __forceinline__ void tmem_ld16x256(uint32_t taddr, uint32_t (&r)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x1.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr)
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Four 8 x 8 bf16 matrices, each given in the mma fragment layout (thread t holds
// row t/4, columns 2 (t%4), +1 of every matrix), stored transposed: row j of
// matrix i goes to the 16 bytes at the address supplied by thread 8 i + j.
__device__ __forceinline__ void stmatrix_x4_trans(uint32_t saddr_row, uint32_t r0, uint32_t r1, uint32_t r2,
                                                  uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(saddr_row),
                 "r"(r0), "r"(r1), "r"(r2), "r"(r3)
                 : "memory");
}

// Zeroes 32 consecutive 32-bit TMEM columns of this thread's lane; waits for completion.
__device__ __forceinline__ void tmem_zero32(uint32_t taddr) {
    asm volatile(
        "{\n .reg .b32 z;\n mov.b32 z, 0;\n"
        " tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{z,z,z,z,z,z,z,z,z,z,z,z,z,z,z,z,z,z,z,z,z,z,z,z,z,z,z,z,z,z,z,z};\n"
        " tcgen05.wait::st.sync.aligned;\n}\n" ::"r"(taddr)
        : "memory");
}
// Waits for four phases, testing all four back to back first.
__device__ __forceinline__ bool mbar_wait4(uint64_t* a, uint32_t pa, uint64_t* b, uint32_t pb, uint64_t* c,
                                           uint32_t pc, uint64_t* d, uint32_t pd, volatile int* abort) {
    const bool ra = mbar_try_wait(a, pa);
    const bool rb = mbar_try_wait(b, pb);
    const bool rc = mbar_try_wait(c, pc);
    const bool rd = mbar_try_wait(d, pd);
    if (ra && rb && rc && rd) return true;
    return (ra || mbar_wait(a, pa, abort)) && (rb || mbar_wait(b, pb, abort)) && (rc || mbar_wait(c, pc, abort)) &&
           (rd || mbar_wait(d, pd, abort));
}
// Waits for three phases, testing all three back to back first.
__device__ __forceinline__ bool mbar_wait3(uint64_t* a, uint32_t pa, uint64_t* b, uint32_t pb, uint64_t* c,
                                           uint32_t pc, volatile int* abort) {
    const bool ra = mbar_try_wait(a, pa);
    const bool rb = mbar_try_wait(b, pb);
    const bool rc = mbar_try_wait(c, pc);
    if (ra && rb && rc) return true;
    return (ra || mbar_wait(a, pa, abort)) && (rb || mbar_wait(b, pb, abort)) && (rc || mbar_wait(c, pc, abort));
}

// 16 consecutive 32-bit TMEM columns of this thread's lane; waits for completion.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n"
        "tcgen05.wait::st.sync.aligned;\n" ::"r"(taddr),
        DN_I8(0), DN_I8(8)
        : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n"
        "tcgen05.wait::st.sync.aligned;\n" ::"r"(taddr),
        DN_I8(0), DN_I8(8), DN_I8(16), DN_I8(24)
        : "memory");
}
#undef DN_R8
#undef DN_I8

// ---- named barriers ------------------------------------------------------------------
__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---- legacy tf32 MMA for the small triangular-solve blocks --------------------------
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void mma_tf32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 128-byte-swizzled byte offset of bf16 element (r, c), c < 64, in a tile whose
// rows are 128 bytes (the TMA / UMMA SWIZZLE_128B pattern).
__device__ __forceinline__ uint32_t swz128(int r, int c) {
    return (uint32_t)(r * 128 + ((((c >> 3) ^ (r & 7))) << 4) + ((c & 7) << 1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace sm100
}  // namespace dn
