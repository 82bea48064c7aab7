// Fifth-generation tensor-core (tcgen05) primitives shared by the sm_100a kernels of libtq:
// shared-memory operand descriptors, MMA issue and commit, TMEM loads and stores, and the
// bounded mbarrier waits of the warp-specialized pipelines.
//
// Operand layout: K-major, 128-byte swizzle. A 128-row operand of 16-bit elements is stored
// as K-blocks of 64 elements; a K-block is [128 rows][128 B] in 8-row atoms of 1024 B, and
// the 16-byte chunk c of row r sits at chunk position c XOR (r mod 8). One K-step of an MMA
// (16 elements = 32 bytes) advances the descriptor's start address by 32 bytes inside a
// K-block.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

#include "tq_device.cuh"

namespace tqtc {

// instruction descriptor, kind::f16 with fp32 accumulation, K-major A and B, M x N
constexpr uint32_t idesc_f16(int m, int n) {
    return (1u << 4) | (((uint32_t)n >> 3) << 17) | (((uint32_t)m >> 4) << 24);
}
// the same with bf16 A and B
constexpr uint32_t idesc_bf16(int m, int n) { return idesc_f16(m, n) | (1u << 7) | (1u << 10); }

// shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart
TQ_DEVICE uint64_t sdesc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// byte offset of 16-byte chunk c (0..7) of row r inside one swizzled K-block
TQ_DEVICE uint32_t sw128(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// D (+)= A B^T, A and B from shared memory
TQ_DEVICE void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %3, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p;\n}\n" ::"r"(d),
        "l"(a), "l"(b), "r"(acc), "r"(idesc));
}
// D (+)= A B^T, A from TMEM (row = lane, two 16-bit elements per column), B from shared memory
TQ_DEVICE void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %3, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %4, p;\n}\n" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(acc), "r"(idesc));
}
// arrive on an mbarrier once every MMA this thread issued before has completed
TQ_DEVICE void commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     tq_smem_addr(bar))
                 : "memory");
}
TQ_DEVICE void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
TQ_DEVICE void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

TQ_DEVICE void tmem_alloc(uint32_t* dst_smem, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tq_smem_addr(dst_smem)),
                 "r"(cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}
TQ_DEVICE void tmem_dealloc(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols));
}

// 16 columns of this thread's TMEM lane, without waiting (twait before use)
TQ_DEVICE void tld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
// wait for this thread's TMEM loads; the registers of the last one are operands, so no use of
// them can be scheduled before the wait
TQ_DEVICE void twait(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15])
                 :
                 : "memory");
}
TQ_DEVICE void tst8(uint32_t taddr, const uint32_t (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"r"(taddr), "r"(v[0]),
                 "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}
TQ_DEVICE void tst16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(
            taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
TQ_DEVICE void twait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

TQ_DEVICE bool mbar_try(uint32_t a, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    return done != 0;
}
// Bounded wait that also gives up when another role has aborted; a wait that runs out sets
// the abort flag itself.
TQ_DEVICE bool wait_bar(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag, uint32_t limit) {
    const uint32_t a = tq_smem_addr(bar);
    for (uint32_t it = 0; it < limit; ++it) {
        if (mbar_try(a, parity)) return true;
        if ((it & 31u) == 31u && *abort_flag) return false;
    }
    *abort_flag = 1u;
    return false;
}
TQ_DEVICE void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tq_smem_addr(bar)) : "memory");
}
TQ_DEVICE void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(tq_smem_addr(bar)), "r"(bytes)
                 : "memory");
}
// bulk copy global -> shared (no multicast), completion counted on an mbarrier
TQ_DEVICE void bulk_copy(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(tq_smem_addr(bar))
                 : "memory");
}

TQ_DEVICE uint32_t pack_half2(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}

}  // namespace tqtc
