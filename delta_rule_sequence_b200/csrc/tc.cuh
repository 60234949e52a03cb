// tc.cuh -- hand-written sm_100a tensor-core primitives: tcgen05 MMA from shared memory into
// tensor memory (TMEM), TMEM allocation and loads, mbarriers with bounded waits, and the
// canonical swizzled shared-memory layouts the MMA descriptors describe.
//
// Encodings follow the PTX ISA for tcgen05 (shared-memory matrix descriptor: start address,
// leading/stride byte offsets, version 1, swizzle mode in bits 61-63; instruction descriptor for
// kind::f16: D format bits 4-5, A/B formats bits 7-12, A/B major bits 15-16, N>>3 bits 17-22,
// M>>4 bits 24-28).
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace prism {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------------------------------------
// canonical layouts (all tiles start on a 1024-byte boundary)
//
// SW128 tile: rows of 128 bytes (64 bf16), 8-row atoms of 1 KB, the 16-byte chunk index XORed
// with (row % 8).  A matrix wider than 64 elements is stored as consecutive 64-column blocks,
// `block_bytes` apart.  SW64 tile: rows of 64 bytes (32 bf16), chunk index XORed with
// ((row / 2) % 4).

__device__ __forceinline__ uint32_t sw128_off(int row, int col, uint32_t block_bytes) {
    const int blk = col >> 6, c = col & 63;
    return blk * block_bytes + row * 128 + ((((c >> 3) ^ (row & 7)) & 7) << 4) + ((c & 7) << 1);
}

__device__ __forceinline__ uint32_t sw64_off(int row, int col) {
    return row * 64 + ((((col >> 3) ^ (row >> 1)) & 3) << 4) + ((col & 7) << 1);
}

// Shared-memory matrix descriptor.  layout: 2 = 128B swizzle, 4 = 64B swizzle.
__device__ __forceinline__ uint64_t make_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t layout) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version for sm_100
    d |= (uint64_t)(layout & 7u) << 61;
    return d;
}

// K-major SW128 operand (rows = M or N, contiguous K), k-step `ks` of 16 elements.
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t base, int ks, uint32_t block_bytes) {
    const int k = ks * 16;
    return make_desc(base + (k >> 6) * block_bytes + (k & 63) * 2, 16, 1024, 2);
}

// MN-major SW128 operand stored [k][mn] (contiguous MN, 64-element blocks `block_bytes` apart),
// k-step `ks` of 16 rows.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t base, int ks, uint32_t block_bytes) {
    return make_desc(base + ks * 16 * 128, block_bytes, 1024, 2);
}

// MN-major SW64 operand stored [k][mn] with 32 MN elements per row, k-step `ks` of 16 rows.
__device__ __forceinline__ uint64_t desc_mn_sw64(uint32_t base, int ks) {
    return make_desc(base + ks * 16 * 64, 0, 512, 4);
}

// k-step offsets of an operand, in the descriptor's 16-byte address units (added to a base
// descriptor: the start-address field cannot carry because shared addresses stay below 256 KB).
__host__ __device__ constexpr uint32_t koff_k_sw128(int ks, uint32_t block_bytes) {
    return (((uint32_t)(ks * 16) >> 6) * block_bytes + (uint32_t)((ks * 16) & 63) * 2) >> 4;
}
__host__ __device__ constexpr uint32_t koff_mn_sw128(int ks) { return (uint32_t)ks * 128; }
__host__ __device__ constexpr uint32_t koff_mn_sw64(int ks) { return (uint32_t)ks * 64; }

// NKS k-steps of 16 into accumulator d: A and B base descriptors plus per-step offsets.
template <int NKS, class OA, class OB>
__device__ __forceinline__ void mma_steps(uint32_t d, uint32_t idesc, uint64_t a, uint64_t b, OA oa,
                                          OB ob, bool accumulate) {
#pragma unroll
    for (int ks = 0; ks < NKS; ++ks)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
            :
            : "r"(d), "l"(a + oa(ks)), "l"(b + ob(ks)), "r"(idesc),
              "r"((accumulate || ks > 0) ? 1u : 0u));
}

// mma_steps with an output-lane mask: TMEM lanes whose bit is set in `off` (lane i <-> bit i % 32
// of off[i / 32]) keep their contents; the other lanes receive the product as usual.
template <int NKS, class OA, class OB>
__device__ __forceinline__ void mma_steps_lanes(uint32_t d, uint32_t idesc, uint64_t a, uint64_t b, OA oa,
                                                OB ob, bool accumulate, const uint32_t (&off)[4]) {
#pragma unroll
    for (int ks = 0; ks < NKS; ++ks)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
            :
            : "r"(d), "l"(a + oa(ks)), "l"(b + ob(ks)), "r"(idesc),
              "r"((accumulate || ks > 0) ? 1u : 0u), "r"(off[0]), "r"(off[1]), "r"(off[2]),
              "r"(off[3]));
}

// 4-D tiled TMA load of one box into shared memory, completing on `bar` (tx bytes).
__device__ __forceinline__ void tma_load_4d(void *dst, const void *tmap, int x, int y, int z, int w,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4, %5}], [%6];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(w),
          "r"(smem_u32(bar))
        : "memory");
}

// Prefetch of one 4-D tiled box into L2 (no shared memory, no completion signal).
__device__ __forceinline__ void tma_prefetch_4d(const void *tmap, int x, int y, int z, int w) {
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];"
                 ::"l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(w)
                 : "memory");
}

// Prefetch of `bytes` contiguous bytes into L2 (16-byte aligned, a multiple of 16; no completion).
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Plain (untiled) bulk copy global -> shared, completing on `bar` (tx bytes); 16-byte aligned.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// Plain bulk copy shared -> global (16-byte aligned, size a multiple of 16), in a bulk group.
__device__ __forceinline__ void bulk_s2g(void *dst, const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 ::"l"(dst), "r"(smem_u32(src)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until this thread's bulk groups have finished reading shared memory / completed entirely.
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// ... all but this thread's N most recent bulk groups have finished reading shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read_n() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Instruction descriptor: bf16 x bf16 -> fp32, M x N, A/B K-major (0) or MN-major (1).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------------------------------------------
// tcgen05

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        :
        : "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :
                 : "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Make this thread's generic-proxy shared-memory writes visible to the tensor core (async proxy).
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// TMEM allocation: one full warp executes these.  The base address lands in *dst (shared).
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :
                 : "r"(smem_u32(dst)), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives lane (base lane + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// 32 lanes x 8 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 4 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float (&v)[4]) {
    uint32_t r[4];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}
// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// TMEM address of (lane, column).
__device__ __forceinline__ uint32_t taddr(uint32_t base, int lane, int col) {
    return base + ((uint32_t)lane << 16) + (uint32_t)col;
}

// ------------------------------------------------------------------------------------------------
// mbarriers with bounded waits

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ uint32_t mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok;
}

__device__ __forceinline__ uint32_t mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok;
}
// The same wait by non-suspending polls (64 per unit of the limit), for a thread every one of
// whose waits is on the critical path (a suspended try_wait can wake later than the completion).
__device__ __forceinline__ bool mbar_wait_spin(uint64_t *bar, uint32_t parity, uint32_t *status, uint32_t limit) {
    for (uint32_t i = 0; i < 64u * limit; ++i)
        if (mbar_test_wait(bar, parity)) return true;
    record_status(status, PRISM_ERR_TIMEOUT);
    return false;
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Barrier among `nthreads` threads (whole warps) on hardware barrier `id` (0 is __syncthreads).
__device__ __forceinline__ void named_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Barrier among `nthreads` threads that also ORs a predicate across them (uniform result).
__device__ __forceinline__ bool named_sync_or(uint32_t id, uint32_t nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// Wait for phase `parity` of `bar` to complete.  Gives up after `limit` polls (each poll blocks
// for a bounded, implementation-defined time), records PRISM_ERR_TIMEOUT and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t *status,
                                          uint32_t limit = kWaitPolls) {
    for (uint32_t i = 0; i < limit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
    }
    record_status(status, PRISM_ERR_TIMEOUT);
    return false;
}

// bf16 pack of two floats (round to nearest even), low half = a.
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

}  // namespace tc
}  // namespace prism
