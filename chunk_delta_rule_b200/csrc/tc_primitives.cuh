// sm_100a primitives used by the tensor-core chunk kernel: shared-memory
// matrix descriptors, tcgen05 MMA / TMEM access, mbarriers with bounded waits,
// and TMA tile copies.  Inline PTX written from the public PTX ISA.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace comba {
namespace tc {

// ---------------------------------------------------------------- addresses
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2, version 1).
//   K-major operand  : rows (M or N) at 128 B pitch, 8-row groups every `sbo`
//                      bytes; 64 bf16 of K per 128 B row; `lbo` unused (16).
//   MN-major operand : 64 bf16 of M/N contiguous per 128 B row, one row per K
//                      index, 8-row K groups every `sbo` bytes, 64-element M/N
//                      atoms every `lbo` bytes.
// The tile base must be 1024-byte aligned; a start address may move by a
// multiple of 32 B inside the 128 B row to select a 16-element K slice.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;   // descriptor version for sm_100
    d |= (uint64_t)2 << 61;   // SWIZZLE_128B
    return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4)                         // D format: f32
         | (1u << 7)                         // A format: bf16
         | (1u << 10)                        // B format: bf16
         | ((a_mn ? 1u : 0u) << 15)          // A major: 0 = K, 1 = MN
         | ((b_mn ? 1u : 0u) << 16)          // B major
         | ((uint32_t)(N >> 3) << 17)
         | ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor for kind::tf32 (fp32 storage, tf32 products, fp32
// accumulation).  An A operand taken from TMEM is always K-major.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4)                         // D format: f32
         | (2u << 7)                         // A format: tf32
         | (2u << 10)                        // B format: tf32
         | ((a_mn ? 1u : 0u) << 15)
         | ((b_mn ? 1u : 0u) << 16)
         | ((uint32_t)(N >> 3) << 17)
         | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------- mbarriers
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n"
        ".reg .pred p;\n"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        "selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Non-blocking test of a phase.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n"
        ".reg .pred p;\n"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        "selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// try_wait with a suspend-time hint: the thread sleeps (issuing nothing) until
// the phase completes or about `hint_ns` pass.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n"
        ".reg .pred p;\n"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        "selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns) : "memory");
    return ok != 0;
}

// Bounded wait: false if the phase has not completed after `timeout_ns`.
// Waiting threads sleep in the barrier instead of spinning, so they leave
// issue slots to the other warps of the SM.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 200000u)) return true;
        if (globaltimer_ns() - t0 > timeout_ns) return false;
    }
}

// ---------------------------------------------------------------- fences
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---------------------------------------------------------------- TMEM
// Whole warp: allocates `ncols` TMEM columns, writes the base address to *dst.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(dst)), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                 ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T (called by a whole warp; one elected lane issues)
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n"
        ".reg .pred p, e;\n"
        "elect.sync _|e, 0xffffffff;\n"
        "setp.ne.b32 p, %4, 0;\n"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n"
        "}\n"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, bf16 (A: lane = row, two bf16 per column,
// the lower K index in the low half)
__device__ __forceinline__ void mma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n"
        ".reg .pred p, e;\n"
        "elect.sync _|e, 0xffffffff;\n"
        "setp.ne.b32 p, %4, 0;\n"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n"
        "}\n"
        ::"r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, tf32 (A: lane = row, one fp32 per column)
__device__ __forceinline__ void mma_tf32_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n"
        ".reg .pred p, e;\n"
        "elect.sync _|e, 0xffffffff;\n"
        "setp.ne.b32 p, %4, 0;\n"
        "@e tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n"
        "}\n"
        ::"r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

// Arrives on `bar` once all previously issued MMAs of the issuing lane complete.
// Like the MMA helpers above, it is called by all 32 lanes of one converged warp
// and issued by the lane elect.sync picks (the same lane every time for a full
// mask), so the operands stay warp-uniform and no per-lane serialisation is needed.
// Callers reconverge the warp (__syncwarp) before an issue block that follows
// divergent code: without it the compiler may leave the warp split across the
// block, which was measured to slow the whole kernel by half.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile(
        "{\n"
        ".reg .pred e;\n"
        "elect.sync _|e, 0xffffffff;\n"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n"
        "}\n"
        ::"r"(smem_u32(bar)) : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp receives lane
// (warp%4)*32 + t, columns [col, col + 32).
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

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 16 consecutive 32-bit columns (the 16-column form of tmem_st32).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])),
          "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])),
          "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
          "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
          "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
          "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
        : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])),
          "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])),
          "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
          "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
          "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
          "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
          "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
          "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
          "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
          "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
          "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y, int z, int w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z),
          "r"(w), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* src, int x, int y,
                                             int z, int w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];"
        ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z), "r"(w)
        : "memory");
}

// Untiled bulk copy of `bytes` from global memory into this CTA's shared memory,
// completing that many bytes of transaction count on `bar` (no multicast).  Both
// addresses 16-byte aligned, `bytes` a multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Waits until all committed bulk stores of this thread have finished reading smem.
__device__ __forceinline__ void bulk_wait_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Waits until all committed bulk stores of this thread are complete.
__device__ __forceinline__ void bulk_wait0() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- MMA issue
// Every helper issues `ksteps` MMAs (K = 16 for bf16, K = 8 for tf32) from one
// converged warp; the first accumulates into D only if `acc0` is set, the rest
// always do.  Shapes are taken from `idesc`.  Byte arguments are shared-memory
// addresses.  Each descriptor is built once: the start address sits in its low
// 14 bits (address / 16, below 2^14 for any shared-memory address), so a
// k-step's operand offset is added to the descriptor directly.  The loops are
// unrolled by COMBA_MMA_UNROLL (default: rolled).  Issue runs at the tensor pipe's
// pace either way once a warp is dedicated to it, and the rolled loops keep that
// warp's code small (instruction fetch stalls were the largest stall reason with
// every loop unrolled).
#ifndef COMBA_MMA_UNROLL
#define COMBA_MMA_UNROLL 1
#endif
constexpr int kMmaUnroll = COMBA_MMA_UNROLL;

__device__ __forceinline__ uint32_t katom_off(int ks, uint32_t atom) {   // K-major k-step offset
    return (uint32_t)(ks >> 2) * atom + (uint32_t)(ks & 3) * 32u;
}

// A K-major (128 rows, 64-element K atoms `a_atom` bytes apart),
// B K-major (N rows, K atoms `b_atom` bytes apart; 0 re-reads atom 0).
__device__ __forceinline__ void mma_ak_bk(uint32_t d, uint32_t a, uint32_t a_atom, uint32_t b,
                                          uint32_t b_atom, uint32_t idesc, int ksteps,
                                          uint32_t acc0) {
    const uint64_t ad0 = sdesc_sw128(a, 16, 1024), bd0 = sdesc_sw128(b, 16, 1024);
#pragma unroll kMmaUnroll
    for (int ks = 0; ks < ksteps; ++ks)
        mma_bf16(d, ad0 + (katom_off(ks, a_atom) >> 4), bd0 + (katom_off(ks, b_atom) >> 4), idesc,
                 (ks > 0) ? 1u : acc0);
}

// A MN-major (M in 64-element atoms `a_lbo` bytes apart; one 128 B row per K
// index), B K-major (N rows, K within one 64-element atom).
__device__ __forceinline__ void mma_amn_bk(uint32_t d, uint32_t a, uint32_t a_lbo, uint32_t b,
                                           uint32_t idesc, int ksteps, uint32_t acc0) {
    const uint64_t ad0 = sdesc_sw128(a, a_lbo, 1024), bd0 = sdesc_sw128(b, 16, 1024);
#pragma unroll kMmaUnroll
    for (int ks = 0; ks < ksteps; ++ks)
        mma_bf16(d, ad0 + (uint32_t)(ks * (2048 >> 4)), bd0 + (uint32_t)(ks * (32 >> 4)), idesc,
                 (ks > 0) ? 1u : acc0);
}

// A K-major (128 rows, K atoms `a_atom` apart), B MN-major (N in atoms
// `b_lbo` apart; one 128 B row per K index; the K row index wraps every
// `kwrap` steps so a K extent can be re-read, e.g. for a hi/lo split of A).
__device__ __forceinline__ void mma_ak_bmn(uint32_t d, uint32_t a, uint32_t a_atom, uint32_t b,
                                           uint32_t b_lbo, uint32_t idesc, int ksteps, int kwrap,
                                           uint32_t acc0) {
    const uint64_t ad0 = sdesc_sw128(a, 16, 1024), bd0 = sdesc_sw128(b, b_lbo, 1024);
#pragma unroll kMmaUnroll
    for (int ks = 0; ks < ksteps; ++ks)
        mma_bf16(d, ad0 + (katom_off(ks, a_atom) >> 4), bd0 + (uint32_t)((ks % kwrap) * (2048 >> 4)),
                 idesc, (ks > 0) ? 1u : acc0);
}

// tf32, A from TMEM (K = 8 columns per MMA), B K-major fp32 (N rows; 32-element
// K atoms `b_atom` bytes apart).
__device__ __forceinline__ void mma_tf32_ta_bk(uint32_t d, uint32_t a_tmem, uint32_t b,
                                               uint32_t b_atom, uint32_t idesc, int ksteps,
                                               uint32_t acc0) {
    const uint64_t bd0 = sdesc_sw128(b, 16, 1024);
#pragma unroll kMmaUnroll
    for (int ks = 0; ks < ksteps; ++ks)
        mma_tf32_ta(d, a_tmem + ks * 8, bd0 + (katom_off(ks, b_atom) >> 4), idesc, (ks > 0) ? 1u : acc0);
}

// bf16, A from TMEM (K = 16 per MMA = 8 packed columns), B K-major (N rows, K
// atoms `b_atom` apart).
__device__ __forceinline__ void mma_bf16_ta_bk(uint32_t d, uint32_t a_tmem, uint32_t b,
                                               uint32_t b_atom, uint32_t idesc, int ksteps,
                                               uint32_t acc0) {
    const uint64_t bd0 = sdesc_sw128(b, 16, 1024);
#pragma unroll kMmaUnroll
    for (int ks = 0; ks < ksteps; ++ks)
        mma_bf16_ta(d, a_tmem + ks * 8, bd0 + (katom_off(ks, b_atom) >> 4), idesc, (ks > 0) ? 1u : acc0);
}

// bf16, A from TMEM, B MN-major (N in atoms `b_lbo` apart; one 128 B row per K index).
__device__ __forceinline__ void mma_bf16_ta_bmn(uint32_t d, uint32_t a_tmem, uint32_t b,
                                                uint32_t b_lbo, uint32_t idesc, int ksteps,
                                                uint32_t acc0) {
    const uint64_t bd0 = sdesc_sw128(b, b_lbo, 1024);
#pragma unroll kMmaUnroll
    for (int ks = 0; ks < ksteps; ++ks)
        mma_bf16_ta(d, a_tmem + ks * 8, bd0 + (uint32_t)(ks * (2048 >> 4)), idesc, (ks > 0) ? 1u : acc0);
}

// bf16, A and B both MN-major from shared memory (M and N in 64-element atoms
// `a_lbo` / `b_lbo` bytes apart; one 128 B row per K index in each).
__device__ __forceinline__ void mma_amn_bmn(uint32_t d, uint32_t a, uint32_t a_lbo, uint32_t b,
                                            uint32_t b_lbo, uint32_t idesc, int ksteps, uint32_t acc0) {
    const uint64_t ad0 = sdesc_sw128(a, a_lbo, 1024), bd0 = sdesc_sw128(b, b_lbo, 1024);
#pragma unroll kMmaUnroll
    for (int ks = 0; ks < ksteps; ++ks)
        mma_bf16(d, ad0 + (uint32_t)(ks * (2048 >> 4)), bd0 + (uint32_t)(ks * (2048 >> 4)), idesc,
                 (ks > 0) ? 1u : acc0);
}

// ---------------------------------------------------------------- warp MMA (legacy)
// fp32 -> tf32 (10 stored mantissa bits, the low 13 bits cleared), rounded to
// nearest with ties away from zero: adding half a tf32 unit to the magnitude and
// truncating does exactly that on a sign-magnitude bit pattern (the largest
// finite values round up to infinity).  The same result as cvt.rna.tf32.f32 for
// every non-NaN input (a NaN whose payload lies only in the low 13 bits becomes
// infinity), in two integer operations instead of a conversion with about 15
// cycles of latency on this part.
__device__ __forceinline__ uint32_t f32_to_tf32(float x) {
    return (__float_as_uint(x) + 0x1000u) & 0xffffe000u;
}

// d[16x8] += a[16x8] * b[8x8], tf32 inputs, fp32 accumulation, one warp.  Not
// volatile: a pure register operation the compiler may schedule among the loads
// that feed it.
__device__ __forceinline__ void mma_sync_tf32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void named_barrier(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Producer side of a named barrier: counts this warp's threads without waiting.
__device__ __forceinline__ void named_barrier_arrive(int id, int nthreads) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier that also ORs a per-thread failure flag across the
// participating threads: returns true only if no thread reported failure, so
// every thread of the group takes the same decision.
__device__ __forceinline__ bool named_barrier_all_ok(int id, int nthreads, bool ok) {
    uint32_t any_fail;
    asm volatile(
        "{\n"
        ".reg .pred pf, pa;\n"
        "setp.eq.u32 pf, %1, 0;\n"
        "bar.red.or.pred pa, %2, %3, pf;\n"
        "selp.u32 %0, 1, 0, pa;\n"
        "}\n"
        : "=r"(any_fail) : "r"((uint32_t)ok), "r"(id), "r"(nthreads) : "memory");
    return any_fail == 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// ---------------------------------------------------------------- shared memory
// Explicit shared-space accesses by 32-bit shared address.  Loads are issued
// unconditionally (callers select the value), which keeps element loops free
// of divergent branches.
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ float lds_f32(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ float4 lds_f32x4(uint32_t a) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ uint4 lds_u32x4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ void sts_f32(uint32_t a, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
__device__ __forceinline__ void sts_f32x4(uint32_t a, float4 v) {
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};"
                 ::"r"(a), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w) : "memory");
}
__device__ __forceinline__ void sts_u32x4(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                 ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
__device__ __forceinline__ void sts_u32(uint32_t a, uint32_t v) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void sts_u16(uint32_t a, unsigned short v) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(a), "h"(v) : "memory");
}

// ---------------------------------------------------------------- swizzle
// Byte offset of the 16-byte chunk `c` (0..7) of row `r` in a 128B-swizzled
// tile whose rows are 128 bytes apart.
__device__ __forceinline__ uint32_t sw128(uint32_t r, uint32_t c) {
    return r * 128u + ((c ^ (r & 7u)) << 4);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&t);
}

}  // namespace tc
}  // namespace comba
