// gla_tcgen05.cuh -- helpers for the 5th-generation tensor cores (sm_100a):
// shared-memory matrix descriptors, instruction descriptors, MMA issue and
// commit, tensor-memory loads, and bounded mbarrier waits.  Shared by the
// tcgen05 kernels of the GLA mixer.
#pragma once

#include <stdint.h>

namespace gtr {

// Shared-memory matrix descriptor, 128-byte swizzle, version 1 (sm_100).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;   // descriptor version
    d |= (uint64_t)2 << 61;   // SWIZZLE_128B
    return d;
}

// Instruction descriptor of kind::f16 with fp32 accumulation: A and B both
// fp16 (ab_bf16 = 0) or both bf16 (ab_bf16 = 1), each K-major (0) or
// MN-major (1); M in {64, 128}, N a multiple of 8 up to 256.
__host__ __device__ constexpr uint32_t umma_idesc(int a_mn_major, int b_mn_major, uint32_t M, uint32_t N,
                                                  int ab_bf16 = 0) {
    return (1u << 4)                                              // D format fp32
           | ((uint32_t)ab_bf16 << 7) | ((uint32_t)ab_bf16 << 10)  // A, B format
           | ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16)
           | ((N >> 3) << 17)                                     // N
           | ((M >> 4) << 24);                                    // M
}

// kind::f16, fp16 A and B, fp32 D, M = 64, N = 64.
__host__ __device__ constexpr uint32_t umma_idesc_f16(int a_mn_major, int b_mn_major) {
    return umma_idesc(a_mn_major, b_mn_major, 64u, 64u, 0);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}\n"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u));
}

__device__ __forceinline__ void umma_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(mbar)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void fence_async_shared() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

// 16 TMEM lanes x 64 fp32 columns -> 32 registers in the m16n8 fragment
// layout: r[4n + i] is element i of the 8-column tile n.
__device__ __forceinline__ void tmem_ld_16x64(uint32_t taddr, float (&r)[32]) {
    uint32_t *u = reinterpret_cast<uint32_t *>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15]),
          "=r"(u[16]), "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]),
          "=r"(u[24]), "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]), "=r"(u[31])
        : "r"(taddr));
}

__device__ __forceinline__ void mbar_arrive(uint32_t mbar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(mbar) : "memory");
}
__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(mbar), "r"(count) : "memory");
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
    return t;
}

// Bound of a wait for tensor-core work this CTA issued itself: about one
// second of wall time.  Fixed, so that no caller-tunable limit can make a
// CTA give up on MMAs that are still in flight.
constexpr uint64_t kMmaWaitNs = 1000000000ull;

// Wait for the given phase parity of an mbarrier that tensor-core commits
// complete; returns false only if the fixed bound ran out (an error is
// recorded by the caller; the CTA keeps its program order, so its TMEM
// deallocation still follows its last commit).
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity) {
    uint64_t t0 = 0;
    for (uint32_t i = 0;; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.b32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (done) return true;
        if ((i & 63u) == 0) {
            const uint64_t t = global_ns();
            if (i == 0)
                t0 = t;
            else if (t - t0 > kMmaWaitNs)
                return false;
        }
    }
}

// Byte offset of element (row, col) in a 64 x 64 fp16 tile with 128-byte rows,
// 128-byte swizzle.
__device__ __forceinline__ uint32_t sw128(int row, int col) {
    return (uint32_t)(row * 128 + ((((col >> 3) ^ (row & 7)) & 7) << 4) + ((col & 7) << 1));
}

// 16 TMEM lanes x 32 fp32 columns -> 16 registers (four 8-column tiles).
__device__ __forceinline__ void tmem_ld_16x32(uint32_t taddr, float (&r)[16]) {
    uint32_t *u = reinterpret_cast<uint32_t *>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
        : "r"(taddr));
}

}  // namespace gtr
