// sm_100a building blocks: mbarriers with time-bounded waits, TMA tile loads,
// tcgen05 (5th-generation tensor core) MMA with accumulators in tensor memory.
//
// Every wait here gives up after a cycle budget (kWaitBudgetCycles, about two
// seconds, unless the host set another one), records a code in the library's
// device error word (its address is passed to each kernel; the host reads and
// clears it with rtp_poll_device_error) and lets the kernel wind down, so a
// protocol mistake can never hang the GPU.  Winding down still waits (bounded)
// for the asynchronous copies and tensor-core operations already issued.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace rtp {

constexpr int kDevErrTimeout = 1;  // value written to the device error word
constexpr long long kWaitBudgetCycles = 4000000000LL;  // ~2 s at 1.9 GHz; the default wait budget

RTP_DEVICE uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// ---- mbarrier --------------------------------------------------------------
RTP_DEVICE void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(count));
}
RTP_DEVICE void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory"); }
RTP_DEVICE void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_addr(bar)) : "memory");
}
RTP_DEVICE void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}
#ifndef RTP_MBAR_TEST_WAIT
#define RTP_MBAR_TEST_WAIT 0
#endif
RTP_DEVICE bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
#if RTP_MBAR_TEST_WAIT
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
#else
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
#endif
  return ok != 0;
}
// Wait for the phase with the given parity to complete; false on timeout
// (the error word is set).  `budget` is the number of clock cycles the wait
// may take (kWaitBudgetCycles unless the host set another budget).  Once any
// wait of the kernel timed out, `alive` is false and later waits return at
// once.
RTP_DEVICE bool mbar_wait(uint64_t* bar, uint32_t parity, bool& alive, int* err, long long budget) {
  if (!alive) return false;
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try(bar, parity)) {
    if (clock64() - t0 > budget) {
      atomicExch(err, kDevErrTimeout);
      alive = false;
      return false;
    }
  }
  return true;
}

// Wind-down wait for an asynchronous operation this CTA already issued (a TMA
// load or a tensor-core commit): it ignores `alive`, because such an operation
// completes on its own and must land before the CTA frees its tensor memory or
// exits.  Bounded by kWaitBudgetCycles all the same; a give-up is recorded.
RTP_DEVICE void mbar_drain(uint64_t* bar, uint32_t parity, int* err) {
  if (mbar_try(bar, parity)) return;
  const long long t0 = clock64();
  while (!mbar_try(bar, parity)) {
    if (clock64() - t0 > kWaitBudgetCycles) {
      atomicExch(err, kDevErrTimeout);
      return;
    }
  }
}

// ---- TMA -------------------------------------------------------------------
// 4-D tiled load (dims innermost first), completion counted on `bar`.
RTP_DEVICE void tma_load_4d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];\n" ::"r"(smem_addr(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// ---- tcgen05 ---------------------------------------------------------------
// Shared-memory matrix descriptor of a K-major operand tile laid out with the
// 32-byte swizzle (rows of 32 bytes = 16 bf16, 8-row atoms 256 bytes apart),
// which is what a TMA load with CU_TENSOR_MAP_SWIZZLE_32B writes.
RTP_DEVICE uint64_t umma_desc_k_sw32(const void* tile) {
  const uint64_t addr = smem_addr(tile);
  return ((addr >> 4) & 0x3FFFull)      // start address
         | (1ull << 16)                 // leading byte offset (16 B; unused for this layout)
         | ((256ull >> 4) << 32)        // stride byte offset: 8 rows x 32 B
         | (1ull << 46)                 // descriptor version
         | (6ull << 61);                // layout: 32-byte swizzle
}

// Shared-memory matrix descriptor of a 128-byte-swizzled tile as a TMA load
// with CU_TENSOR_MAP_SWIZZLE_128B writes it: rows of 128 bytes (64 bf16),
// 8-row atoms 1024 bytes apart (stride byte offset).  K-major operands (Q, K):
// one MMA K-slice of 16 elements is 32 bytes of a row, so slice k of a
// 64-column half starts `32 * k` bytes in; the leading byte offset is unused.
// MN-major operands (V as the B operand of P V, keys on K, head dims on N):
// the leading byte offset is the distance between the two 64-column halves
// of the tile, and slice k (16 keys) starts `16 * 128 * k` bytes in.
RTP_DEVICE uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo_bytes) {
  return ((uint64_t)(saddr >> 4) & 0x3FFFull)                // start address
         | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16)    // leading byte offset
         | ((uint64_t)(1024u >> 4) << 32)                     // stride byte offset: 8 rows x 128 B
         | (1ull << 46)                                       // descriptor version
         | (2ull << 61);                                      // layout: 128-byte swizzle
}

// Instruction descriptor: D fp32, A/B bf16, both K-major, shape M x N.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_f32(int M, int N) {
  return (1u << 4)                      // D format fp32
         | (1u << 7)                    // A bf16
         | (1u << 10)                   // B bf16
         | ((uint32_t)(N >> 3) << 17)   // N / 8
         | ((uint32_t)(M >> 4) << 24);  // M / 16
}

RTP_DEVICE void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
// The same MMA with the A operand (M x 16, bf16 pairs packed in 32-bit columns,
// row m in lane m) read from tensor memory at `tmem_a`.
RTP_DEVICE void umma_f16_tmem_a(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
// Arrive on `bar` once all previously issued tcgen05.mma of this thread completed.
RTP_DEVICE void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_addr(bar))
               : "memory");
}
RTP_DEVICE void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
RTP_DEVICE void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

// Warp-wide TMEM allocation of `cols` columns; the base address lands in *slot.
RTP_DEVICE void tmem_alloc(uint32_t* slot, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_addr(slot)),
               "r"(cols));
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
}
RTP_DEVICE void tmem_free(uint32_t base, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(base), "r"(cols));
}

// 32 lanes x 32 consecutive fp32 columns: thread (lane l of the warp's
// quadrant) receives row (quadrant*32 + l), columns col .. col+31.
RTP_DEVICE void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// 32 lanes x 16 consecutive fp32 columns.
RTP_DEVICE void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
RTP_DEVICE void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }

// 32 lanes x 16 consecutive 32-bit columns from registers: thread (lane l of
// the warp's quadrant) writes row (quadrant*32 + l), columns col .. col+15.
RTP_DEVICE void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::
          "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
// 32 lanes x 8 consecutive 32-bit columns from registers.
RTP_DEVICE void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
RTP_DEVICE void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

}  // namespace rtp
