// Device helpers of the tcgen05 kernels: mbarriers with bounded waits, TMA
// tile loads, tcgen05 MMA issue and commit, TMEM loads, the shared-memory
// matrix descriptor, and H_128 written as a K-major operand.
#pragma once

#include <cuda.h>

#include <cstdint>

#include "hadq_common.cuh"

namespace hadq {

constexpr unsigned long long kTcWaitNs = 1000000000ull;  // about one second per wait

// ------------------------------------------------------------- PTX wrappers

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(b)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_addr(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait for the phase of `parity` to complete.  False after kTcWaitNs, or as
// soon as another role has given up (abort set; a null abort waits out the
// time limit, for copies and MMAs still in flight).
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, const volatile uint32_t* abort) {
  if (mbar_test(b, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
    if (mbar_test(b, parity)) return true;
    if (abort && *abort) return false;
    if (global_ns() - t0 > kTcWaitNs) return false;
  }
}
// Record a fault (the word hadq_device_status reads) and tell the CTA's
// other roles to leave their loops.
__device__ __forceinline__ void tc_give_up(uint32_t* abort, unsigned* fault) {
  atomicOr(fault, 1u);
  *reinterpret_cast<volatile uint32_t*>(abort) = 1u;
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: start address, leading and stride byte
// offsets (16-byte units), the fixed version field, the swizzle mode
// (2 = 128-byte, 4 = 64-byte).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t swizzle) {
  return uint64_t((addr & 0x3FFFFu) >> 4) | (uint64_t(lbo >> 4) << 16) | (uint64_t(sbo >> 4) << 32) | (1ull << 46) |
         (uint64_t(swizzle) << 61);
}
// Instruction descriptor of kind::f16 with D float32 and A, B bf16: M, N,
// and whether B is MN-major (A is K-major).
__host__ __device__ constexpr uint32_t tc_idesc_bf16(uint32_t m, uint32_t n, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(b_mn_major) << 16) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

// D[tmem] (+)= A B over K = 16 (both operands from shared memory; B as laid
// out by its descriptor and the instruction descriptor's major bit).
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// 32 lanes x 32 columns of 32 bits from TMEM (lane = thread, register j =
// column + j), waited for inside the same statement so that no use of the
// registers can be scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&a)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int j = 0; j < 32; ++j) a[j] = __uint_as_float(r[j]);
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// H_128 (+-1 in bf16) as a 128 x 128 K-major operand with the 128-byte
// swizzle, rows 1024-byte aligned at `dst`: element (m, k) at (k / 64) * 16384
// + (m / 8) * 1024 + (m % 8) * 128 + 16 * ((k % 64) / 8 XOR m % 8) + 2 (k % 8);
// one 16-byte piece (8 k) per iteration of the CTA's threads.  The caller
// fences the writes for the async proxy before the tensor cores read them.
__device__ __forceinline__ void write_h128_kmajor(uint8_t* dst, int nthreads) {
  for (int i = threadIdx.x; i < 128 * 16; i += nthreads) {
    const int m = i >> 4, kc = i & 15;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int k = 8 * kc + 2 * e;
      const uint32_t lo = (__popc(m & k) & 1) ? 0xBF80u : 0x3F80u;
      const uint32_t hi = (__popc(m & (k + 1)) & 1) ? 0xBF80u : 0x3F80u;
      w[e] = lo | (hi << 16);
    }
    const int off = (kc >> 3) * 16384 + (m >> 3) * 1024 + (m & 7) * 128 + (((kc & 7) ^ (m & 7)) << 4);
    *reinterpret_cast<uint4*>(dst + off) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace hadq
