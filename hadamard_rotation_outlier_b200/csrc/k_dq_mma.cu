// Inverse of 128-point blocks with the first 16-point stage on tensor cores.
#include "hadq_dq_mma.cuh"
#include "hadq_kernels.h"

namespace hadq {

template <int BITS>
static const void* pick_dq(bool signs, bool f32) {
  if (signs) return f32 ? (const void*)dq_chunk_mma_kernel<BITS, true, true> : (const void*)dq_chunk_mma_kernel<BITS, true, false>;
  return f32 ? (const void*)dq_chunk_mma_kernel<BITS, false, true> : (const void*)dq_chunk_mma_kernel<BITS, false, false>;
}

const void* dq_chunk_mma_kernel_ptr(int bits, bool signs, bool f32) {
  return bits == 8 ? pick_dq<8>(signs, f32) : pick_dq<4>(signs, f32);
}

}  // namespace hadq
