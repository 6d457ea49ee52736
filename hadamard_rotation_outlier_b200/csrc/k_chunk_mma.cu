// 128-point Hadamard blocks (with or without signs) with the first 16-point
// stage on tensor cores.
#include "hadq_chunk_mma.cuh"
#include "hadq_kernels.h"

namespace hadq {

template <int BITS>
static const void* pick(bool signs, bool rot) {
  if (signs) return rot ? (const void*)rq_chunk_mma_kernel<BITS, true, true> : (const void*)rq_chunk_mma_kernel<BITS, true, false>;
  return rot ? (const void*)rq_chunk_mma_kernel<BITS, false, true> : (const void*)rq_chunk_mma_kernel<BITS, false, false>;
}

const void* chunk_mma_kernel_ptr(int bits, bool signs, bool rot) { return bits == 8 ? pick<8>(signs, rot) : pick<4>(signs, rot); }

}  // namespace hadq
