// 128-point Hadamard blocks with the first 16-point stage on tensor cores.
#include "hadq_chunk_mma.cuh"
#include "hadq_kernels.h"

namespace hadq {

const void* chunk_mma_kernel_ptr(int bits, bool rot) {
  if (bits == 8) return rot ? (const void*)rq_chunk_mma_kernel<8, true> : (const void*)rq_chunk_mma_kernel<8, false>;
  return rot ? (const void*)rq_chunk_mma_kernel<4, true> : (const void*)rq_chunk_mma_kernel<4, false>;
}

}  // namespace hadq
