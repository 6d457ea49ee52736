// Kept-token (mixed-precision) variants of the chunk quantiser (groups of 128
// columns or more, warp teams) and of the 128-point tensor-core quantiser.
#include "hadq_kernels.h"
#include "hadq_chunk.cuh"
#include "hadq_chunk_mma.cuh"

namespace hadq {
namespace {

template <int BITS, bool SIGNS>
const void* keep_fn(int B) {
  switch (B) {
    case 8: return (const void*)rq_chunk_kernel<3, BITS, SIGNS, true, 32, true>;
    case 16: return (const void*)rq_chunk_kernel<4, BITS, SIGNS, true, 32, true>;
    case 32: return (const void*)rq_chunk_kernel<5, BITS, SIGNS, true, 32, true>;
    case 64: return (const void*)rq_chunk_kernel<6, BITS, SIGNS, true, 32, true>;
    default: return (const void*)rq_chunk_kernel<7, BITS, SIGNS, true, 32, true>;
  }
}

}  // namespace

const void* keep_chunk_kernel_ptr(int bits, int B, bool signs) {
  if (bits == 8) return signs ? keep_fn<8, true>(B) : keep_fn<8, false>(B);
  return signs ? keep_fn<4, true>(B) : keep_fn<4, false>(B);
}

const void* keep_chunk_mma_kernel_ptr(int bits, bool signs) {
  if (bits == 8)
    return signs ? (const void*)rq_chunk_mma_kernel<8, true, false, true> : (const void*)rq_chunk_mma_kernel<8, false, false, true>;
  return signs ? (const void*)rq_chunk_mma_kernel<4, true, false, true> : (const void*)rq_chunk_mma_kernel<4, false, false, true>;
}

}  // namespace hadq
