// Kept-token (mixed-precision) variants of the chunk quantiser: groups of 128
// columns or more, warp teams.
#include "hadq_kernels.h"
#include "hadq_chunk.cuh"

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

}  // namespace hadq
