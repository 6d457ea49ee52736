// Kernel pointers of one kernel family, instantiated in this translation unit
// (the families compile in parallel; the C ABI in hadq_api.cu only calls these).
#include "hadq_kernels.h"
#include "hadq_chunk.cuh"

namespace hadq {
namespace {

template <int BITS, bool SIGNS, bool WIDE_G>
const void* chunk_fn(int B) {
  switch (B) {
    case 8: return (const void*)rq_chunk_kernel<3, BITS, SIGNS, WIDE_G>;
    case 16: return (const void*)rq_chunk_kernel<4, BITS, SIGNS, WIDE_G>;
    case 32: return (const void*)rq_chunk_kernel<5, BITS, SIGNS, WIDE_G>;
    case 64: return (const void*)rq_chunk_kernel<6, BITS, SIGNS, WIDE_G>;
    default: return (const void*)rq_chunk_kernel<7, BITS, SIGNS, WIDE_G>;
  }
}

template <int BITS, bool SIGNS>
const void* chunk_fn_g(int B, bool wide_g) {
  return wide_g ? chunk_fn<BITS, SIGNS, true>(B) : chunk_fn<BITS, SIGNS, false>(B);
}

}  // namespace

const void* chunk_kernel_ptr(int bits, int B, bool signs, bool wide_g) {
  return bits == 8 ? (signs ? chunk_fn_g<8, true>(B, wide_g) : chunk_fn_g<8, false>(B, wide_g))
                   : (signs ? chunk_fn_g<4, true>(B, wide_g) : chunk_fn_g<4, false>(B, wide_g));
}

}  // namespace hadq
