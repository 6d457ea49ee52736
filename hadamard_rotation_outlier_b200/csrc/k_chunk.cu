// Kernel pointers of one kernel family, instantiated in this translation unit
// (the families compile in parallel; the C ABI in hadq_api.cu only calls these).
#include "hadq_kernels.h"
#include "hadq_chunk.cuh"

namespace hadq {
namespace {

template <int BITS, bool SIGNS, bool WIDE_G, int TEAM>
const void* chunk_fn(int B) {
  switch (B) {
    case 8: return (const void*)rq_chunk_kernel<3, BITS, SIGNS, WIDE_G, TEAM>;
    case 16: return (const void*)rq_chunk_kernel<4, BITS, SIGNS, WIDE_G, TEAM>;
    case 32: return (const void*)rq_chunk_kernel<5, BITS, SIGNS, WIDE_G, TEAM>;
    case 64: return (const void*)rq_chunk_kernel<6, BITS, SIGNS, WIDE_G, TEAM>;
    default: return (const void*)rq_chunk_kernel<7, BITS, SIGNS, WIDE_G, TEAM>;
  }
}

// Small groups always use warp teams; chunk-wide groups use either.
template <int BITS, bool SIGNS>
const void* chunk_fn_g(int B, bool wide_g, int team) {
  if (!wide_g) return chunk_fn<BITS, SIGNS, false, 32>(B);
  return team == 32 ? chunk_fn<BITS, SIGNS, true, 32>(B) : chunk_fn<BITS, SIGNS, true, kCT>(B);
}

}  // namespace

const void* wide4096_kernel_ptr(int bits, bool signs) {
  if (bits == 8) return signs ? (const void*)rq_wide4096_kernel<8, true> : (const void*)rq_wide4096_kernel<8, false>;
  return signs ? (const void*)rq_wide4096_kernel<4, true> : (const void*)rq_wide4096_kernel<4, false>;
}

const void* chunk_kernel_ptr(int bits, int B, bool signs, bool wide_g, int team) {
  return bits == 8 ? (signs ? chunk_fn_g<8, true>(B, wide_g, team) : chunk_fn_g<8, false>(B, wide_g, team))
                   : (signs ? chunk_fn_g<4, true>(B, wide_g, team) : chunk_fn_g<4, false>(B, wide_g, team));
}

}  // namespace hadq
