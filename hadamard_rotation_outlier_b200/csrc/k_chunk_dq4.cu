// Kernel pointers of one kernel family, instantiated in this translation unit
// (the families compile in parallel; the C ABI in hadq_api.cu only calls these).
#include "hadq_kernels.h"
#include "hadq_chunk.cuh"

namespace hadq {
namespace {

template <int LOG_B, int BITS, bool SIGNS, bool SF>
const void* dq_chunk_f(bool f32) {
  return f32 ? (const void*)dq_chunk_kernel<LOG_B, BITS, SIGNS, SF, true>
             : (const void*)dq_chunk_kernel<LOG_B, BITS, SIGNS, SF, false>;
}

template <int BITS, bool SIGNS, bool SF>
const void* dq_chunk_b(int B, bool f32) {
  switch (B) {
    case 8: return dq_chunk_f<3, BITS, SIGNS, SF>(f32);
    case 16: return dq_chunk_f<4, BITS, SIGNS, SF>(f32);
    case 32: return dq_chunk_f<5, BITS, SIGNS, SF>(f32);
    case 64: return dq_chunk_f<6, BITS, SIGNS, SF>(f32);
    default: return dq_chunk_f<7, BITS, SIGNS, SF>(f32);
  }
}

template <int BITS>
const void* dq_chunk_s(int B, bool signs, bool scale_first, bool f32) {
  if (signs) return scale_first ? dq_chunk_b<BITS, true, true>(B, f32) : dq_chunk_b<BITS, true, false>(B, f32);
  return scale_first ? dq_chunk_b<BITS, false, true>(B, f32) : dq_chunk_b<BITS, false, false>(B, f32);
}

}  // namespace

const void* dq_chunk_kernel_ptr_4(int B, bool signs, bool scale_first, bool f32) {
  return dq_chunk_s<4>(B, signs, scale_first, f32);
}

}  // namespace hadq
