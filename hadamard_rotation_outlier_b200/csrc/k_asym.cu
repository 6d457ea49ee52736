// Asymmetric (zero-point) rotate+quantise and its inverse.
#include "hadq_asym.cuh"
#include "hadq_kernels.h"

namespace hadq {
namespace {

template <int BITS, bool SIGNS>
const void* asym_fn(int B) {
  switch (B) {
    case 8: return (const void*)rq_chunk_asym_kernel<3, BITS, SIGNS>;
    case 16: return (const void*)rq_chunk_asym_kernel<4, BITS, SIGNS>;
    case 32: return (const void*)rq_chunk_asym_kernel<5, BITS, SIGNS>;
    case 64: return (const void*)rq_chunk_asym_kernel<6, BITS, SIGNS>;
    default: return (const void*)rq_chunk_asym_kernel<7, BITS, SIGNS>;
  }
}

template <int LOG_B, int BITS, bool SIGNS>
const void* asym_dq_f(bool f32) {
  return f32 ? (const void*)dq_chunk_asym_kernel<LOG_B, BITS, SIGNS, true>
             : (const void*)dq_chunk_asym_kernel<LOG_B, BITS, SIGNS, false>;
}

template <int BITS, bool SIGNS>
const void* asym_dq_fn(int B, bool f32) {
  switch (B) {
    case 8: return asym_dq_f<3, BITS, SIGNS>(f32);
    case 16: return asym_dq_f<4, BITS, SIGNS>(f32);
    case 32: return asym_dq_f<5, BITS, SIGNS>(f32);
    case 64: return asym_dq_f<6, BITS, SIGNS>(f32);
    default: return asym_dq_f<7, BITS, SIGNS>(f32);
  }
}

}  // namespace

const void* asym_chunk_kernel_ptr(int bits, int B, bool signs) {
  if (bits == 8) return signs ? asym_fn<8, true>(B) : asym_fn<8, false>(B);
  return signs ? asym_fn<4, true>(B) : asym_fn<4, false>(B);
}

const void* asym_dq_chunk_kernel_ptr(int bits, int B, bool signs, bool f32) {
  if (bits == 8) return signs ? asym_dq_fn<8, true>(B, f32) : asym_dq_fn<8, false>(B, f32);
  return signs ? asym_dq_fn<4, true>(B, f32) : asym_dq_fn<4, false>(B, f32);
}

}  // namespace hadq
