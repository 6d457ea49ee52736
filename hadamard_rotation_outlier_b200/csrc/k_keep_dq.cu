// Kept-token (mixed-precision) variants of the chunk dequantiser: groups of
// 128 columns or more (so every Hadamard block lies inside one group).
#include "hadq_kernels.h"
#include "hadq_chunk.cuh"

namespace hadq {
namespace {

template <int LOG_B, int BITS, bool SIGNS>
const void* keep_dq_f(bool f32) {
  return f32 ? (const void*)dq_chunk_kernel<LOG_B, BITS, SIGNS, false, true, true>
             : (const void*)dq_chunk_kernel<LOG_B, BITS, SIGNS, false, false, true>;
}

template <int BITS, bool SIGNS>
const void* keep_dq_b(int B, bool f32) {
  switch (B) {
    case 8: return keep_dq_f<3, BITS, SIGNS>(f32);
    case 16: return keep_dq_f<4, BITS, SIGNS>(f32);
    case 32: return keep_dq_f<5, BITS, SIGNS>(f32);
    case 64: return keep_dq_f<6, BITS, SIGNS>(f32);
    default: return keep_dq_f<7, BITS, SIGNS>(f32);
  }
}

}  // namespace

const void* keep_dq_chunk_kernel_ptr(int bits, int B, bool signs, bool f32) {
  if (bits == 8) return signs ? keep_dq_b<8, true>(B, f32) : keep_dq_b<8, false>(B, f32);
  return signs ? keep_dq_b<4, true>(B, f32) : keep_dq_b<4, false>(B, f32);
}

}  // namespace hadq
