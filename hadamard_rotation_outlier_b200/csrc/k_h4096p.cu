// 4096-point Hadamard blocks on warp pairs, first 16-point stage on tensor cores.
#include "hadq_h4096p.cuh"
#include "hadq_kernels.h"

namespace hadq {

template <int BITS, bool SIGNS>
static const void* h4096p_for(bool rot) {
  return rot ? (const void*)rq_h4096_pair_kernel<BITS, SIGNS, true> : (const void*)rq_h4096_pair_kernel<BITS, SIGNS, false>;
}

const void* h4096_pair_kernel_ptr(int bits, bool signs, bool rot) {
  if (bits == 8) return signs ? h4096p_for<8, true>(rot) : h4096p_for<8, false>(rot);
  return signs ? h4096p_for<4, true>(rot) : h4096p_for<4, false>(rot);
}

}  // namespace hadq
