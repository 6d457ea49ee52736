// Kernel pointers of one kernel family, instantiated in this translation unit
// (the families compile in parallel; the C ABI in hadq_api.cu only calls these).
#include "hadq_kernels.h"
#include "hadq_generic.cuh"

namespace hadq {

const void* generic_kernel_ptr(int direction, int bits) {
  if (direction == 0) return bits == 8 ? (const void*)rq_generic_kernel<8> : (const void*)rq_generic_kernel<4>;
  return bits == 8 ? (const void*)dq_generic_kernel<8> : (const void*)dq_generic_kernel<4>;
}

}  // namespace hadq
