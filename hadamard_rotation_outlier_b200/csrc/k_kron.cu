// Kronecker rotation F (x) H_b fused with the quantiser, and its inverse.
#include "hadq_kernels.h"
#include "hadq_kron.cuh"

namespace hadq {

const void* kron16_kernel_ptr(int bits) {
  return bits == 8 ? (const void*)rq_kron16_kernel<8> : (const void*)rq_kron16_kernel<4>;
}

const void* kron_kernel_ptr(int direction, int bits) {
  if (direction == 0) return bits == 8 ? (const void*)rq_kron_kernel<8> : (const void*)rq_kron_kernel<4>;
  return bits == 8 ? (const void*)dq_kron_kernel<8> : (const void*)dq_kron_kernel<4>;
}

}  // namespace hadq
