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

template <int BITS, int NS, bool S256>
static const void* kron_tc_for(int ka) {
  switch (ka) {
    case 1: return (const void*)rq_kron_tc_kernel<BITS, 1, NS, S256>;
    case 2: return (const void*)rq_kron_tc_kernel<BITS, 2, NS, S256>;
    case 3: return (const void*)rq_kron_tc_kernel<BITS, 3, NS, S256>;
    case 4: return (const void*)rq_kron_tc_kernel<BITS, 4, NS, S256>;
    default: return nullptr;
  }
}

template <int BITS, int NS>
static const void* kron_tc_for_b(int ka, bool s256) {
  return s256 ? kron_tc_for<BITS, NS, true>(ka) : kron_tc_for<BITS, NS, false>(ka);
}

const void* kron_tc_kernel_ptr(int bits, int ka, bool pm1, bool s256) {
  if (pm1) return bits == 8 ? kron_tc_for_b<8, 1>(ka, s256) : kron_tc_for_b<4, 1>(ka, s256);
  return bits == 8 ? kron_tc_for_b<8, 3>(ka, s256) : kron_tc_for_b<4, 3>(ka, s256);
}

}  // namespace hadq
