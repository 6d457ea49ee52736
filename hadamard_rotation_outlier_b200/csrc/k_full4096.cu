// Kernel pointers of one kernel family, instantiated in this translation unit
// (the families compile in parallel; the C ABI in hadq_api.cu only calls these).
#include "hadq_kernels.h"
#include "hadq_full4096.cuh"

namespace hadq {
namespace {

template <int BITS, bool SIGNS>
const void* full_fn(int logG) {
  switch (logG) {
    case 6: return (const void*)rq_full4096_kernel<BITS, SIGNS, 6>;
    case 7: return (const void*)rq_full4096_kernel<BITS, SIGNS, 7>;
    case 8: return (const void*)rq_full4096_kernel<BITS, SIGNS, 8>;
    case 9: return (const void*)rq_full4096_kernel<BITS, SIGNS, 9>;
    case 10: return (const void*)rq_full4096_kernel<BITS, SIGNS, 10>;
    case 11: return (const void*)rq_full4096_kernel<BITS, SIGNS, 11>;
    default: return (const void*)rq_full4096_kernel<BITS, SIGNS, 12>;
  }
}

}  // namespace

const void* full4096_kernel_ptr(int bits, bool signs, int logG) {
  return bits == 8 ? (signs ? full_fn<8, true>(logG) : full_fn<8, false>(logG))
                   : (signs ? full_fn<4, true>(logG) : full_fn<4, false>(logG));
}

}  // namespace hadq
