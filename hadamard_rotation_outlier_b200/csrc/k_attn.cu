// Decode attention over the rotated INT4 KV cache.
#include "hadq_attn.cuh"
#include "hadq_kernels.h"

namespace hadq {

const void* kv_decode_attn_kernel_ptr(int ng) {
  if (ng == 4) return reinterpret_cast<const void*>(&kv_decode_attn_kernel<kAttnStages, 4>);
  if (ng == 2) return reinterpret_cast<const void*>(&kv_decode_attn_kernel<kAttnStages, 2>);
  return reinterpret_cast<const void*>(&kv_decode_attn_kernel<kAttnStages, 1>);
}

// Scratch of the allocation-free entry point: a static device array, zero
// when the module loads (so its arrival counters start at zero); every call
// leaves the counters at zero again.
__device__ __align__(256) unsigned char g_attn_scratch[kAttnStaticScratchBytes];

void* attn_static_scratch() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_attn_scratch) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return p;
}

}  // namespace hadq
