// Decode attention over the rotated INT4 or INT8 KV cache.
#include "hadq_attn.cuh"
#include "hadq_kernels.h"

namespace hadq {

const void* kv_decode_attn_kernel_ptr(int ng, int bits) {
  if (bits == 8) {
    if (ng == 4) return reinterpret_cast<const void*>(&kv_decode_attn_kernel<kAttnStages8, 4, 8>);
    if (ng == 2) return reinterpret_cast<const void*>(&kv_decode_attn_kernel<kAttnStages8, 2, 8>);
    return reinterpret_cast<const void*>(&kv_decode_attn_kernel<kAttnStages8, 1, 8>);
  }
  if (ng == 4) return reinterpret_cast<const void*>(&kv_decode_attn_kernel<kAttnStages, 4, 4>);
  if (ng == 2) return reinterpret_cast<const void*>(&kv_decode_attn_kernel<kAttnStages, 2, 4>);
  return reinterpret_cast<const void*>(&kv_decode_attn_kernel<kAttnStages, 1, 4>);
}

size_t kv_decode_attn_smem(int ng, int bits) {
  if (bits == 8)
    return ng == 4 ? sizeof(AttnSmem<kAttnStages8, 4, 8>)
                   : ng == 2 ? sizeof(AttnSmem<kAttnStages8, 2, 8>) : sizeof(AttnSmem<kAttnStages8, 1, 8>);
  return ng == 4 ? sizeof(AttnSmem<kAttnStages, 4, 4>)
                 : ng == 2 ? sizeof(AttnSmem<kAttnStages, 2, 4>) : sizeof(AttnSmem<kAttnStages, 1, 4>);
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
