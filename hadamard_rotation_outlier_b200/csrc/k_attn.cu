// Decode attention over the rotated INT4 KV cache.
#include "hadq_attn.cuh"
#include "hadq_kernels.h"

namespace hadq {

const void* kv_decode_attn_kernel_ptr() { return reinterpret_cast<const void*>(&kv_decode_attn_kernel<kAttnStages>); }

}  // namespace hadq
