// 4096-point Hadamard blocks on tcgen05 tensor cores: instantiations, the
// TMA tensor map of the input and the device fault word of the bounded waits.
#include <cudaTypedefs.h>

#include <mutex>

#include "hadq_h4096_tc.cuh"
#include "hadq_kernels.h"

namespace hadq {

__device__ unsigned int g_tc_fault;

const void* h4096_tc_kernel_ptr(int bits, bool signs) {
  if (bits == 8) return signs ? (const void*)rq_h4096_tc_kernel<8, true> : (const void*)rq_h4096_tc_kernel<8, false>;
  return signs ? (const void*)rq_h4096_tc_kernel<4, true> : (const void*)rq_h4096_tc_kernel<4, false>;
}

size_t h4096_tc_smem() { return h4096_tc_smem_bytes(); }
int h4096_tc_threads() { return kTcThreads; }

unsigned* tc_fault_word() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_tc_fault) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return static_cast<unsigned*>(p);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (the
// library does not link the driver library itself).
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// 3-D map of nblocks 4096-point bf16 blocks as [block][h = 128][l = 32], box
// [4][128][32] (one tile), 64-byte swizzle, zero fill past the last block.
bool h4096_tc_encode_map(void* map, const void* x, int64_t nblocks) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {32, 128, cuuint64_t(nblocks)};
  cuuint64_t strides[2] = {64, 8192};
  cuuint32_t box[3] = {32, 128, kTcTileBlocks};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(static_cast<CUtensorMap*>(map), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace hadq
