// Host-side accessors of the kernel instantiations, one per kernel family.
// Each returns the address to pass to cudaLaunchKernel.
#pragma once

#include <cstddef>
#include <cstdint>

namespace hadq {

// direction 0 = rotate+quantise, 1 = dequantise+inverse; threads = CTA size.
const void* blocked_kernel_ptr(int direction, int bits, int B, bool signs, bool f32, int threads);
// wide_g: the scale group covers whole 128-column chunks (G >= 128);
// team: 32 (warp teams) or 128 (CTA teams, for groups of more than 32 chunks
// or of a chunk count that does not divide 32).
const void* chunk_kernel_ptr(int bits, int B, bool signs, bool wide_g, int team);
// scale_first: some Hadamard block spans several scale groups (G < B).
const void* dq_chunk_kernel_ptr_8(int B, bool signs, bool scale_first, bool f32);
const void* dq_chunk_kernel_ptr_4(int B, bool signs, bool scale_first, bool f32);
inline const void* dq_chunk_kernel_ptr(int bits, int B, bool signs, bool scale_first, bool f32) {
  return bits == 8 ? dq_chunk_kernel_ptr_8(B, signs, scale_first, f32) : dq_chunk_kernel_ptr_4(B, signs, scale_first, f32);
}
// Kept-token variants (groups of >= 128 columns, warp teams).
const void* keep_chunk_kernel_ptr(int bits, int B, bool signs);
const void* keep_dq_chunk_kernel_ptr(int bits, int B, bool signs, bool f32);
// Kept-token variant of the 128-point tensor-core quantiser (B = G = 128).
const void* keep_chunk_mma_kernel_ptr(int bits, bool signs);
// Kronecker rotation F (x) H_b (direction 0 forward, 1 inverse), 256 threads.
const void* kron_kernel_ptr(int direction, int bits);
// Forward register variant (b and G in 16..512, dim / 16 threads per CTA).
const void* kron16_kernel_ptr(int bits);
// Forward tensor-core variant (a <= 32, ka = ceil(a / 8); dim / 16 threads);
// pm1: the factor is a +-1 matrix times 1 / sqrt(a); s256: b = 256 (strided
// shared-memory pass instead of lane shuffles).
const void* kron_tc_kernel_ptr(int bits, int ka, bool pm1, bool s256);
// Asymmetric (zero-point) variants (groups of 128 x 2^k columns, warp teams).
const void* asym_chunk_kernel_ptr(int bits, int B, bool signs);
const void* asym_dq_chunk_kernel_ptr(int bits, int B, bool signs, bool f32);
// 128-point blocks, one scale per block, with or without signs: first
// 16-point stage on tensor cores (warp teams of 32 blocks).
const void* chunk_mma_kernel_ptr(int bits, bool signs, bool rot);
// Inverse of 128-point blocks whose scale group covers whole blocks: first
// 16-point stage on tensor cores (f16 MMA on the integer codes).
const void* dq_chunk_mma_kernel_ptr(int bits, bool signs, bool f32);
// 4096-column blocks, one scale per block, one block per warp.
const void* wide4096_kernel_ptr(int bits, bool signs);
// The same with the first 16-point stage on tensor cores (kH4096Warps warps).
const void* h4096_mma_kernel_ptr(int bits, bool signs, bool rot);
// The same blocks on tcgen05 tensor cores (H_128 GEMM + five register
// stages), fed by TMA; one persistent CTA of h4096_tc_threads() per SM.
const void* h4096_tc_kernel_ptr(int bits, bool signs);
size_t h4096_tc_smem();
int h4096_tc_threads();
// Tensor map (a CUtensorMap, 64-byte aligned) of nblocks bf16 blocks at x
// (16-byte aligned); false if the driver entry point or the encode fails.
bool h4096_tc_encode_map(void* map, const void* x, int64_t nblocks);
// Device address of the word the bounded waits of the tcgen05 kernels set.
unsigned* tc_fault_word();
const void* full4096_kernel_ptr(int bits, bool signs, int logG);
const void* generic_kernel_ptr(int direction, int bits);

}  // namespace hadq

namespace hadq {

// Decode attention over the rotated INT4 or INT8 KV cache (head dim 128, ng =
// 1, 2 or 4 scales per cached row: groups of 128, 64 or 32 columns), 128
// threads per CTA, kv_decode_attn_smem(ng, bits) bytes of dynamic shared memory.
const void* kv_decode_attn_kernel_ptr(int ng, int bits);
size_t kv_decode_attn_smem(int ng, int bits);
// Device address (current device) of the library's static attention scratch
// of kAttnStaticScratchBytes, or NULL if the runtime cannot resolve it.
void* attn_static_scratch();

}  // namespace hadq
