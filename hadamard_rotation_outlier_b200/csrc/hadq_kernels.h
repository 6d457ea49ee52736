// Host-side accessors of the kernel instantiations, one per kernel family.
// Each returns the address to pass to cudaLaunchKernel.
#pragma once

namespace hadq {

// direction 0 = rotate+quantise, 1 = dequantise+inverse; threads = CTA size.
const void* blocked_kernel_ptr(int direction, int bits, int B, bool signs, bool f32, int threads);
// wide_g: the scale group covers whole 128-column chunks (G >= 128).
const void* chunk_kernel_ptr(int bits, int B, bool signs, bool wide_g);
const void* full4096_kernel_ptr(int bits, bool signs, int logG);
const void* generic_kernel_ptr(int direction, int bits);

}  // namespace hadq
