// Kronecker rotation y = (F (x) H_b)(x * s) fused with the symmetric
// quantiser, and its inverse.
//
// The online down_proj rotation of QuaRot uses a Kronecker-product matrix,
// and widths without a Sylvester matrix take a stored Hadamard matrix
// ("QuaRot: rotation-based outlier suppression", msModelSlim, online
// rotation and FAQ).  The row of width a * b is viewed as X[a][b] (element
// i * b + j): y = vec(F X H_b^T) with F the caller's a x a factor (for a
// stored Hadamard matrix S_a: F = S_a / sqrt(a)) and H_b the Sylvester matrix.
//
// One CTA per row (grid-stride), the row in shared memory as float32:
//   1. butterflies along each b-wide sub-block (unnormalised H_b),
//   2. mixing across the a sub-blocks: out[r][j] = sum_i C[r][i] in[i][j],
//      with C = F (forward) or F^T (inverse) held transposed in shared memory;
//      a thread computes kKronR outputs of one column j from one read of each
//      input and 128-bit broadcast reads of the coefficients,
//   3. the quantiser of the generic path (forward) or the output (inverse).
// The 1/sqrt(b) of H_b is folded into the scale, as everywhere else.
#pragma once

#include "hadq_generic.cuh"

namespace hadq {

constexpr int kKronR = 8;  // outputs per thread in the mixing step

struct KronArgs {
  GenericArgs g;   // x / codes_in, scales, signs, codes / out, rows, dim = a * b, block = b, group
  const float* f;  // [a][a] factor, row-major, device memory
  int a;
  int ap;          // a rounded up to a multiple of kKronR (pitch of the transposed coefficients)
};

// Shared memory: in[dim] | out[dim] | coefficients [a][ap] | codes [dim] (int8);
// the register variant pads in and out by 4 floats per 32 (see kron_pad) and
// has no code area, which fits in the same size.
__host__ __device__ inline size_t kron_smem_bytes(int dim, int a) {
  const int ap = (a + kKronR - 1) / kKronR * kKronR;
  return size_t(2) * dim * 4 + size_t(a) * ap * 4 + ((size_t(dim) + 15) & ~size_t(15));
}

// Coefficients of the mixing step, transposed: ct[i * ap + r] = C[r][i] for
// C = F (transpose == false) or C = F^T; columns r >= a are zero.
__device__ __forceinline__ void kron_load_coeffs(const float* f, int a, int ap, bool transpose, float* ct) {
  for (int e = threadIdx.x; e < a * ap; e += blockDim.x) {
    const int i = e / ap, r = e - i * ap;
    ct[e] = r < a ? (transpose ? f[i * a + r] : f[r * a + i]) : 0.0f;
  }
}

// Shared-memory index of row element e in the register variant: 4 floats of
// padding after every 32, so that 16-float runs owned by consecutive threads
// move with conflict-free 128-bit accesses.
__device__ __forceinline__ int kron_pad(int e) { return e + ((e >> 5) << 2); }

// out[r][j] = sum_i C[r][i] in[i][j] over the a x b row (b = 2^lb).
// PAD: in and out use kron_pad indices.
template <bool PAD>
__device__ __forceinline__ void kron_mix(const float* in, float* out, const float* ct, int a, int ap, int lb) {
  const int b = 1 << lb;
  const int tiles = ap / kKronR;
  for (int o = threadIdx.x; o < tiles * b; o += blockDim.x) {
    const int rt = o >> lb, j = o & (b - 1);
    float acc[kKronR];
#pragma unroll
    for (int r = 0; r < kKronR; ++r) acc[r] = 0.0f;
    const float* cp = ct + rt * kKronR;
#pragma unroll 4
    for (int i = 0; i < a; ++i) {
      const float z = in[PAD ? kron_pad(i * b + j) : i * b + j];
      const float4 c0 = *reinterpret_cast<const float4*>(cp + i * ap);
      const float4 c1 = *reinterpret_cast<const float4*>(cp + i * ap + 4);
      acc[0] = fmaf(c0.x, z, acc[0]);
      acc[1] = fmaf(c0.y, z, acc[1]);
      acc[2] = fmaf(c0.z, z, acc[2]);
      acc[3] = fmaf(c0.w, z, acc[3]);
      acc[4] = fmaf(c1.x, z, acc[4]);
      acc[5] = fmaf(c1.y, z, acc[5]);
      acc[6] = fmaf(c1.z, z, acc[6]);
      acc[7] = fmaf(c1.w, z, acc[7]);
    }
#pragma unroll
    for (int r = 0; r < kKronR; ++r)
      if (rt * kKronR + r < a) {
        const int e = (rt * kKronR + r) * b + j;
        out[PAD ? kron_pad(e) : e] = acc[r];
      }
  }
}

__host__ __device__ inline int kron_log2(int b) {
  int l = 0;
  while ((1 << l) < b) ++l;
  return l;
}

template <int BITS>
__global__ void __launch_bounds__(256) rq_kron_kernel(KronArgs k) {
  constexpr float QMAX = (float)((1 << (BITS - 1)) - 1);
  const GenericArgs& a = k.g;
  extern __shared__ __align__(16) float kbuf[];
  const int dim = a.dim, G = a.group, b = a.block;
  float* sin = kbuf;
  float* sout = kbuf + dim;
  float* ct = kbuf + 2 * dim;
  int8_t* scode = reinterpret_cast<int8_t*>(ct + k.a * k.ap);
  const int ngroups = dim / G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  kron_load_coeffs(k.f, k.a, k.ap, false, ct);

  for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
    const int64_t base = row * dim;
    for (int i = threadIdx.x; i < dim; i += blockDim.x) {
      float f = __uint_as_float((uint32_t)a.x[base + i] << 16);
      if (a.signs && a.signs[i] < 0) f = -f;
      sin[i] = f;
    }
    __syncthreads();
    generic_stages(sin, dim, b);
    kron_mix<false>(sin, sout, ct, k.a, k.ap, kron_log2(b));
    __syncthreads();

    if (G <= 32) {
      for (int g = threadIdx.x; g < ngroups; g += blockDim.x) {
        float m = 0.0f;
        for (int i = 0; i < G; ++i) m = fmaxf(m, fabsf(sout[g * G + i]));
        a.scales[row * ngroups + g] = m * a.scale_mul;
        for (int i = 0; i < G; ++i) scode[g * G + i] = (int8_t)code_of(sout[g * G + i], m, QMAX);
      }
    } else {
      for (int g = warp; g < ngroups; g += nwarps) {
        float m = 0.0f;
        for (int i = lane; i < G; i += 32) m = fmaxf(m, fabsf(sout[g * G + i]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) a.scales[row * ngroups + g] = m * a.scale_mul;
        for (int i = lane; i < G; i += 32) scode[g * G + i] = (int8_t)code_of(sout[g * G + i], m, QMAX);
      }
    }
    if (a.rot)
      for (int i = threadIdx.x; i < dim; i += blockDim.x) a.rot[base + i] = sout[i] * a.rsqrt_b;
    __syncthreads();

    if constexpr (BITS == 8) {
      for (int i = threadIdx.x; i < dim; i += blockDim.x) a.codes[base + i] = (uint8_t)scode[i];
    } else {
      for (int p = threadIdx.x; p < dim / 2; p += blockDim.x)
        a.codes[base / 2 + p] = (uint8_t)((scode[2 * p] & 0xf) | ((scode[2 * p + 1] & 0xf) << 4));
    }
    __syncthreads();
  }
}

// Inverse: q * scale -> mixing with F^T -> butterflies -> signs -> output.
// Rows whose scales fall below 2^-100 run at 2^64 scale and are scaled back
// once at the end (the factor may mix every block, so the row is one unit).
template <int BITS>
__global__ void __launch_bounds__(256) dq_kron_kernel(KronArgs k, bool out_f32) {
  const GenericArgs& a = k.g;
  extern __shared__ __align__(16) float kbuf[];
  const int dim = a.dim, G = a.group, b = a.block;
  float* sin = kbuf;
  float* sout = kbuf + dim;
  float* ct = kbuf + 2 * dim;
  int* stiny = reinterpret_cast<int*>(ct + k.a * k.ap);
  const int ngroups = dim / G;
  kron_load_coeffs(k.f, k.a, k.ap, true, ct);

  for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
    const int64_t base = row * dim;
    const float* srow = a.scales_in + row * ngroups;
    if (threadIdx.x == 0) *stiny = 0;
    __syncthreads();
    for (int g = threadIdx.x; g < ngroups; g += blockDim.x)
      if (srow[g] < kTinyScale && srow[g] != 0.0f) *stiny = 1;
    __syncthreads();
    const bool tiny = *stiny != 0;
    const float pre = (tiny ? kUp64 : 1.0f) * a.rsqrt_b;
    for (int i = threadIdx.x; i < dim; i += blockDim.x) {
      int qv;
      if constexpr (BITS == 8) {
        qv = (int8_t)a.codes_in[base + i];
      } else {
        const uint32_t byte = a.codes_in[(base + i) >> 1];
        qv = ((int32_t)((byte >> (4 * (i & 1))) << 28)) >> 28;
      }
      sin[i] = (float)qv * (srow[i / G] * pre);
    }
    __syncthreads();
    kron_mix<false>(sin, sout, ct, k.a, k.ap, kron_log2(b));
    __syncthreads();
    generic_stages(sout, dim, b);
    for (int i = threadIdx.x; i < dim; i += blockDim.x) {
      float f = sout[i];
      if (tiny) f *= kDown64;
      if (a.signs && a.signs[i] < 0) f = -f;
      if (out_f32) {
        a.rot[base + i] = f;
      } else {
        uint32_t bb = __float_as_uint(f);
        a.out_bf16[base + i] = (uint16_t)((bb + 0x7fffu + ((bb >> 16) & 1u)) >> 16);
      }
    }
    __syncthreads();
  }
}

// Register variant for b in 16..512 and groups of 16..512 columns (powers of
// two): one thread per 16 consecutive elements of the row (dim / 16 threads,
// at most 1024), so
//   - the b-butterflies run on bits 0-3 in registers and on the remaining
//     bits across the b / 16 lanes of the sub-block (lane shuffles, inside
//     one warp since b / 16 <= 32),
//   - the mixing goes through shared memory as above,
//   - each group's maximum is a shuffle over its G / 16 lanes and the codes
//     leave from registers.
template <int BITS>
__global__ void __launch_bounds__(1024) rq_kron16_kernel(KronArgs k) {
  constexpr float QMAX = (float)((1 << (BITS - 1)) - 1);
  const GenericArgs& a = k.g;
  extern __shared__ __align__(16) float kbuf[];
  const int dim = a.dim, b = a.block, G = a.group;
  const int pdim = kron_pad(dim);  // padded row length (a multiple of 4)
  float* sin = kbuf;
  float* sout = kbuf + pdim;
  float* ct = kbuf + 2 * pdim;
  const int t = threadIdx.x;
  const int e0 = 16 * t;
  const int lane = t & 31;
  const int lanes_b = b >> 4;  // lanes per sub-block
  const int lanes_g = G >> 4;  // lanes per scale group
  const int lb = kron_log2(b);
  kron_load_coeffs(k.f, k.a, k.ap, false, ct);
  // sign masks of this thread's 16 columns (bf16 pairs)
  uint32_t smask[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) smask[i] = 0u;
  if (a.signs) {
    const uint4 sg = *reinterpret_cast<const uint4*>(a.signs + e0);
    const uint32_t w[4] = {sg.x, sg.y, sg.z, sg.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t word = w[i >> 1];
      const int sh = 16 * (i & 1);
      smask[i] = (((word >> (sh + 7)) & 1u) << 15) | (((word >> (sh + 15)) & 1u) << 31);
    }
  }

  for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
    const int64_t base = row * dim;
    float v[16];
    {
      const uint4* src = reinterpret_cast<const uint4*>(a.x + base + e0);
      const uint4 r0 = src[0], r1 = src[1];
      const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) bf16_pair_stage1(w[i] ^ smask[i], v[2 * i], v[2 * i + 1]);
    }
    reg_fwht_from<16, 1, 4>(v);
    for (int m = 1; m < lanes_b; m <<= 1) {  // bits 4.. of the sub-block index: lanes
      const float sg = (lane & m) ? -1.0f : 1.0f;
      lane_stage<16>(v, m, sg);
    }
#pragma unroll
    for (int i = 0; i < 16; i += 4)
      *reinterpret_cast<float4*>(sin + kron_pad(e0 + i)) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    __syncthreads();
    kron_mix<true>(sin, sout, ct, k.a, k.ap, lb);
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 16; i += 4) {
      const float4 q = *reinterpret_cast<const float4*>(sout + kron_pad(e0 + i));
      v[i] = q.x;
      v[i + 1] = q.y;
      v[i + 2] = q.z;
      v[i + 3] = q.w;
    }
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
    for (int o = 1; o < lanes_g; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((t & (lanes_g - 1)) == 0) a.scales[(base + e0) / G] = m * a.scale_mul;
    if (a.rot) {
      float4* dst = reinterpret_cast<float4*>(a.rot + base + e0);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        dst[i] = make_float4(v[4 * i] * a.rsqrt_b, v[4 * i + 1] * a.rsqrt_b, v[4 * i + 2] * a.rsqrt_b,
                             v[4 * i + 3] * a.rsqrt_b);
    }
    uint32_t cc0[8], cc1[8];
    quantize8(v, m, QMAX, cc0);
    quantize8(v + 8, m, QMAX, cc1);
    if constexpr (BITS == 8) {
      *reinterpret_cast<uint4*>(a.codes + base + e0) =
          make_uint4(pack_i8x4(cc0[0], cc0[1], cc0[2], cc0[3]), pack_i8x4(cc0[4], cc0[5], cc0[6], cc0[7]),
                     pack_i8x4(cc1[0], cc1[1], cc1[2], cc1[3]), pack_i8x4(cc1[4], cc1[5], cc1[6], cc1[7]));
    } else {
      *reinterpret_cast<uint2*>(a.codes + (base + e0) / 2) = make_uint2(pack_i4x8(cc0), pack_i4x8(cc1));
    }
    __syncthreads();  // sin / sout are reused by the next row
  }
}

}  // namespace hadq
