// Generic path: any valid (dim, block, group, bits), any 2-byte alignment.
//
// One CTA per row at a time (grid-stride over rows).  The row is held in
// shared memory as float32; each butterfly stage is one pass over dim/2 pairs
// followed by a barrier.  Groups of up to 32 columns are reduced by one thread
// each, wider groups by one warp each.  Codes are staged in shared memory so
// that INT4 bytes whose two elements belong to different groups are written
// by one thread.  This path favours generality over speed; the blocked and
// 4096-point paths cover the common shapes.
#pragma once

#include "hadq_common.cuh"

namespace hadq {

struct GenericArgs {
  const uint16_t* x;
  const uint8_t* codes_in;
  const float* scales_in;
  const int8_t* signs;
  uint8_t* codes;
  float* scales;
  float* rot;        // forward: optional fp32 y; inverse: fp32 output
  uint16_t* out_bf16;
  int64_t rows;
  int dim;
  int block;         // B (power of two dividing dim)
  int group;         // G (divides dim)
  float scale_mul;   // 1 / (sqrt(B) * qmax)
  float rsqrt_b;     // 1 / sqrt(B)
};

// Integer code of v against the group maximum m (see quantize8).
__device__ __forceinline__ int code_of(float v, float m, float qmax) {
  uint32_t b;
  if (m >= kTinyMax) {
    b = magic_code(v, qmax / m);
  } else {
    const float pre = 18446744073709551616.0f;  // 2^64
    b = magic_code(v * pre, m > 0.0f ? qmax / (m * pre) : 0.0f);
  }
  return (int)(b - 0x4b400000u);  // bit pattern of kMagic
}

__device__ __forceinline__ void generic_stages(float* buf, int dim, int B) {
  for (int h = 1; h < B; h <<= 1) {
    for (int p = threadIdx.x; p < dim / 2; p += blockDim.x) {
      const int i = ((p & ~(h - 1)) << 1) | (p & (h - 1));
      const float x0 = buf[i], x1 = buf[i + h];
      buf[i] = x0 + x1;
      buf[i + h] = x0 - x1;
    }
    __syncthreads();
  }
}

template <int BITS>
__global__ void __launch_bounds__(256) rq_generic_kernel(GenericArgs a) {
  constexpr float QMAX = (float)((1 << (BITS - 1)) - 1);
  extern __shared__ __align__(16) float sbuf[];
  const int dim = a.dim, G = a.group;
  int8_t* scode = reinterpret_cast<int8_t*>(sbuf + dim);
  const int ngroups = dim / G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;

  for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
    const int64_t base = row * dim;
    for (int i = threadIdx.x; i < dim; i += blockDim.x) {
      float f = __uint_as_float((uint32_t)a.x[base + i] << 16);
      if (a.signs && a.signs[i] < 0) f = -f;
      sbuf[i] = f;
    }
    __syncthreads();
    generic_stages(sbuf, dim, a.block);

    if (G <= 32) {
      for (int g = threadIdx.x; g < ngroups; g += blockDim.x) {
        float m = 0.0f;
        for (int i = 0; i < G; ++i) m = fmaxf(m, fabsf(sbuf[g * G + i]));
        a.scales[row * ngroups + g] = m * a.scale_mul;
        for (int i = 0; i < G; ++i) scode[g * G + i] = (int8_t)code_of(sbuf[g * G + i], m, QMAX);
      }
    } else {
      for (int g = warp; g < ngroups; g += nwarps) {
        float m = 0.0f;
        for (int i = lane; i < G; i += 32) m = fmaxf(m, fabsf(sbuf[g * G + i]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) a.scales[row * ngroups + g] = m * a.scale_mul;
        for (int i = lane; i < G; i += 32) scode[g * G + i] = (int8_t)code_of(sbuf[g * G + i], m, QMAX);
      }
    }
    if (a.rot)
      for (int i = threadIdx.x; i < dim; i += blockDim.x) a.rot[base + i] = sbuf[i] * a.rsqrt_b;
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

template <int BITS>
__global__ void __launch_bounds__(256) dq_generic_kernel(GenericArgs a, bool out_f32) {
  extern __shared__ __align__(16) float sbuf[];
  const int dim = a.dim, G = a.group, B = a.block;
  const int ngroups = dim / G;
  const int nblk = dim / B;
  uint8_t* sflag = reinterpret_cast<uint8_t*>(sbuf + dim);  // per block: computed at 2^64 scale

  for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
    const int64_t base = row * dim;
    const float* srow = a.scales_in + row * ngroups;
    for (int b = threadIdx.x; b < nblk; b += blockDim.x) {
      bool tiny = false;
      for (int g = (b * B) / G; g <= ((b + 1) * B - 1) / G; ++g) {
        const float sc = srow[g];
        tiny |= sc < kTinyScale && sc != 0.0f;
      }
      sflag[b] = tiny;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < dim; i += blockDim.x) {
      int qv;
      if constexpr (BITS == 8) {
        qv = (int8_t)a.codes_in[base + i];
      } else {
        const uint32_t byte = a.codes_in[(base + i) >> 1];
        qv = ((int32_t)((byte >> (4 * (i & 1))) << 28)) >> 28;
      }
      const float pre = sflag[i / B] ? kUp64 : 1.0f;
      sbuf[i] = (float)qv * (srow[i / G] * pre * a.rsqrt_b);
    }
    __syncthreads();
    generic_stages(sbuf, dim, B);
    for (int i = threadIdx.x; i < dim; i += blockDim.x) {
      float f = sbuf[i];
      if (sflag[i / B]) f *= kDown64;
      if (a.signs && a.signs[i] < 0) f = -f;
      if (out_f32) {
        a.rot[base + i] = f;
      } else {
        uint32_t b = __float_as_uint(f);
        a.out_bf16[base + i] = (uint16_t)((b + 0x7fffu + ((b >> 16) & 1u)) >> 16);
      }
    }
    __syncthreads();
  }
}

}  // namespace hadq
