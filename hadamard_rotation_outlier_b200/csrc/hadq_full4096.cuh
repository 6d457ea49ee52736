// Full 4096-point path: one Hadamard block over a 4096-wide row.
//
// 64 threads (two warps) own one row, 64 elements each, and the 12 butterfly
// stages run in two register phases joined by one shared-memory transpose:
//
//   P1 (load layout)   thread u holds x[512 j + 8 u + k], j,k = 0..7, loaded as
//                      eight coalesced 16-byte vectors.  Registers cover index
//                      bits {0,1,2} (k) and {9,10,11} (j): six stages.
//   transpose          values go to shared memory as A[hi][k][m] (hi = bits
//                      9..11, k = bits 0..2, m = bits 3..8), rows of 64 floats
//                      padded to 68 so both sides are conflict-free.
//   P2                 thread t = (hi, k) reads A[hi][k][0..63] with 16-byte
//                      loads: registers cover bits 3..8, six more stages.  All
//                      12 stages are now done; group maxima and codes are
//                      computed here.
//   code transpose     codes go to shared memory as bytes in natural order
//                      (padded), and P3 reads them back in the load layout so
//                      the global stores are 8-byte (INT8) or 4-byte (INT4)
//                      vectors of consecutive elements.
//
// Scale groups are G = 2^LOG_G columns (template), 64 <= G <= 4096.
#pragma once

#include "hadq_common.cuh"

namespace hadq {

struct FullArgs {
  const uint16_t* x;
  const int8_t* signs;
  uint8_t* codes;
  float* scales;
  float* rot;
  int64_t rows;
  float scale_mul;  // 1 / (64 * qmax)
  float rsqrt_b;    // 1 / 64
};

constexpr int kF_ROWF = 68;   // padded row of the float transpose (floats)
constexpr int kF_ROWC = 520;  // padded 512-byte chunk of the code transpose

template <int BITS, bool SIGNS, int LOG_G>
__global__ void __launch_bounds__(64) rq_full4096_kernel(FullArgs a) {
  constexpr float QMAX = (float)((1 << (BITS - 1)) - 1);
  constexpr int IN = (LOG_G - 3) < 6 ? (LOG_G - 3) : 6;  // register bits inside one group (P2)
  constexpr int NP = 64 >> IN;                            // group partials per thread (P2)
  static_assert(LOG_G >= 6 && LOG_G <= 12, "group size 64..4096");

  __shared__ __align__(16) float sA[64 * kF_ROWF];
  __shared__ __align__(16) uint8_t sC[8 * kF_ROWC];
  __shared__ float sRed[2][2];

  const int u = threadIdx.x;     // P1/P3 role
  const int hi = u >> 3;         // P2 role: index bits 9..11
  const int kk = u & 7;          // P2 role: index bits 0..2
  const int warp = u >> 5;

  uint32_t msk[SIGNS ? 32 : 1];
  if constexpr (SIGNS) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint2 s2 = *reinterpret_cast<const uint2*>(a.signs + 512 * j + 8 * u);
      uint32_t w[2] = {s2.x, s2.y};
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int p = 0; p < 2; ++p)
          msk[4 * j + 2 * h + p] = pair_sign_mask((int8_t)(w[h] >> (16 * p)), (int8_t)(w[h] >> (16 * p + 8)));
    }
  }

  int par = 0;
  for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
    const uint16_t* xr = a.x + row * 4096;
    float v[64];
    {
      uint4 raw[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) raw[j] = __ldg(reinterpret_cast<const uint4*>(xr + 512 * j + 8 * u));
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t w[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          uint32_t ww = w[p];
          if constexpr (SIGNS) ww ^= msk[4 * j + p];
          v[8 * j + 2 * p] = bf16lo(ww);
          v[8 * j + 2 * p + 1] = bf16hi(ww);
        }
      }
    }
    reg_fwht<64, 6>(v);  // bits 0..2 and 9..11

#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int k = 0; k < 8; ++k) sA[(j * 8 + k) * kF_ROWF + u] = v[8 * j + k];
    __syncthreads();

#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float4 f = *reinterpret_cast<const float4*>(&sA[u * kF_ROWF + 4 * i]);  // u = hi*8 + k
      v[4 * i] = f.x;
      v[4 * i + 1] = f.y;
      v[4 * i + 2] = f.z;
      v[4 * i + 3] = f.w;
    }
    reg_fwht<64, 6>(v);  // bits 3..8: all 12 stages done; v[m] is element (hi<<9)|(m<<3)|kk

    // group maxima over index bits < LOG_G
    float pm[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      float m = 0.0f;
#pragma unroll
      for (int r = 0; r < (1 << IN); ++r) m = fmaxf(m, fabsf(v[(p << IN) + r]));
      pm[p] = m;
    }
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      pm[p] = fmaxf(pm[p], __shfl_xor_sync(0xffffffffu, pm[p], 1));
      pm[p] = fmaxf(pm[p], __shfl_xor_sync(0xffffffffu, pm[p], 2));
      pm[p] = fmaxf(pm[p], __shfl_xor_sync(0xffffffffu, pm[p], 4));
      if constexpr (LOG_G > 9) pm[p] = fmaxf(pm[p], __shfl_xor_sync(0xffffffffu, pm[p], 8));
      if constexpr (LOG_G > 10) pm[p] = fmaxf(pm[p], __shfl_xor_sync(0xffffffffu, pm[p], 16));
    }
    if constexpr (LOG_G > 11) {
      if ((u & 31) == 0) sRed[par][warp] = pm[0];
      __syncthreads();
      pm[0] = fmaxf(sRed[par][0], sRed[par][1]);
      par ^= 1;
    }

    // scales: the thread holding the first element of each group writes it
    constexpr int HI_IN = LOG_G > 9 ? (1 << (LOG_G - 9)) - 1 : 0;  // hi bits inside a group
    if (kk == 0 && (hi & HI_IN) == 0) {
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const int e0 = (hi << 9) | (p << (3 + IN));
        a.scales[row * (4096 >> LOG_G) + (e0 >> LOG_G)] = pm[p] * a.scale_mul;
      }
    }
    if (a.rot) {
      float* rr = a.rot + row * 4096 + (hi << 9) + kk;
#pragma unroll
      for (int m = 0; m < 64; ++m) rr[m << 3] = v[m] * a.rsqrt_b;
    }

    uint8_t* cw = sC + hi * kF_ROWC + kk;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      uint32_t cc[8];
#pragma unroll
      for (int r0 = 0; r0 < (1 << IN); r0 += 8) {
        quantize8(v + (p << IN) + r0, pm[p], QMAX, cc);
#pragma unroll
        for (int r = 0; r < 8; ++r) cw[((p << IN) + r0 + r) << 3] = (uint8_t)cc[r];
      }
    }
    __syncthreads();

    // P3: codes back in the load layout
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint2 w = *reinterpret_cast<const uint2*>(sC + j * kF_ROWC + 8 * u);
      const int64_t e = row * 4096 + 512 * j + 8 * u;
      if constexpr (BITS == 8) {
        *reinterpret_cast<uint2*>(a.codes + e) = w;
      } else {
        *reinterpret_cast<uint32_t*>(a.codes + e / 2) = nibble_pack(w.x, w.y);
      }
    }
    // The next row's writes to sA follow this row's reads of sA (before the
    // second barrier); its writes to sC follow the next row's first barrier,
    // which every thread reaches only after these reads of sC.
  }
}

}  // namespace hadq
