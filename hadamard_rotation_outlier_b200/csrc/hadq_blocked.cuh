// Blocked path: Hadamard blocks of B = 32..256 columns, rows up to 16384 wide.
//
// Thread layout.  Every thread owns E = 32 elements of one block: four 16-byte
// vectors j = 0..3 of 8 bf16 each.  The T = B/32 threads of a block are
// consecutive lanes q = 0..T-1, and vector j of lane q holds block elements
//     e = 8*T*j + 8*q + k,   k = 0..7.
// So element-index bits 0..2 (k) and the two top bits (j) live in registers
// and are transformed in place (five stages); the log2(T) middle bits (q) are
// transformed with lane shuffles.  All loads and stores are 16/8/4-byte
// vectors, and the 4 lanes x 16 B of one vector index form whole 32-byte
// sectors.
//
// CTA size.  MAXT = 256 threads for rows up to 8192 wide (several rows per
// CTA), 512 for wider rows (one row per CTA).
//
// Row slabs.  A CTA handles whole rows: the dim/32 threads of a row are
// consecutive, a CTA holds rpi rows, and it walks over slabs of rpi rows with
// a grid-stride loop.  A thread therefore always sees the same columns, so its
// sign masks are loaded once.  Scale groups inside a block (G <= B, G = 2^g >= 8)
// reduce in registers and shuffles; groups spanning several blocks (G a
// multiple of B) add one shared-memory max per slab.
#pragma once

#include "hadq_common.cuh"

namespace hadq {

struct BlockedArgs {
  const uint16_t* x;      // forward: bf16 input
  const uint8_t* codes_in;  // inverse: codes
  const float* scales_in;   // inverse: scales
  const int8_t* signs;
  uint8_t* codes;         // forward outputs
  float* scales;
  float* rot;             // optional fp32 copy of y (forward) / fp32 output (inverse)
  uint16_t* out_bf16;     // inverse bf16 output
  int64_t rows;
  int64_t nslabs;
  int dim;
  int group;              // G in columns (already resolved from -1)
  int rpi;                // rows per slab
  int tpr;                // threads per row = dim / 32
  float scale_mul;        // 1 / (sqrt(B) * qmax): y-scale from the max of unnormalised values
  float rsqrt_b;          // 1 / sqrt(B)
};

template <int LOG_B>
struct BlockedGeom {
  static constexpr int B = 1 << LOG_B;
  static constexpr int T = B / 32;          // lanes per block
  static constexpr int LOG_T = LOG_B - 5;
};

// Forward: bf16 -> signs -> H_B -> absmax -> codes + scales.
template <int LOG_B, int BITS, bool SIGNS, int MAXT>
__global__ void __launch_bounds__(MAXT, MAXT == 256 ? 3 : 1) rq_blocked_kernel(BlockedArgs a) {
  using Geo = BlockedGeom<LOG_B>;
  constexpr int B = Geo::B, T = Geo::T, LOG_T = Geo::LOG_T;
  constexpr float QMAX = (float)((1 << (BITS - 1)) - 1);
  extern __shared__ uint32_t s_gmax[];  // [3][rpi][ngroups] for groups wider than a block

  const int tid = threadIdx.x;
  const int rho = tid / a.tpr;          // row inside the slab
  const int u = tid - rho * a.tpr;      // thread inside the row
  const int c = u / T;                  // block index inside the row
  const int q = u - c * T;              // lane inside the block
  const bool lane_ok = rho < a.rpi;
  const int dim = a.dim;
  const int G = a.group;
  const bool wide = G > B;
  const int ngroups = dim / G;
  const int col0 = c * B + 8 * q;       // column of element (j=0, k=0)

  uint32_t msk[SIGNS ? 16 : 1];
  if constexpr (SIGNS) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint2 s2 = lane_ok ? *reinterpret_cast<const uint2*>(a.signs + col0 + 8 * T * j) : make_uint2(0, 0);
      uint32_t w[2] = {s2.x, s2.y};
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int p = 0; p < 2; ++p)
          msk[4 * j + 2 * h + p] = pair_sign_mask((int8_t)(w[h] >> (16 * p)), (int8_t)(w[h] >> (16 * p + 8)));
    }
  }

  if (wide) {
    for (int i = tid; i < 3 * a.rpi * ngroups; i += blockDim.x) s_gmax[i] = 0u;
    __syncthreads();
  }

  float sgn[LOG_T > 0 ? LOG_T : 1];
#pragma unroll
  for (int b = 0; b < LOG_T; ++b) sgn[b] = ((q >> b) & 1) ? -1.0f : 1.0f;

  int buf = 0;
  for (int64_t slab = blockIdx.x; slab < a.nslabs; slab += gridDim.x) {
    const int64_t row = slab * a.rpi + rho;
    const bool active = lane_ok && row < a.rows;
    const int64_t base = row * dim + col0;

    float v[32];
    {
      uint4 raw[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        raw[j] = active ? __ldg(reinterpret_cast<const uint4*>(a.x + base + 8 * T * j)) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
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

    reg_fwht<32, 5>(v);
#pragma unroll
    for (int b = 0; b < LOG_T; ++b) lane_stage<32>(v, 1 << b, sgn[b]);

    // ---- group maxima of |y| (unnormalised) ----
    float gm[4];
    if (G >= B) {
      float m = 0.0f;
#pragma unroll
      for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
#pragma unroll
      for (int b = 0; b < LOG_T; ++b) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1 << b));
      if (wide) {
        uint32_t* slot = s_gmax + (buf * a.rpi + (lane_ok ? rho : 0)) * ngroups + (c * B) / G;
        if (active && q == 0) atomicMax(slot, __float_as_uint(m));
        __syncthreads();
        m = __uint_as_float(*slot);
        // clear the buffer used two slabs ahead (no thread can still read it)
        const int nb = (buf + 2) % 3;
        for (int i = tid; i < a.rpi * ngroups; i += blockDim.x) s_gmax[nb * a.rpi * ngroups + i] = 0u;
        buf = (buf + 1) % 3;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) gm[j] = m;
    } else {
      // G = 2^g with 8 <= G < B: reduce element bits below g only.
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float m = 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k) m = fmaxf(m, fabsf(v[8 * j + k]));
        gm[j] = m;
      }
      if (G > 8 * T) {  // j bit 0 (element bit 3+LOG_T) is inside the group
        float t0 = fmaxf(gm[0], gm[1]), t1 = fmaxf(gm[2], gm[3]);
        gm[0] = gm[1] = t0;
        gm[2] = gm[3] = t1;
      }
#pragma unroll
      for (int b = 0; b < LOG_T; ++b) {
        if (G > (8 << b)) {
#pragma unroll
          for (int j = 0; j < 4; ++j) gm[j] = fmaxf(gm[j], __shfl_xor_sync(0xffffffffu, gm[j], 1 << b));
        }
      }
    }

    if (active) {
      // scales: written by the thread holding the first element of each group
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = c * B + 8 * T * j + 8 * q;
        if ((e % G) == 0) a.scales[row * ngroups + e / G] = gm[j] * a.scale_mul;
      }
      if (a.rot) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float4* dst = reinterpret_cast<float4*>(a.rot + base + 8 * T * j);
          dst[0] = make_float4(v[8 * j] * a.rsqrt_b, v[8 * j + 1] * a.rsqrt_b, v[8 * j + 2] * a.rsqrt_b, v[8 * j + 3] * a.rsqrt_b);
          dst[1] = make_float4(v[8 * j + 4] * a.rsqrt_b, v[8 * j + 5] * a.rsqrt_b, v[8 * j + 6] * a.rsqrt_b, v[8 * j + 7] * a.rsqrt_b);
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t cc[8];
        quantize8(v + 8 * j, gm[j], QMAX, cc);
        if constexpr (BITS == 8) {
          uint2 w = make_uint2(pack_i8x4(cc[0], cc[1], cc[2], cc[3]), pack_i8x4(cc[4], cc[5], cc[6], cc[7]));
          *reinterpret_cast<uint2*>(a.codes + base + 8 * T * j) = w;
        } else {
          *reinterpret_cast<uint32_t*>(a.codes + (base + 8 * T * j) / 2) = pack_i4x8(cc);
        }
      }
    }
  }
}

// Inverse: codes * scale -> H_B -> signs -> bf16 or fp32.
template <int LOG_B, int BITS, bool SIGNS, bool OUT_F32, int MAXT>
__global__ void __launch_bounds__(MAXT, MAXT == 256 ? 3 : 1) dq_blocked_kernel(BlockedArgs a) {
  using Geo = BlockedGeom<LOG_B>;
  constexpr int B = Geo::B, T = Geo::T, LOG_T = Geo::LOG_T;

  const int tid = threadIdx.x;
  const int rho = tid / a.tpr;
  const int u = tid - rho * a.tpr;
  const int c = u / T;
  const int q = u - c * T;
  const bool lane_ok = rho < a.rpi;
  const int dim = a.dim;
  const int G = a.group;
  const int ngroups = dim / G;
  const int col0 = c * B + 8 * q;

  uint32_t msk[SIGNS ? 16 : 1];
  if constexpr (SIGNS) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint2 s2 = lane_ok ? *reinterpret_cast<const uint2*>(a.signs + col0 + 8 * T * j) : make_uint2(0, 0);
      uint32_t w[2] = {s2.x, s2.y};
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int p = 0; p < 2; ++p)
          msk[4 * j + 2 * h + p] = pair_sign_mask((int8_t)(w[h] >> (16 * p)), (int8_t)(w[h] >> (16 * p + 8)));
    }
  }

  float sgn[LOG_T > 0 ? LOG_T : 1];
#pragma unroll
  for (int b = 0; b < LOG_T; ++b) sgn[b] = ((q >> b) & 1) ? -1.0f : 1.0f;

  for (int64_t slab = blockIdx.x; slab < a.nslabs; slab += gridDim.x) {
    const int64_t row = slab * a.rpi + rho;
    const bool active = lane_ok && row < a.rows;
    const int64_t base = row * dim + col0;

    // Blocks with a scale below 2^-100 would run the butterflies on subnormal
    // values (each add rounding to the 2^-149 grid); they run at 2^64 times
    // their value instead and are scaled back once at the end (exact factors).
    float sc[4];
    bool tiny = false;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = c * B + 8 * T * j + 8 * q;
      sc[j] = active ? __ldg(a.scales_in + row * ngroups + e / G) : 0.0f;
      tiny |= sc[j] < kTinyScale && sc[j] != 0.0f;
    }
#pragma unroll
    for (int b = 0; b < LOG_T; ++b) tiny |= __shfl_xor_sync(0xffffffffu, (int)tiny, 1 << b) != 0;
    const float pre = tiny ? kUp64 : 1.0f;

    float v[32];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float s = sc[j] * pre * a.rsqrt_b;
      if constexpr (BITS == 8) {
        uint2 w = active ? __ldg(reinterpret_cast<const uint2*>(a.codes_in + base + 8 * T * j)) : make_uint2(0, 0);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          v[8 * j + k] = i8_at(w.x, k) * s;
          v[8 * j + 4 + k] = i8_at(w.y, k) * s;
        }
      } else {
        uint32_t w = active ? __ldg(reinterpret_cast<const uint32_t*>(a.codes_in + (base + 8 * T * j) / 2)) : 0u;
#pragma unroll
        for (int k = 0; k < 8; ++k) v[8 * j + k] = i4_at(w, k) * s;
      }
    }

    reg_fwht<32, 5>(v);
#pragma unroll
    for (int b = 0; b < LOG_T; ++b) lane_stage<32>(v, 1 << b, sgn[b]);
    if (tiny) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= kDown64;
    }

    if (active) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if constexpr (OUT_F32) {
          uint32_t o[8];
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            uint32_t lo = __float_as_uint(v[8 * j + 2 * p]), hi = __float_as_uint(v[8 * j + 2 * p + 1]);
            if constexpr (SIGNS) {
              lo ^= msk[4 * j + p] << 16;
              hi ^= msk[4 * j + p] & 0x80000000u;
            }
            o[2 * p] = lo;
            o[2 * p + 1] = hi;
          }
          uint4* dst = reinterpret_cast<uint4*>(a.rot + base + 8 * T * j);
          dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
          dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
        } else {
          uint32_t o[4];
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            o[p] = pack_bf16x2(v[8 * j + 2 * p], v[8 * j + 2 * p + 1]);
            if constexpr (SIGNS) o[p] ^= msk[4 * j + p];
          }
          *reinterpret_cast<uint4*>(a.out_bf16 + base + 8 * T * j) = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
    }
  }
}

}  // namespace hadq
