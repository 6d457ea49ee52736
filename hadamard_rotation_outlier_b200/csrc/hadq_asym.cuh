// Asymmetric (zero-point) rotate+quantise and its inverse, on the chunk
// pipeline (warp teams, one 128-column chunk per thread, slabs staged through
// shared memory, groups of 128 x {1, 2, 4, .., 32} columns).
//
// Quantiser ("Hartmann rotation, lightweight QAT, streaming attention",
// section 2, the FakeQuantize forward): x_int = round(x / scale) + zero_point,
// clamped to [0, 2^b - 1], dequantised as (x_int - zero_point) * scale.  Scale
// and zero point come from the group's range, which always holds 0:
//   lo = min(0, min y), hi = max(0, max y), scale = (hi - lo) / (2^b - 1),
//   zero_point = clamp(round(-lo / scale), 0, 2^b - 1).
// In the unnormalised butterfly units v = sqrt(B) y the multiplier is
// inv = (2^b - 1) / (hi_v - lo_v): the sqrt(B) cancels, as in the symmetric
// kernels, and scale = (hi_v - lo_v) * rsqrt(B) / (2^b - 1).
#pragma once

#include "hadq_chunk.cuh"

namespace hadq {

struct ChunkAsymArgs : ChunkArgs {
  uint8_t* zp;           // forward output: one zero point per group
  const uint8_t* zp_in;  // inverse input
};

__device__ __forceinline__ float min3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Unsigned codes of eight values: round(v * inv) (half to even, from the
// magic-number sum) plus the zero point, clamped to [0, qmax]; the low bits of
// each result are the code.
__device__ __forceinline__ void asym_codes8(const float* v, float inv, int zp, int qmax, uint32_t (&c)[8]) {
  const int off = zp - int(__float_as_uint(kMagic));
#pragma unroll
  for (int k = 0; k < 8; k += 2) {
    uint32_t b0, b1;
    magic_code2(v[k], v[k + 1], inv, b0, b1);
    c[k] = uint32_t(min(max(int(b0) + off, 0), qmax));
    c[k + 1] = uint32_t(min(max(int(b1) + off, 0), qmax));
  }
}

// Forward: bf16 -> signs -> H_B (B = 2^LOG_B, 8..128) -> group range -> codes,
// scale and zero point.
template <int LOG_B, int BITS, bool SIGNS>
__global__ void __launch_bounds__(kCT, 3) rq_chunk_asym_kernel(ChunkAsymArgs a) {
  using T = Team<32>;
  constexpr int QMAXU = (1 << BITS) - 1;
  constexpr int CB = BITS == 8 ? 128 : 64;  // code bytes per chunk
  extern __shared__ __align__(16) uint8_t smem[];
  uint4* s_tab = reinterpret_cast<uint4*>(smem + 2 * chunk_stage_bytes());
  uint32_t* s_bits = reinterpret_cast<uint32_t*>(smem + 2 * chunk_stage_bytes() + kSignTabBytes);
  const int tt = T::tid();
  if constexpr (SIGNS) {
    load_sign_tables(a.signs, a.dim, s_tab, s_bits);
    __syncthreads();
  }
  const uint8_t* xsrc = reinterpret_cast<const uint8_t*>(a.x);
  const int64_t nslabs = (a.nchunks + 31) / 32;
  int colc = SIGNS ? (int)((T::first() * 32 + tt) % a.cpr) : 0;
  const int col_step = SIGNS ? (int)((T::stride() * 32) % a.cpr) : 0;
  const bool glead = (tt % a.gpc) == 0;
  uint8_t* st0 = T::stage(smem, 0);
  uint8_t* st1 = T::stage(smem, 1);

  int64_t slab = T::first();
  if (slab < nslabs) chunk_load<16, 32>(xsrc + slab * 32 * 256, slab_count(slab * 32, a.nchunks, 32), st0, tt);
  cp_async_commit();
  for (int it = 0; slab < nslabs; ++it, slab += T::stride()) {
    uint8_t* cur = (it & 1) ? st1 : st0;
    const int64_t c = slab * 32;
    cp_async_wait<0>();
    T::sync();
    {
      const int64_t nx = slab + T::stride();
      if (nx < nslabs) chunk_load<16, 32>(xsrc + nx * 32 * 256, slab_count(nx * 32, a.nchunks, 32), (it & 1) ? st0 : st1, tt);
      cp_async_commit();
    }
    const int nch = slab_count(c, a.nchunks, 32);
    const int64_t ch = c + tt;
    const bool active = tt < nch;  // a group's chunks are all active or all idle
    const int col0 = colc * kCK;
    if constexpr (SIGNS) {
      colc += col_step;
      if (colc >= a.cpr) colc -= a.cpr;
    }
    uint8_t* mine = cur + tt * kCPad;

    float v[kCK];
    float mn = 0.0f, mx = 0.0f;
    if (active) {
      uint4 sb = make_uint4(0, 0, 0, 0);
      if constexpr (SIGNS) sb = *reinterpret_cast<const uint4*>(s_bits + col0 / 32);
#pragma unroll
      for (int p = 0; p < 16; ++p) {
        const uint4 r = *reinterpret_cast<const uint4*>(mine + 16 * p);
        uint32_t w[4] = {r.x, r.y, r.z, r.w};
        if constexpr (SIGNS) {
          const uint4 m4 = sign_masks8(s_tab, sb, p);
          w[0] ^= m4.x;
          w[1] ^= m4.y;
          w[2] ^= m4.z;
          w[3] ^= m4.w;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) bf16_pair_stage1(w[i], v[8 * p + 2 * i], v[8 * p + 2 * i + 1]);
      }
      reg_fwht_from<kCK, 1, LOG_B>(v);
      float m0 = v[0], m1 = v[1], n0 = v[0], n1 = v[1];
#pragma unroll
      for (int i = 2; i < kCK; i += 4) {
        m0 = max3(m0, v[i], v[i + 1]);
        n0 = min3(n0, v[i], v[i + 1]);
        if (i + 3 < kCK) {
          m1 = max3(m1, v[i + 2], v[i + 3]);
          n1 = min3(n1, v[i + 2], v[i + 3]);
        }
      }
      mx = fmaxf(m0, m1);
      mn = fminf(n0, n1);
    }
    for (int b = 1; b < a.gpc; b <<= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, b));
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, b));
    }
    if (active) {
      const float lo = fminf(mn, 0.0f), hi = fmaxf(mx, 0.0f);
      const float range = hi - lo;
      const QInv q = make_qinv(range, float(QMAXU));
      const float los = q.tiny ? lo * kUp64 : lo;
      const int zp = int(fminf(fmaxf(rintf(-los * q.inv), 0.0f), float(QMAXU)));
      if (glead) {
        const int64_t g = ch / a.gpc;
        a.scales[g] = range * a.scale_mul;
        a.zp[g] = uint8_t(zp);
      }
      if (q.tiny) {
#pragma unroll
        for (int i = 0; i < kCK; i += 2) mul2(v[i], v[i + 1], kUp64);
      }
#pragma unroll
      for (int p = 0; p < 16; p += 2) {
        uint32_t c0[8], c1[8];
        asym_codes8(v + 8 * p, q.inv, zp, QMAXU, c0);
        asym_codes8(v + 8 * p + 8, q.inv, zp, QMAXU, c1);
        if constexpr (BITS == 8) {
          *reinterpret_cast<uint4*>(mine + 8 * p) =
              make_uint4(pack_i8x4(c0[0], c0[1], c0[2], c0[3]), pack_i8x4(c0[4], c0[5], c0[6], c0[7]),
                         pack_i8x4(c1[0], c1[1], c1[2], c1[3]), pack_i8x4(c1[4], c1[5], c1[6], c1[7]));
        } else {
          *reinterpret_cast<uint2*>(mine + 4 * p) = make_uint2(pack_i4x8(c0), pack_i4x8(c1));
        }
      }
    }
    T::sync();
    chunk_store<CB / 16, 32>(cur, nch, a.codes + c * CB, tt);
  }
  cp_async_wait<0>();
}

// Unsigned codes to floats minus the zero point, exactly: a code u placed in
// the low mantissa byte of 2^23 gives 2^23 + u; subtracting 2^23 + zp leaves
// u - zp.  Eight 4-bit codes of word w -> v[0..7].
__device__ __forceinline__ void u4x8_to_float(uint32_t w, float bias, float* v) {
  const uint32_t e = w & 0x0f0f0f0fu;         // elements 0, 2, 4, 6
  const uint32_t o = (w >> 4) & 0x0f0f0f0fu;  // elements 1, 3, 5, 7
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(__byte_perm(e, 0x4b000000u, 0x7440 + i));
    v[2 * i + 1] = __uint_as_float(__byte_perm(o, 0x4b000000u, 0x7440 + i));
  }
#pragma unroll
  for (int i = 0; i < 8; i += 2) add2(v[i], v[i + 1], bias);
}
// Four 8-bit codes of word w -> v[0..3].
__device__ __forceinline__ void u8x4_to_float(uint32_t w, float bias, float* v) {
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(__byte_perm(w, 0x4b000000u, 0x7440 + i));
#pragma unroll
  for (int i = 0; i < 4; i += 2) add2(v[i], v[i + 1], bias);
}

// Inverse: (codes - zero point) -> H_B on the integers (exact) -> * scale /
// sqrt(B) -> signs -> bf16 (or fp32).  The group's scale and zero point are
// read one slab ahead.
template <int LOG_B, int BITS, bool SIGNS, bool OUT_F32>
__global__ void __launch_bounds__(kCT, 3) dq_chunk_asym_kernel(ChunkAsymArgs a) {
  using T = Team<32>;
  constexpr int CB = BITS == 8 ? 128 : 64;
  extern __shared__ __align__(16) uint8_t smem[];
  uint4* s_tab = reinterpret_cast<uint4*>(smem + 2 * chunk_stage_bytes());
  uint32_t* s_bits = reinterpret_cast<uint32_t*>(smem + 2 * chunk_stage_bytes() + kSignTabBytes);
  const int tt = T::tid();
  if constexpr (SIGNS) {
    load_sign_tables(a.signs, a.dim, s_tab, s_bits);
    __syncthreads();
  }
  const int64_t nslabs = (a.nchunks + 31) / 32;
  int colc = SIGNS ? (int)((T::first() * 32 + tt) % a.cpr) : 0;
  const int col_step = SIGNS ? (int)((T::stride() * 32) % a.cpr) : 0;
  uint8_t* st0 = T::stage(smem, 0);
  uint8_t* st1 = T::stage(smem, 1);

  int64_t slab = T::first();
  float sc_next = 0.0f;
  int zp_next = 0;
  if (slab < nslabs) {
    const int64_t c0 = slab * 32;
    chunk_load<CB / 16, 32>(a.codes_in + c0 * CB, slab_count(c0, a.nchunks, 32), st0, tt);
    if (c0 + tt < a.nchunks) {
      sc_next = __ldg(a.scales_in + (c0 + tt) / a.gpc);
      zp_next = __ldg(a.zp_in + (c0 + tt) / a.gpc);
    }
  }
  cp_async_commit();
  for (int it = 0; slab < nslabs; ++it, slab += T::stride()) {
    uint8_t* cur = (it & 1) ? st1 : st0;
    const int64_t c = slab * 32;
    const float sc = sc_next;
    const int zp = zp_next;
    cp_async_wait<0>();
    T::sync();
    {
      const int64_t nx = slab + T::stride();
      if (nx < nslabs) {
        const int64_t cn = nx * 32;
        chunk_load<CB / 16, 32>(a.codes_in + cn * CB, slab_count(cn, a.nchunks, 32), (it & 1) ? st0 : st1, tt);
        if (cn + tt < a.nchunks) {
          sc_next = __ldg(a.scales_in + (cn + tt) / a.gpc);
          zp_next = __ldg(a.zp_in + (cn + tt) / a.gpc);
        }
      }
      cp_async_commit();
    }
    const int nch = slab_count(c, a.nchunks, 32);
    const int64_t ch = c + tt;
    const bool active = tt < nch;
    const int col0 = colc * kCK;
    if constexpr (SIGNS) {
      colc += col_step;
      if (colc >= a.cpr) colc -= a.cpr;
    }
    uint8_t* mine = cur + tt * kCPad;

    if (active) {
      const float bias = -(8388608.0f + float(zp));  // -(2^23 + zp)
      float v[kCK];
#pragma unroll
      for (int q4 = 0; q4 < CB / 16; ++q4) {
        const uint4 r = *reinterpret_cast<const uint4*>(mine + 16 * q4);
        if constexpr (BITS == 8) {
          u8x4_to_float(r.x, bias, v + 16 * q4);
          u8x4_to_float(r.y, bias, v + 16 * q4 + 4);
          u8x4_to_float(r.z, bias, v + 16 * q4 + 8);
          u8x4_to_float(r.w, bias, v + 16 * q4 + 12);
        } else {
          u4x8_to_float(r.x, bias, v + 32 * q4);
          u4x8_to_float(r.y, bias, v + 32 * q4 + 8);
          u4x8_to_float(r.z, bias, v + 32 * q4 + 16);
          u4x8_to_float(r.w, bias, v + 32 * q4 + 24);
        }
      }
      reg_fwht<kCK, LOG_B>(v);  // integers below 2^15 in magnitude: exact
      // scales below 2^-100: factor at 2^64 scale, then one exact 2^-64
      const bool tiny = sc < kTinyScale && sc != 0.0f;
      const float f = (tiny ? sc * kUp64 : sc) * a.rsqrt_b;
#pragma unroll
      for (int i = 0; i < kCK; i += 2) mul2(v[i], v[i + 1], f);
      if (tiny) {
#pragma unroll
        for (int i = 0; i < kCK; i += 2) mul2(v[i], v[i + 1], kDown64);
      }
      uint4 sb = make_uint4(0, 0, 0, 0);
      if constexpr (SIGNS) sb = *reinterpret_cast<const uint4*>(s_bits + col0 / 32);
      if constexpr (OUT_F32) {
        float* dst = a.rot + ch * kCK;
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          uint32_t o[8];
          uint4 m4 = make_uint4(0, 0, 0, 0);
          if constexpr (SIGNS) m4 = sign_masks8(s_tab, sb, p);
          const uint32_t mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t lo = __float_as_uint(v[8 * p + 2 * i]), hi = __float_as_uint(v[8 * p + 2 * i + 1]);
            if constexpr (SIGNS) {
              lo ^= mm[i] << 16;
              hi ^= mm[i] & 0x80000000u;
            }
            o[2 * i] = lo;
            o[2 * i + 1] = hi;
          }
          reinterpret_cast<uint4*>(dst + 8 * p)[0] = make_uint4(o[0], o[1], o[2], o[3]);
          reinterpret_cast<uint4*>(dst + 8 * p)[1] = make_uint4(o[4], o[5], o[6], o[7]);
        }
      } else {
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t r;
            asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(v[8 * p + 2 * i + 1]), "f"(v[8 * p + 2 * i]));
            o[i] = r;
          }
          if constexpr (SIGNS) {
            const uint4 m4 = sign_masks8(s_tab, sb, p);
            o[0] ^= m4.x;
            o[1] ^= m4.y;
            o[2] ^= m4.z;
            o[3] ^= m4.w;
          }
          *reinterpret_cast<uint4*>(mine + 16 * p) = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
    }
    if constexpr (!OUT_F32) {
      T::sync();
      chunk_store<16, 32>(cur, nch, reinterpret_cast<uint8_t*>(a.out_bf16) + c * 256, tt);
    }
  }
  cp_async_wait<0>();
}

}  // namespace hadq
