// Device helpers shared by the rotate+quantise and dequantise kernels.
//
// Conventions used in every kernel:
//  * A row of `dim` bfloat16 values is cut into Hadamard blocks of B = 2^LOG_B
//    elements.  The transform inside a block is the Sylvester H_B, which is the
//    tensor product of one 2-point butterfly per bit of the element index, so
//    the stages can run in any order and on any placement of the index bits
//    (registers, lanes, shared memory).  The 1/sqrt(B) normalisation is never
//    applied to the data: it cancels in the codes (q = y / (max|y|/qmax)) and
//    is folded into the stored scale and into the optional float output.
//  * Codes are produced with the float "magic number" rounding: for |t| < 2^22,
//    fmaf(v, inv, 1.5*2^23) rounds v*inv to the nearest integer, ties to even,
//    and its low bits hold that integer in two's complement.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace hadq {

constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23

// Below this group maximum qmax/max would overflow float; such groups take a
// rescaled path (all their values are then subnormal-sized).
constexpr float kTinyMax = 1.0e-36f;

// Dequantisation: blocks with a scale below kTinyScale (2^-100) are computed at
// 2^64 times their value and scaled back once, so the butterflies never run
// on subnormal numbers.  Both factors are exact powers of two.
constexpr float kTinyScale = 7.888609052210118e-31f;  // 2^-100
constexpr float kUp64 = 18446744073709551616.0f;      // 2^64
constexpr float kDown64 = 5.421010862427522e-20f;     // 2^-64

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Sign mask for the bf16 pair (s0 -> low half, s1 -> high half): XOR-ing it into
// the packed pair flips the sign of the elements whose sign entry is negative.
__device__ __forceinline__ uint32_t pair_sign_mask(int8_t s0, int8_t s1) {
  return (s0 < 0 ? 0x00008000u : 0u) | (s1 < 0 ? 0x80000000u : 0u);
}

// Round-to-nearest-even bf16 pair from two floats (finite inputs).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t a = __float_as_uint(lo), b = __float_as_uint(hi);
  a = (a + 0x7fffu + ((a >> 16) & 1u)) >> 16;
  b = (b + 0x7fffu + ((b >> 16) & 1u)) & 0xffff0000u;
  return a | b;
}

// One radix-2 butterfly.
__device__ __forceinline__ void bfly(float& a, float& b) {
  float s = a + b;
  b = a - b;
  a = s;
}

// Two butterflies on packed float pairs (a0,a1) and (b0,b1) with the sm_100
// paired-FP32 add/sub: (a0,a1) <- (a0+b0, a1+b1), (b0,b1) <- (a0-b0, a1-b1).
__device__ __forceinline__ void bfly2(float& a0, float& a1, float& b0, float& b1) {
  uint64_t A, Bv, S, D;
  asm("mov.b64 %0, {%1, %2};" : "=l"(A) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(Bv) : "f"(b0), "f"(b1));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(S) : "l"(A), "l"(Bv));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(D) : "l"(A), "l"(Bv));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(S));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(b0), "=f"(b1) : "l"(D));
}

// bf16 pair (x0 low half, x1 high half) -> first butterfly stage (x0 + x1,
// x0 - x1) with the mixed bf16/f32 add and subtract: x1 is widened by masking,
// x0 is read directly as a bf16 operand.  Same rounding as adding the widened
// values.
__device__ __forceinline__ void bf16_pair_stage1(uint32_t w, float& s, float& d) {
  const float x1 = __uint_as_float(w & 0xffff0000u);
  unsigned short x0 = (unsigned short)(w & 0xffffu);
  asm("add.rn.f32.bf16 %0, %1, %2;" : "=f"(s) : "h"(x0), "f"(x1));
  asm("sub.rn.f32.bf16 %0, %1, %2;" : "=f"(d) : "h"(x0), "f"(x1));
}

// In-register butterfly stage over register-index bit `h` (stride h) of an
// array of N floats.  Pairs whose partners are two apart or more use the
// paired add/sub on neighbouring registers.
template <int N, int H>
__device__ __forceinline__ void reg_stage(float (&v)[N]) {
  if constexpr (H == 1) {
#pragma unroll
    for (int i = 0; i < N; i += 2) bfly(v[i], v[i + 1]);
  } else {
#pragma unroll
    for (int i = 0; i < N; i += 2 * H) {
#pragma unroll
      for (int t = 0; t < H; t += 2) bfly2(v[i + t], v[i + t + 1], v[i + t + H], v[i + t + H + 1]);
    }
  }
}

// In-register stages over register-index bits [FIRST, LOG_N).
template <int N, int FIRST, int LOG_N>
__device__ __forceinline__ void reg_fwht_from(float (&v)[N]) {
  if constexpr (FIRST <= 0 && LOG_N >= 1) reg_stage<N, 1>(v);
  if constexpr (FIRST <= 1 && LOG_N >= 2) reg_stage<N, 2>(v);
  if constexpr (FIRST <= 2 && LOG_N >= 3) reg_stage<N, 4>(v);
  if constexpr (FIRST <= 3 && LOG_N >= 4) reg_stage<N, 8>(v);
  if constexpr (FIRST <= 4 && LOG_N >= 5) reg_stage<N, 16>(v);
  if constexpr (FIRST <= 5 && LOG_N >= 6) reg_stage<N, 32>(v);
  if constexpr (FIRST <= 6 && LOG_N >= 7) reg_stage<N, 64>(v);
}

// All in-register stages over register-index bits [0, LOG_N).
template <int N, int LOG_N>
__device__ __forceinline__ void reg_fwht(float (&v)[N]) {
  if constexpr (LOG_N >= 1) reg_stage<N, 1>(v);
  if constexpr (LOG_N >= 2) reg_stage<N, 2>(v);
  if constexpr (LOG_N >= 3) reg_stage<N, 4>(v);
  if constexpr (LOG_N >= 4) reg_stage<N, 8>(v);
  if constexpr (LOG_N >= 5) reg_stage<N, 16>(v);
  if constexpr (LOG_N >= 6) reg_stage<N, 32>(v);
  if constexpr (LOG_N >= 7) reg_stage<N, 64>(v);
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// The last butterfly stage (stride H, paired FP32) fused with the maximum of
// |y| over its outputs: max(|a + b|, |a - b|) = |a| + |b|, and the rounded
// value of whichever of a + b, a - b has that magnitude equals the rounded
// |a| + |b|, so the maximum is exact.  Returns the maximum over all N outputs.
template <int N, int H>
__device__ __forceinline__ float reg_stage_absmax(float (&v)[N]) {
  static_assert(H >= 2, "paired stage");
  float m0 = 0.0f, m1 = 0.0f;
#pragma unroll
  for (int i = 0; i < N; i += 2 * H) {
#pragma unroll
    for (int t = 0; t < H; t += 2) {
      const float s0 = fabsf(v[i + t]) + fabsf(v[i + t + H]);
      const float s1 = fabsf(v[i + t + 1]) + fabsf(v[i + t + H + 1]);
      if (((i + t) / 2) & 1) m1 = max3(m1, s0, s1); else m0 = max3(m0, s0, s1);
      bfly2(v[i + t], v[i + t + 1], v[i + t + H], v[i + t + H + 1]);
    }
  }
  return fmaxf(m0, m1);
}

// Butterfly stage across lanes: partner = lane ^ m.  The lane whose bit is set
// keeps (partner - own), the other keeps (own + partner).
template <int N>
__device__ __forceinline__ void lane_stage(float (&v)[N], int m, float sgn) {
#pragma unroll
  for (int i = 0; i < N; ++i) {
    float p = __shfl_xor_sync(0xffffffffu, v[i], m);
    v[i] = fmaf(v[i], sgn, p);
  }
}

// Code of t = v*inv as the low bits of a float's bit pattern (see header note).
__device__ __forceinline__ uint32_t magic_code(float v, float inv) {
  return __float_as_uint(fmaf(v, inv, kMagic));
}

// Codes of two values against one multiplier with the paired fused multiply-add.
__device__ __forceinline__ void magic_code2(float v0, float v1, float inv, uint32_t& c0, uint32_t& c1) {
  uint64_t V, I, M, R;
  asm("mov.b64 %0, {%1, %2};" : "=l"(V) : "f"(v0), "f"(v1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(I) : "f"(inv));
  asm("mov.b64 %0, {%1, %1};" : "=l"(M) : "f"(kMagic));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(R) : "l"(V), "l"(I), "l"(M));
  asm("mov.b64 {%0, %1}, %2;" : "=r"(c0), "=r"(c1) : "l"(R));
}

// Four codes (low byte of each) -> one word of int8 codes.
__device__ __forceinline__ uint32_t pack_i8x4(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3) {
  uint32_t lo = __byte_perm(c0, c1, 0x0040);
  uint32_t hi = __byte_perm(c2, c3, 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}

// Two words of int8 codes (elements 0..3 and 4..7, values in [-8, 7]) -> one
// word of int4 codes, element 0 in bits 0..3.
__device__ __forceinline__ uint32_t nibble_pack(uint32_t b03, uint32_t b47) {
  const uint32_t e = __byte_perm(b03, b47, 0x6420);  // elements 0, 2, 4, 6
  const uint32_t o = __byte_perm(b03, b47, 0x7531);  // elements 1, 3, 5, 7
  return (e & 0x0f0f0f0fu) | ((o << 4) & 0xf0f0f0f0u);
}

// Eight codes (low nibble of each) -> one word of int4 codes, element 0 in bits
// 0..3: bytes of the even elements, and of the odd elements shifted up a nibble.
__device__ __forceinline__ uint32_t pack_i4x8(const uint32_t (&c)[8]) {
  const uint32_t e = pack_i8x4(c[0], c[2], c[4], c[6]);
  const uint32_t o = pack_i8x4(c[1], c[3], c[5], c[7]);
  return (e & 0x0f0f0f0fu) | ((o << 4) & 0xf0f0f0f0u);
}

// Codes of eight values against one group maximum `m` (of the same, unnormalised
// values): t = v * qmax / m, rounded half to even.  Groups whose maximum is so
// small that qmax/m would overflow are rescaled by 2^64 first (exact).
__device__ __forceinline__ void quantize8(const float* v, float m, float qmax, uint32_t (&cc)[8]) {
  if (m >= kTinyMax) {
    const float inv = qmax / m;
#pragma unroll
    for (int k = 0; k < 8; ++k) cc[k] = magic_code(v[k], inv);
  } else {
    const float pre = 18446744073709551616.0f;  // 2^64
    const float inv = m > 0.0f ? qmax / (m * pre) : 0.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) cc[k] = magic_code(v[k] * pre, inv);
  }
}

// 16-byte asynchronous global -> shared copy (L2 only), with group commit/wait.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Bulk prefetch of a global range into L2 (no data comes back to the SM):
// 16-byte-aligned address, size a multiple of 16 bytes.  A warp issues it for
// the slab after the one it is staging, so that the staging copy hits L2.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Bulk asynchronous copy of `bytes` (a multiple of 16, both addresses 16-byte
// aligned) from shared to global memory by the copy engine, in the issuing
// thread's bulk group.  The writers of the shared source first make their
// stores visible to the copy engine with fence_async_shared() and a barrier.
__device__ __forceinline__ void bulk_store_s2g(void* gdst, const void* ssrc, uint32_t bytes) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(ssrc);
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(s), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// The issuing thread's bulk copies have read their shared-memory sources.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// The issuing thread's bulk copies are complete.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_shared() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Code multiplier of one group: inv = qmax / m, or, for a group maximum so
// small that this overflows, qmax / (m * 2^64) applied to v * 2^64.
struct QInv {
  float inv;
  bool tiny;
};
__device__ __forceinline__ QInv make_qinv(float m, float qmax) {
  if (m >= kTinyMax) return {qmax / m, false};
  return {m > 0.0f ? qmax / (m * 18446744073709551616.0f) : 0.0f, true};
}
__device__ __forceinline__ void quantize8q(const float* v, QInv q, uint32_t (&cc)[8]) {
  if (!q.tiny) {
#pragma unroll
    for (int k = 0; k < 8; ++k) cc[k] = magic_code(v[k], q.inv);
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) cc[k] = magic_code(v[k] * 18446744073709551616.0f, q.inv);
  }
}

// Paired FP32 ops on two registers with one shared operand.
__device__ __forceinline__ void add2(float& a, float& b, float c) {
  uint64_t X, C, R;
  asm("mov.b64 %0, {%1, %2};" : "=l"(X) : "f"(a), "f"(b));
  asm("mov.b64 %0, {%1, %1};" : "=l"(C) : "f"(c));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(R) : "l"(X), "l"(C));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(R));
}
__device__ __forceinline__ void mul2(float& a, float& b, float c) {
  uint64_t X, C, R;
  asm("mov.b64 %0, {%1, %2};" : "=l"(X) : "f"(a), "f"(b));
  asm("mov.b64 %0, {%1, %1};" : "=l"(C) : "f"(c));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(R) : "l"(X), "l"(C));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(R));
}

// Codes to floats without integer-to-float conversions: a biased code u
// (0 <= u < 256) placed in the low mantissa byte of 2^23 gives the float
// 2^23 + u exactly; subtracting 2^23 + bias recovers the signed code.
// Eight int4 codes of word w -> v[0..7].
__device__ __forceinline__ void i4x8_to_float(uint32_t w, float* v) {
  const uint32_t x = w ^ 0x88888888u;           // nibble n -> n + 8 in [0, 15]
  const uint32_t e = x & 0x0f0f0f0fu;           // elements 0, 2, 4, 6
  const uint32_t o = (x >> 4) & 0x0f0f0f0fu;    // elements 1, 3, 5, 7
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(__byte_perm(e, 0x4b000000u, 0x7440 + i));
    v[2 * i + 1] = __uint_as_float(__byte_perm(o, 0x4b000000u, 0x7440 + i));
  }
#pragma unroll
  for (int i = 0; i < 8; i += 2) add2(v[i], v[i + 1], -8388616.0f);  // -(2^23 + 8)
}
// Four int8 codes of word w -> v[0..3].
__device__ __forceinline__ void i8x4_to_float(uint32_t w, float* v) {
  const uint32_t x = w ^ 0x80808080u;           // n -> n + 128 in [0, 255]
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(__byte_perm(x, 0x4b000000u, 0x7440 + i));
#pragma unroll
  for (int i = 0; i < 4; i += 2) add2(v[i], v[i + 1], -8388736.0f);  // -(2^23 + 128)
}

// Sign-extended int4 nibble k of word w, as float.
__device__ __forceinline__ float i4_at(uint32_t w, int k) {
  return (float)(((int32_t)(w << (28 - 4 * k))) >> 28);
}

__device__ __forceinline__ float i8_at(uint32_t w, int k) {
  return (float)(((int32_t)(w << (24 - 8 * k))) >> 24);
}

}  // namespace hadq
