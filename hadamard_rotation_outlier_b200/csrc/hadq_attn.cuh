// Decode attention over the rotated, quantised KV cache.
//
// One new query token per head attends over a cache whose K and V rows were
// rotated by H_128 (after the optional sign flip) and stored as INT4 or INT8
// codes with one float32 scale per row or per group of 64 or 32 columns, i.e.
// the output of the rotate+quantise kernels at dim 128, block 128.  The maths ("Hartmann rotation, lightweight
// QAT, streaming attention", section 1; "QuaRot hands-on", sections 2.2-2.3):
//
//   q_rot = (q * s) H                     rotate the query like the keys
//   score_t = softmax_scale * q_rot . (kcode_t * kscale_t)   (= q . k_t)
//   p = softmax(score)                    over the cached tokens
//   o_rot = sum_t p_t * vcode_t * vscale_t
//   o = (o_rot H) * s                     one inverse rotation per output row
//
// Work split: a CTA (4 warps) serves one KV head, up to 4 of the query heads
// that share it, and one contiguous token range (split-K).  Each warp streams
// 16-token tiles through its own cp.async ring in shared memory and keeps an
// online softmax (running max m, sum l, output O) in registers.  The CTA
// merges its warps, writes one partial (m, l, O) per head to the workspace, and
// the last CTA of a head group merges all partials, applies H and the signs
// and writes the output.
//
// Tensor-core use (mma.sync; the contraction has only 4 query rows per KV
// head, far below the 64-row minimum of a tcgen05 tile, and its operands are
// born in registers):
//  * QK: m16n8k32 s8 x s8 -> s32.  B = key codes as int8: INT4 nibbles
//    shifted into the high half of a byte (16 * code, one shift and one mask
//    per 8 codes); INT8 codes as they are (two byte permutes per 8 codes
//    split even and odd dims).  A = the scaled rotated query as a 24-bit
//    fixed-point number cut into three signed 8-bit digits (rows = head x
//    digit).  The integer sums are exact; score = (d0 + 2^8 d1 + 2^16 d2) *
//    2^-E * kscale (/ 16 for INT4).
//  * PV: m16n8k16 bf16 x bf16 -> f32.  B = value codes as exact bf16 values
//    (INT4: the nibble placed in a bf16 mantissa, then 136 subtracted; INT8:
//    see int8x2_to_bf16x2).  A = p * vscale cut into three bf16 parts hi +
//    mid + lo (rows = head x part), which together carry the full float32
//    value.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "hadq_common.cuh"

namespace hadq {

constexpr int kAttnDim = 128;
constexpr int kAttnWarps = 4;
constexpr int kAttnThreads = 32 * kAttnWarps;
constexpr int kAttnHeads = 4;                                   // query heads per CTA
constexpr int kAttnTile = 16;                                   // tokens per tile
constexpr int kAttnStages = 4;                                  // ring depth per warp, INT4 caches
constexpr int kAttnStages8 = 3;                                 // INT8 caches (twice the bytes per tile)
// Per-stage layout of a cache of BITS-bit codes: 16 K rows at pitch KP, 16 V
// rows at pitch VROW (pitches padded so that the fragment reads are
// conflict-free), then [16 tokens][NG] K scales and as many V scales (NG =
// 128 / G scale groups per row).  KROW = bytes of codes per token in global
// memory.
template <int BITS>
struct AttnRows {
  static constexpr int KROW = 16 * BITS;                        // 64 or 128
  static constexpr int KP = BITS == 8 ? KROW + 16 : KROW;
  static constexpr int VROW = KROW + 16;
  static constexpr int STV = kAttnTile * KP;
  static constexpr int STS = STV + kAttnTile * VROW;
};
__host__ __device__ constexpr int attn_stage_bytes(int ng, int bits = 4) {
  return (bits == 8 ? AttnRows<8>::STS : AttnRows<4>::STS) + 2 * kAttnTile * 4 * ng;
}
constexpr int kAttnCombPitch = kAttnDim + 4;                    // floats per head in the CTA merge
constexpr int kAttnMaxSplits = 256;
constexpr size_t kAttnStaticScratchBytes = size_t(16) << 20;  // scratch of the allocation-free entry
constexpr float kAttnSlack = 8.0f;  // log2 units the running max may trail the true max

struct AttnArgs {
  const uint16_t* q;         // [batch, nqh, 128] bf16
  const uint8_t* k_codes;    // [batch, nkv, stride, 64]
  const float* k_scales;     // [batch, nkv, stride]
  const uint8_t* v_codes;
  const float* v_scales;
  const int8_t* signs;       // [128] or NULL
  void* out;                 // [batch, nqh, 128] bf16 or f32
  unsigned* counters;        // [groups]
  float* part_ml;            // [groups][splits][4][2]  (m, l)
  float* part_o;             // [groups][splits][4][128] (permuted order, see below)
  int64_t tokens, stride, chunk;
  int nqh, nkv, g, hgroups, splits;
  float qmul;                // softmax_scale * log2(e) / sqrt(128)
  float inv_sqrt_dim;        // 1 / sqrt(128)
  int out_f32;
  uint32_t vmask, vmagic;    // INT4: 0x000F000F and 0x43084308 (see int4x2_to_bf16x2);
                             // INT8: 0x007F007F and 0x43004300 (see int8x2_to_bf16x2)
  uint32_t vsign;            // INT8: 0x00800080
};

template <int STAGES, int NG, int BITS>
struct __align__(16) AttnSmem {
  union {
    uint8_t stage[kAttnWarps][STAGES][attn_stage_bytes(NG, BITS)];
    float comb[kAttnWarps][kAttnHeads][kAttnCombPitch];
  } u;
  int8_t qd[4][kAttnHeads][kAttnDim];  // query digits [digit][head][dim]; digit 3 stays 0
  float qscale[kAttnHeads];
  float m[kAttnWarps][kAttnHeads];
  float l[kAttnWarps][kAttnHeads];
  int last;
};

__device__ __forceinline__ void mma_s8_16832(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// cp.async of 16 (or 4) bytes to a shared-memory address.  The _zfill forms
// read nothing when valid == false and fill the destination with zeros (the
// source must still be a mapped address).
__device__ __forceinline__ void cp_async16(uint32_t smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async16_zfill(uint32_t smem, const void* gmem, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem), "l"(gmem), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async4_zfill(uint32_t smem, const void* gmem, bool valid) {
  const int n = valid ? 4 : 0;
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem), "l"(gmem), "r"(n) : "memory");
}

// Two INT4 codes (nibbles at bits 0-3 and 16-19 of x) -> bf16x2 holding the
// codes exactly: the nibble with its sign bit flipped is c + 8; placed in the
// mantissa of 128.0 it reads 136 + c, and subtracting 136 leaves c.  The mask
// (0x000F000F) and the bit pattern of 136.0 twice (0x43084308) arrive as
// kernel arguments, so that one three-input logic operation does the masking,
// the flip and the exponent at once.
__device__ __forceinline__ uint32_t int4x2_to_bf16x2(uint32_t x, uint32_t mask, uint32_t magic) {
  uint32_t t, r;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(t) : "r"(x), "r"(mask), "r"(magic));  // (x & mask) ^ magic
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(t), "r"(magic));
  return r;
}

// Two INT8 codes (bytes at bits 0-7 and 16-23 of x) -> bf16x2 holding the
// codes exactly.  With the low seven bits of a code c in the mantissa of
// 128.0, the half reads 128 + (c mod 128); the code's sign bit, placed in the
// lowest exponent bit of 128.0, gives 128 (c >= 0) or 256 (c < 0), and the
// difference of the two is c.  Both inputs are one three-input logic
// operation each (masks and patterns arrive as kernel arguments).
__device__ __forceinline__ uint32_t int8x2_to_bf16x2(uint32_t x, uint32_t low7, uint32_t magic, uint32_t sign) {
  uint32_t h, m, r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(h) : "r"(x), "r"(low7), "r"(magic));  // (x & low7) | magic
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(m) : "r"(x), "r"(sign), "r"(magic));  // (x & sign) | magic
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(h), "r"(m));
  return r;
}

// 2^x for the softmax weights (the ISA approximation; results below 2^-126,
// i.e. weights below 2^-126 of the running maximum, flush to zero).
__device__ __forceinline__ float exp2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// bf16x2 of (lo, hi), round to nearest even.
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Cut the float pair (x0, x1) into bf16 pairs hi + mid + lo whose sum carries
// every bit of each float: each part is the bf16 rounding of what the
// previous parts left, and those remainders are exact float differences.
__device__ __forceinline__ void split3_bf16(float x0, float x1, uint32_t& hi, uint32_t& mid, uint32_t& lo) {
  hi = cvt_bf16x2(x0, x1);
  const float r0 = x0 - __uint_as_float(hi << 16);
  const float r1 = x1 - __uint_as_float(hi & 0xffff0000u);
  mid = cvt_bf16x2(r0, r1);
  const float s0 = r0 - __uint_as_float(mid << 16);
  const float s1 = r1 - __uint_as_float(mid & 0xffff0000u);
  lo = cvt_bf16x2(s0, s1);
}

// 8 INT4 codes of one word -> the two int8x4 registers of an s8 MMA operand:
// even elements (low nibbles) and odd elements (high nibbles), each as 16*code.
__device__ __forceinline__ void int4x8_to_s8x16(uint32_t w, uint32_t& even, uint32_t& odd) {
  even = (w << 4) & 0xF0F0F0F0u;
  odd = w & 0xF0F0F0F0u;
}

// STAGES: depth of each warp's cp.async ring (tiles in flight + 1).
// NG: scale groups per cached row (128 / G: 1, 2 or 4).  With NG = 1 a k-step
// of the score MMA spans the four 32-dim quarters of the row; with NG > 1 it
// spans one quarter, so that each quarter (a group of 32, or half a group of
// 64) has its own integer accumulator and is weighted by its own key scale,
// and the value codes are taken four dims per quarter so that every n8 tile
// of the P.V product lies inside one group (the A operand p * vscale is cut
// once per group).
template <int STAGES, int NG, int BITS>
__global__ void __launch_bounds__(kAttnThreads, 3) kv_decode_attn_kernel(const AttnArgs a) {
  static_assert(NG == 1 || NG == 2 || NG == 4, "groups of 128, 64 or 32 columns");
  static_assert(BITS == 4 || BITS == 8, "INT4 or INT8 codes");
  using RW = AttnRows<BITS>;
  constexpr int KROW = RW::KROW, KP = RW::KP, VROW = RW::VROW, STV = RW::STV, STS = RW::STS;
  constexpr int SB = attn_stage_bytes(NG, BITS);
  extern __shared__ __align__(16) uint8_t attn_smem_raw[];
  AttnSmem<STAGES, NG, BITS>& sm = *reinterpret_cast<AttnSmem<STAGES, NG, BITS>*>(attn_smem_raw);
  const int tid = threadIdx.x;
  const int w = tid >> 5;
  const int lane = tid & 31;
  const int g = lane >> 2;  // MMA row group
  const int j = lane & 3;   // thread in group

  const int grp = blockIdx.y;
  const int split = blockIdx.x;
  const int bidx = grp / (a.nkv * a.hgroups);
  const int rem = grp - bidx * a.nkv * a.hgroups;
  const int kvh = rem / a.hgroups;
  const int hg = rem - kvh * a.hgroups;
  const int head0 = kvh * a.g + hg * kAttnHeads;  // first query head of this CTA
  const int hn = min(kAttnHeads, a.g - hg * kAttnHeads);
  const int64_t row0 = (int64_t(bidx) * a.nkv + kvh) * a.stride;

  // ---- query: rotate, scale, cut into digits (warp w handles head w) ----
  {
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    if (w < hn) {
      const uint2 raw =
          *reinterpret_cast<const uint2*>(a.q + (int64_t(bidx) * a.nqh + head0 + w) * kAttnDim + 4 * lane);
      x[0] = bf16lo(raw.x);
      x[1] = bf16hi(raw.x);
      x[2] = bf16lo(raw.y);
      x[3] = bf16hi(raw.y);
      if (a.signs) {
        const uint32_t sg = *reinterpret_cast<const uint32_t*>(a.signs + 4 * lane);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if ((sg >> (8 * i + 7)) & 1u) x[i] = -x[i];
      }
    }
    // H_128: index bits 0-1 in registers, bits 2-6 on lane bits 0-4.
    bfly(x[0], x[1]);
    bfly(x[2], x[3]);
    bfly(x[0], x[2]);
    bfly(x[1], x[3]);
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const bool upper = (lane & m) != 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float o = __shfl_xor_sync(0xffffffffu, x[i], m);
        x[i] = upper ? o - x[i] : x[i] + o;
      }
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[i] *= a.qmul;
      amax = fmaxf(amax, fabsf(x[i]));
    }
#pragma unroll
    for (int m = 16; m; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    // amax < 2^E' with E' = biased exponent - 126; the fixed-point value is
    // x * 2^(22 - E'), so |qf| <= 2^22 and the top digit stays within +-65.
    // A query below 2^-100 in every scaled entry is taken as zero.
    const int E = int((__float_as_uint(amax) >> 23) & 0xffu);
    const bool zero = E < 27;
    const float up = zero ? 0.f : __uint_as_float(uint32_t(148 - E + 127) << 23);
    uint32_t d0 = 0, d1 = 0, d2 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int qf = __float2int_rn(x[i] * up);
      const int e0 = (qf << 24) >> 24;
      const int r1 = (qf - e0) >> 8;
      const int e1 = (r1 << 24) >> 24;
      const int e2 = (r1 - e1) >> 8;
      d0 |= uint32_t(e0 & 0xff) << (8 * i);
      d1 |= uint32_t(e1 & 0xff) << (8 * i);
      d2 |= uint32_t(e2 & 0xff) << (8 * i);
    }
    *reinterpret_cast<uint32_t*>(&sm.qd[0][w][4 * lane]) = d0;
    *reinterpret_cast<uint32_t*>(&sm.qd[1][w][4 * lane]) = d1;
    *reinterpret_cast<uint32_t*>(&sm.qd[2][w][4 * lane]) = d2;
    *reinterpret_cast<uint32_t*>(&sm.qd[3][w][4 * lane]) = 0u;
    // 2^(E' - 22): undo the fixed point (and / 16: the 16 * code of INT4 keys).
    if (lane == 0) sm.qscale[w] = zero ? 0.f : __uint_as_float(uint32_t(BITS == 4 ? E - 25 : E - 21) << 23);
  }
  __syncthreads();

  // A operands of the QK product for k-step s: lane (g, j) holds rows g and
  // g+8 (head g & 3, digits g >> 2 and (g >> 2) + 2) at the dims
  // d0 + {0,2,4,6} (a0, a1) and d0 + {1,3,5,7} (a2, a3), d0 = 32j + 8s (one
  // scale group) or 32s + 8j (NG > 1), the same dims the key operand of that
  // lane carries.
  uint32_t qa[4][4];
  const int hh = g & 3;
  {
    const int dr0 = g >> 2, dr1 = (g >> 2) + 2;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int d0 = NG == 1 ? 32 * j + 8 * s : 32 * s + 8 * j;  // this lane's 8 dims of k-step s
      const uint2 r0 = *reinterpret_cast<const uint2*>(&sm.qd[dr0][hh][d0]);
      const uint2 r1 = *reinterpret_cast<const uint2*>(&sm.qd[dr1][hh][d0]);
      qa[s][0] = __byte_perm(r0.x, r0.y, 0x6420);
      qa[s][1] = __byte_perm(r1.x, r1.y, 0x6420);
      qa[s][2] = __byte_perm(r0.x, r0.y, 0x7531);
      qa[s][3] = __byte_perm(r1.x, r1.y, 0x7531);
    }
  }
  const float qs = sm.qscale[hh];
  const uint32_t vmask = a.vmask, vmagic = a.vmagic, vsign = a.vsign;
  // Digit weights of the two rows this lane holds: rows g (digit g>>2) and
  // g+8 (digit (g>>2)+2; digit 3 is the zero row).
  const float wl = g < 4 ? 1.f : 256.f;
  const float wh = g < 4 ? 65536.f : 0.f;
  const bool low = g < 4;
  const int own = low ? 2 * j : 2 * j + 8;  // first of the two tokens this lane finishes

  // ---- token range of this CTA and the warp's tiles ----
  const int64_t t_begin = int64_t(split) * a.chunk;
  const int64_t t_end = min(a.tokens, t_begin + a.chunk);
  const int n_tok = t_begin < t_end ? int(t_end - t_begin) : 0;  // tokens of this CTA (< 2^31)
  const int ntiles = (n_tok + kAttnTile - 1) / kAttnTile;
  const int nw = ntiles > w ? (ntiles - w + kAttnWarps - 1) / kAttnWarps : 0;

  const uint8_t* kc = a.k_codes + row0 * KROW;
  const uint8_t* vc = a.v_codes + row0 * KROW;
  const float* ksc = a.k_scales + row0 * NG;  // [batch, nkv, stride, NG]
  const float* vsc = a.v_scales + row0 * NG;

  // Copy pattern of one tile (per array, 16 tokens x CPR chunks of 16 bytes):
  // lane covers chunk lane % CPR of tokens lane / CPR + TPP p (p < 16 / TPP);
  // the scale copy takes one float per lane (K scales in lanes 0-15, V scales
  // in 16-31).
  constexpr int CPR = KROW / 16, TPP = 32 / CPR, NPASS = kAttnTile / TPP;
  const int ctok = lane / CPR, cpart = lane % CPR;
  const uint32_t s_ring = static_cast<uint32_t>(__cvta_generic_to_shared(&sm.u.stage[w][0][0]));
  const uint32_t d_k = ctok * KP + cpart * 16;
  const uint32_t d_v = STV + ctok * VROW + cpart * 16;
  const uint32_t d_s = STS + 4 * lane;
  const int64_t lane_tok = t_begin + int64_t(w) * kAttnTile + ctok;  // token of the first chunk, tile 0
  const uint8_t* g_k = kc + lane_tok * KROW + cpart * 16;
  const uint8_t* g_v = vc + lane_tok * KROW + cpart * 16;
  const float* g_s = (lane < 16 ? ksc : vsc) + t_begin + int64_t(w) * kAttnTile + (lane & 15);
  // NG > 1: scales [token][NG] per array; lane p < 4 NG copies K piece p,
  // lanes 4 NG .. 8 NG - 1 the V pieces (16 bytes = 4 / NG tokens each)
  const int sg_piece = lane % (4 * NG);
  const int sg_tok = sg_piece * 4 / NG;  // first token of this lane's piece in the tile
  const uint32_t d_sg = STS + (lane < 4 * NG ? 0u : uint32_t(kAttnTile * 4 * NG)) + 16u * uint32_t(sg_piece);
  const float* g_sg = (lane < 4 * NG ? ksc : vsc) + (t_begin + int64_t(w) * kAttnTile) * NG + 4 * sg_piece;
  constexpr int64_t kStepTok = int64_t(kAttnWarps) * kAttnTile;  // tokens between a warp's tiles

  auto issue = [&](int k) {
    const uint32_t st = s_ring + uint32_t(k % STAGES) * SB;
    const int64_t adv = int64_t(k) * kStepTok;
    const int r0 = (w + kAttnWarps * k) * kAttnTile;  // first token of the tile, from t_begin
    if (r0 + kAttnTile <= n_tok) {
#pragma unroll
      for (int p = 0; p < NPASS; ++p) {
        cp_async16(st + d_k + TPP * p * KP, g_k + (adv + TPP * p) * KROW);
        cp_async16(st + d_v + TPP * p * VROW, g_v + (adv + TPP * p) * KROW);
      }
      if constexpr (NG == 1) {
        cp_async4(st + d_s, g_s + adv);
      } else if (lane < 8 * NG) {  // 4 NG pieces of 16 bytes of K scales, then as many of V
        cp_async16(st + d_sg, g_sg + adv * NG);
      }
    } else {  // ragged last tile: rows past t_end are zero-filled, never read
      // (their source address is replaced by the first row of the head).
      const bool vs = r0 + (lane & 15) < n_tok;
      const float* s0 = lane < 16 ? ksc : vsc;
#pragma unroll
      for (int p = 0; p < NPASS; ++p) {
        const bool vp = r0 + ctok + TPP * p < n_tok;
        cp_async16_zfill(st + d_k + TPP * p * KP, vp ? g_k + (adv + TPP * p) * KROW : kc, vp);
        cp_async16_zfill(st + d_v + TPP * p * VROW, vp ? g_v + (adv + TPP * p) * KROW : vc, vp);
      }
      if constexpr (NG == 1) {
        cp_async4_zfill(st + d_s, vs ? g_s + adv : s0, vs);
      } else if (lane < 8 * NG) {  // the piece's tokens past t_end read nothing (zero fill)
        const int left = (n_tok - r0 - sg_tok) * NG * 4;  // bytes of this piece inside the range
        const int nb = left <= 0 ? 0 : left >= 16 ? 16 : left;
        const float* s0g = (lane < 4 * NG) ? ksc : vsc;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(st + d_sg),
                     "l"(nb > 0 ? g_sg + adv * NG : s0g), "r"(nb) : "memory");
      }
    }
  };

  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;

#pragma unroll
  for (int k = 0; k < STAGES - 1; ++k) {
    if (k < nw) issue(k);
    cp_async_commit();
  }

  for (int k = 0; k < nw; ++k) {
    if (k + STAGES - 1 < nw) issue(k + STAGES - 1);
    cp_async_commit();
    cp_async_wait<STAGES - 1>();
    __syncwarp();

    const uint8_t* st = sm.u.stage[w][k % STAGES];
    const int r0 = (w + kAttnWarps * k) * kAttnTile;

    // --- scores: S^T[head x digit, token] = Qdigits . (16 * kcode), one
    // integer accumulator per scale group (k-steps s with s * NG / 4 = q) ---
    int c0[NG][4], c1[NG][4];
#pragma unroll
    for (int q = 0; q < NG; ++q)
#pragma unroll
      for (int i = 0; i < 4; ++i) c0[q][i] = c1[q][i] = 0;
    if constexpr (BITS == 4) {
      uint32_t kw0[4], kw1[4];
      if constexpr (NG == 1) {
        const uint4 k0 = *reinterpret_cast<const uint4*>(st + g * KP + 16 * j);
        const uint4 k1 = *reinterpret_cast<const uint4*>(st + (g + 8) * KP + 16 * j);
        kw0[0] = k0.x; kw0[1] = k0.y; kw0[2] = k0.z; kw0[3] = k0.w;
        kw1[0] = k1.x; kw1[1] = k1.y; kw1[2] = k1.z; kw1[3] = k1.w;
      } else {  // dims 32 s + 8 j .. + 7 = bytes 16 s + 4 j .. + 3 of a row
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          kw0[s] = *reinterpret_cast<const uint32_t*>(st + g * KP + 16 * s + 4 * j);
          kw1[s] = *reinterpret_cast<const uint32_t*>(st + (g + 8) * KP + 16 * s + 4 * j);
        }
      }
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        uint32_t e, od;
        int4x8_to_s8x16(kw0[s], e, od);
        mma_s8_16832(c0[s * NG / 4], qa[s], e, od);
        int4x8_to_s8x16(kw1[s], e, od);
        mma_s8_16832(c1[s * NG / 4], qa[s], e, od);
      }
    } else {
      // the lane's 8 dims of k-step s are 8 consecutive bytes: even dims
      // (a0, a1 of the query) and odd dims (a2, a3) by two byte permutes
      uint2 kw0[4], kw1[4];
      if constexpr (NG == 1) {  // dims 32 j + 8 s: bytes 32 j .. 32 j + 31
        const uint4 k0a = *reinterpret_cast<const uint4*>(st + g * KP + 32 * j);
        const uint4 k0b = *reinterpret_cast<const uint4*>(st + g * KP + 32 * j + 16);
        const uint4 k1a = *reinterpret_cast<const uint4*>(st + (g + 8) * KP + 32 * j);
        const uint4 k1b = *reinterpret_cast<const uint4*>(st + (g + 8) * KP + 32 * j + 16);
        kw0[0] = make_uint2(k0a.x, k0a.y); kw0[1] = make_uint2(k0a.z, k0a.w);
        kw0[2] = make_uint2(k0b.x, k0b.y); kw0[3] = make_uint2(k0b.z, k0b.w);
        kw1[0] = make_uint2(k1a.x, k1a.y); kw1[1] = make_uint2(k1a.z, k1a.w);
        kw1[2] = make_uint2(k1b.x, k1b.y); kw1[3] = make_uint2(k1b.z, k1b.w);
      } else {  // dims 32 s + 8 j .. + 7
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          kw0[s] = *reinterpret_cast<const uint2*>(st + g * KP + 32 * s + 8 * j);
          kw1[s] = *reinterpret_cast<const uint2*>(st + (g + 8) * KP + 32 * s + 8 * j);
        }
      }
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        mma_s8_16832(c0[s * NG / 4], qa[s], __byte_perm(kw0[s].x, kw0[s].y, 0x6420),
                     __byte_perm(kw0[s].x, kw0[s].y, 0x7531));
        mma_s8_16832(c1[s * NG / 4], qa[s], __byte_perm(kw1[s].x, kw1[s].y, 0x6420),
                     __byte_perm(kw1[s].x, kw1[s].y, 0x7531));
      }
    }
    // Scores.  Every lane holds digit partials of tokens 2j, 2j+1, 2j+8 and
    // 2j+9 for head g & 3; the lane pair (g, g ^ 4) shares that head, and the
    // low lane (g < 4) finishes tokens 2j, 2j+1 while the high lane finishes
    // 2j+8, 2j+9 (`own`), each adding the partner's partials.
    const float* sc = reinterpret_cast<const float*>(st + STS);  // [16][NG] K, then [16][NG] V
    float sv0 = 0.f, sv1 = 0.f;
#pragma unroll
    for (int q = 0; q < NG; ++q) {
      const float pl0 = fmaf(float(c0[q][2]), wh, float(c0[q][0]) * wl);
      const float pl1 = fmaf(float(c0[q][3]), wh, float(c0[q][1]) * wl);
      const float pl2 = fmaf(float(c1[q][2]), wh, float(c1[q][0]) * wl);
      const float pl3 = fmaf(float(c1[q][3]), wh, float(c1[q][1]) * wl);
      const float x0 = __shfl_xor_sync(0xffffffffu, low ? pl2 : pl0, 16);
      const float x1 = __shfl_xor_sync(0xffffffffu, low ? pl3 : pl1, 16);
      const float k0s = sc[own * NG + q], k1s = sc[(own + 1) * NG + q];
      if constexpr (NG == 1) {
        sv0 = ((low ? pl0 : pl2) + x0) * (qs * k0s);
        sv1 = ((low ? pl1 : pl3) + x1) * (qs * k1s);
      } else {
        sv0 = fmaf((low ? pl0 : pl2) + x0, k0s, sv0);
        sv1 = fmaf((low ? pl1 : pl3) + x1, k1s, sv1);
      }
    }
    if constexpr (NG > 1) {
      sv0 *= qs;
      sv1 *= qs;
    }
    if (r0 + kAttnTile > n_tok) {  // ragged last tile (warp-uniform): mask the missing tokens
      if (r0 + own >= n_tok) sv0 = -INFINITY;
      if (r0 + own + 1 >= n_tok) sv1 = -INFINITY;
    }
    float mtile = fmaxf(sv0, sv1);
    mtile = fmaxf(mtile, __shfl_xor_sync(0xffffffffu, mtile, 1));
    mtile = fmaxf(mtile, __shfl_xor_sync(0xffffffffu, mtile, 2));
    mtile = fmaxf(mtile, __shfl_xor_sync(0xffffffffu, mtile, 16));

    // --- online softmax (base 2); the running max is raised only when the
    // tile max exceeds it by more than kAttnSlack, so p stays <= 2^8 ---
    const bool need = mtile > m_run + kAttnSlack;
    if (__any_sync(0xffffffffu, need)) {
      const float alpha = need ? exp2f(m_run - mtile) : 1.f;
      if (need) m_run = mtile;
      l_run *= alpha;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        mul2(o[i][0], o[i][1], alpha);
        mul2(o[i][2], o[i][3], alpha);
      }
    }
    const float p0 = exp2_ftz(sv0 - m_run);
    const float p1 = exp2_ftz(sv1 - m_run);
    l_run += p0 + p1;

    // --- A operand of PV: rows (head, part), part 0/1/2 = hi/mid/lo of
    // p * vscale, part 3 zero.  Lanes g < 4 hold parts 0 and 2, g >= 4 part 1;
    // each lane cut its own two tokens and takes the partner's parts it needs.
    // (NG > 1: one such operand per scale group, with that group's vscale.)
    uint32_t pa[NG][4];
    const float* vsc_s = sc + kAttnTile * NG;
#pragma unroll
    for (int q = 0; q < NG; ++q) {
      uint32_t hi, mid, lo;
      split3_bf16(p0 * vsc_s[own * NG + q], p1 * vsc_s[(own + 1) * NG + q], hi, mid, lo);
      const uint32_t r1 = __shfl_xor_sync(0xffffffffu, low ? mid : hi, 16);
      const uint32_t r2 = __shfl_xor_sync(0xffffffffu, lo, 16);
      pa[q][0] = low ? hi : r1;   // row g, tokens 2j, 2j+1
      pa[q][1] = low ? lo : 0u;   // row g + 8, tokens 2j, 2j+1
      pa[q][2] = low ? r1 : mid;  // row g, tokens 2j+8, 2j+9
      pa[q][3] = low ? r2 : 0u;   // row g + 8, tokens 2j+8, 2j+9
    }

    // --- PV: O[(head, part), dim] += P . V ---
    if constexpr (BITS == 8 && NG == 1) {
      // lane (g, j) feeds the value codes of dims 16g + i (n8 tile i) for
      // tokens 2j, 2j+1 / 2j+8, 2j+9: byte i of each token's 16 bytes
      const uint8_t* svp = st + STV + 16 * g;
      const uint4 va = *reinterpret_cast<const uint4*>(svp + (2 * j) * VROW);
      const uint4 vb = *reinterpret_cast<const uint4*>(svp + (2 * j + 1) * VROW);
      const uint4 vcx = *reinterpret_cast<const uint4*>(svp + (2 * j + 8) * VROW);
      const uint4 vd = *reinterpret_cast<const uint4*>(svp + (2 * j + 9) * VROW);
      const uint32_t wa[4] = {va.x, va.y, va.z, va.w}, wb[4] = {vb.x, vb.y, vb.z, vb.w};
      const uint32_t wc[4] = {vcx.x, vcx.y, vcx.z, vcx.w}, wd[4] = {vd.x, vd.y, vd.z, vd.w};
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint32_t sel = uint32_t((i & 3) | ((4 + (i & 3)) << 8));  // byte i%4 of each word to bytes 0, 2
        mma_bf16_16816(o[i], pa[0], int8x2_to_bf16x2(__byte_perm(wa[i >> 2], wb[i >> 2], sel), vmask, vmagic, vsign),
                       int8x2_to_bf16x2(__byte_perm(wc[i >> 2], wd[i >> 2], sel), vmask, vmagic, vsign));
      }
    } else if constexpr (BITS == 8) {
      // n8 tile i = 4 qt + r: lane (g, j) feeds dim 32 qt + 8 (g >> 1) + 2 r +
      // (g & 1), byte (g & 1) + 2 r of the 8 bytes at 32 qt + 8 (g >> 1)
      const uint8_t* svp = st + STV + 8 * (g >> 1);
      const uint32_t bsel = uint32_t(g & 1);
#pragma unroll
      for (int qt = 0; qt < 4; ++qt) {
        const uint2 wa = *reinterpret_cast<const uint2*>(svp + (2 * j) * VROW + 32 * qt);
        const uint2 wb = *reinterpret_cast<const uint2*>(svp + (2 * j + 1) * VROW + 32 * qt);
        const uint2 wc = *reinterpret_cast<const uint2*>(svp + (2 * j + 8) * VROW + 32 * qt);
        const uint2 wd = *reinterpret_cast<const uint2*>(svp + (2 * j + 9) * VROW + 32 * qt);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const uint32_t b = bsel + 2 * (r & 1);  // byte within the word r >> 1
          const uint32_t sel = b | ((4 + b) << 8);
          const uint32_t xab = __byte_perm(r < 2 ? wa.x : wa.y, r < 2 ? wb.x : wb.y, sel);
          const uint32_t xcd = __byte_perm(r < 2 ? wc.x : wc.y, r < 2 ? wd.x : wd.y, sel);
          mma_bf16_16816(o[4 * qt + r], pa[qt * NG / 4], int8x2_to_bf16x2(xab, vmask, vmagic, vsign),
                         int8x2_to_bf16x2(xcd, vmask, vmagic, vsign));
        }
      }
    } else if constexpr (NG == 1) {
      // lane (g, j) feeds the value codes of dims 16g + i (n8 tile i) for
      // tokens 2j, 2j+1 / 2j+8, 2j+9
      const uint8_t* svp = st + STV + 8 * g;
      const uint2 va = *reinterpret_cast<const uint2*>(svp + (2 * j) * VROW);
      const uint2 vb = *reinterpret_cast<const uint2*>(svp + (2 * j + 1) * VROW);
      const uint2 vcx = *reinterpret_cast<const uint2*>(svp + (2 * j + 8) * VROW);
      const uint2 vd = *reinterpret_cast<const uint2*>(svp + (2 * j + 9) * VROW);
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const uint32_t sel = (h & 1) ? 0x7632u : 0x5410u;
        const uint32_t xab = __byte_perm(h < 2 ? va.x : va.y, h < 2 ? vb.x : vb.y, sel);
        const uint32_t xcd = __byte_perm(h < 2 ? vcx.x : vcx.y, h < 2 ? vd.x : vd.y, sel);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          mma_bf16_16816(o[4 * h + e], pa[0], int4x2_to_bf16x2(xab >> (4 * e), vmask, vmagic),
                         int4x2_to_bf16x2(xcd >> (4 * e), vmask, vmagic));
      }
    } else {
      // n8 tile i = 4 qt + r (quarter qt of the row, group qt * NG / 4): lane
      // (g, j) feeds dim 32 qt + 8 (g >> 1) + 2 r + (g & 1), i.e. nibble g & 1
      // of byte r of the word at byte 16 qt + 4 (g >> 1) of the token's row
      const uint8_t* svp = st + STV + 4 * (g >> 1);
      const int nsh = 4 * (g & 1);
#pragma unroll
      for (int qt = 0; qt < 4; ++qt) {
        const uint32_t wa = *reinterpret_cast<const uint32_t*>(svp + (2 * j) * VROW + 16 * qt);
        const uint32_t wb = *reinterpret_cast<const uint32_t*>(svp + (2 * j + 1) * VROW + 16 * qt);
        const uint32_t wc = *reinterpret_cast<const uint32_t*>(svp + (2 * j + 8) * VROW + 16 * qt);
        const uint32_t wd = *reinterpret_cast<const uint32_t*>(svp + (2 * j + 9) * VROW + 16 * qt);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const uint32_t sel = uint32_t(r | (r << 4) | ((4 + r) << 8) | ((4 + r) << 12));  // byte r of each word
          const uint32_t xab = __byte_perm(wa, wb, sel) >> nsh;
          const uint32_t xcd = __byte_perm(wc, wd, sel) >> nsh;
          mma_bf16_16816(o[4 * qt + r], pa[qt * NG / 4], int4x2_to_bf16x2(xab, vmask, vmagic),
                         int4x2_to_bf16x2(xcd, vmask, vmagic));
        }
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();

  // ---- merge the warp's parts and store it for the CTA merge ----
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);
  float oa[16], ob[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    oa[i] = o[i][0] + o[i][2];
    ob[i] = o[i][1] + o[i][3];
    oa[i] += __shfl_xor_sync(0xffffffffu, oa[i], 16);
    ob[i] += __shfl_xor_sync(0xffffffffu, ob[i], 16);
  }
  __syncthreads();  // every warp is done with its ring: the merge area may reuse it
  // Lane (g < 4, j) holds head g at dims 32j + i (oa) and 32j + 16 + i (ob).
  // The merge area and the workspace keep a head's 128 values in the order
  // idx = 8 * (dim & 15) + 4 * ((dim >> 4) & 1) + (dim >> 5), a permutation of
  // the index bits, under which H_128 is unchanged.
  if (g < 4) {
    float* cb = sm.u.comb[w][g];
    if constexpr (NG == 1) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        cb[8 * i + j] = oa[i];
        cb[8 * i + 4 + j] = ob[i];
      }
    } else {
      // oa[i] holds dim 32 (i >> 2) + 8 j + 2 (i & 3), ob[i] the next one;
      // idx(dim) = 8 (dim & 15) + 4 ((dim >> 4) & 1) + (dim >> 5)
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int lo = 8 * (j & 1) + 2 * (i & 3);  // (dim & 15) of oa[i]
        const int idx = 8 * lo + 4 * (j >> 1) + (i >> 2);
        cb[idx] = oa[i];
        cb[idx + 8] = ob[i];  // dim + 1: (dim & 15) + 1
      }
    }
    if (j == 0) {
      sm.m[w][g] = m_run;
      sm.l[w][g] = l_run;
    }
  }
  __syncthreads();

  // ---- CTA merge: thread (head w, lane) owns idx 4*lane .. 4*lane+3 ----
  const int64_t slot = (int64_t(grp) * a.splits + split) * kAttnHeads + w;
  {
    float M = -INFINITY;
#pragma unroll
    for (int u = 0; u < kAttnWarps; ++u) M = fmaxf(M, sm.m[u][w]);
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < kAttnWarps; ++u) {
      const float mu = sm.m[u][w];
      const float f = mu == -INFINITY ? 0.f : exp2f(mu - M);
      L = fmaf(f, sm.l[u][w], L);
      const float4 v = *reinterpret_cast<const float4*>(&sm.u.comb[u][w][4 * lane]);
      acc.x = fmaf(f, v.x, acc.x);
      acc.y = fmaf(f, v.y, acc.y);
      acc.z = fmaf(f, v.z, acc.z);
      acc.w = fmaf(f, v.w, acc.w);
    }
    *reinterpret_cast<float4*>(a.part_o + slot * kAttnDim + 4 * lane) = acc;
    if (lane == 0) *reinterpret_cast<float2*>(a.part_ml + slot * 2) = make_float2(M, L);
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) sm.last = atomicAdd(a.counters + grp, 1u) == unsigned(a.splits - 1);
  __syncthreads();
  if (!sm.last) return;
  __threadfence();

  // ---- last CTA of the group: merge all splits, undo the rotation ----
  // Pass 1: every thread fetches (m, l) pairs at once; each warp then reduces
  // its head's maximum M and sum L and keeps the weights 2^(m - M) in shared
  // memory.  Pass 2: independent loads of the partial outputs, weighted.
  float2* ml_s = reinterpret_cast<float2*>(&sm.u.stage[0][0][0]);           // [splits][4]
  float* f_s = reinterpret_cast<float*>(ml_s + kAttnMaxSplits * kAttnHeads);  // [4][splits]
  const float2* pml = reinterpret_cast<const float2*>(a.part_ml) + int64_t(grp) * a.splits * kAttnHeads;
  for (int i = tid; i < a.splits * kAttnHeads; i += kAttnThreads) ml_s[i] = __ldcg(pml + i);
  __syncthreads();
  if (w < hn) {
    float M = -INFINITY;
    for (int sp = lane; sp < a.splits; sp += 32) M = fmaxf(M, ml_s[sp * kAttnHeads + w].x);
#pragma unroll
    for (int m = 16; m; m >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, m));
    float L = 0.f;
    for (int sp = lane; sp < a.splits; sp += 32) {
      const float2 ml = ml_s[sp * kAttnHeads + w];
      const float f = ml.x == -INFINITY ? 0.f : exp2f(ml.x - M);
      f_s[w * kAttnMaxSplits + sp] = f;
      L = fmaf(f, ml.y, L);
    }
#pragma unroll
    for (int m = 16; m; m >>= 1) L += __shfl_xor_sync(0xffffffffu, L, m);
    __syncwarp();
    const float4* po = reinterpret_cast<const float4*>(a.part_o + (int64_t(grp) * a.splits * kAttnHeads + w) *
                                                                      kAttnDim) + lane;
    const float* fw = f_s + w * kAttnMaxSplits;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int sp = 0;
    for (; sp + 8 <= a.splits; sp += 8) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldcg(po + int64_t(sp + u) * kAttnHeads * (kAttnDim / 4));
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float f = fw[sp + u];
        acc.x = fmaf(f, v[u].x, acc.x);
        acc.y = fmaf(f, v[u].y, acc.y);
        acc.z = fmaf(f, v[u].z, acc.z);
        acc.w = fmaf(f, v[u].w, acc.w);
      }
    }
    for (; sp < a.splits; ++sp) {
      const float4 v = __ldcg(po + int64_t(sp) * kAttnHeads * (kAttnDim / 4));
      const float f = fw[sp];
      acc.x = fmaf(f, v.x, acc.x);
      acc.y = fmaf(f, v.y, acc.y);
      acc.z = fmaf(f, v.z, acc.z);
      acc.w = fmaf(f, v.w, acc.w);
    }
    const float inv = a.inv_sqrt_dim / L;
    float y[4] = {acc.x, acc.y, acc.z, acc.w};
    // H_128 on the permuted index: bits 0-1 in registers, bits 2-6 on lanes.
    bfly(y[0], y[1]);
    bfly(y[2], y[3]);
    bfly(y[0], y[2]);
    bfly(y[1], y[3]);
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const bool upper = (lane & m) != 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float ov = __shfl_xor_sync(0xffffffffu, y[i], m);
        y[i] = upper ? ov - y[i] : y[i] + ov;
      }
    }
    const int64_t orow = (int64_t(bidx) * a.nqh + head0 + w) * kAttnDim;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      // idx = 4*lane + r  ->  dim = 32 r + 16 (lane & 1) + (lane >> 1)
      const int dim = 32 * r + 16 * (lane & 1) + (lane >> 1);
      float v = y[r] * inv;
      if (a.signs && a.signs[dim] < 0) v = -v;
      if (a.out_f32)
        static_cast<float*>(a.out)[orow + dim] = v;
      else
        static_cast<uint16_t*>(a.out)[orow + dim] = uint16_t(pack_bf16x2(v, 0.f) & 0xffffu);
    }
  }
  if (tid == 0) a.counters[grp] = 0u;  // ready for the next call
}

}  // namespace hadq
