// Chunk path: Hadamard blocks of B = 8..128 columns, dim a multiple of 128.
//
// Every thread owns one 128-element chunk of a row (chunks never cross rows),
// so all log2(B) butterfly stages run in registers with no shuffles.
//
// Teams.  Work is dealt in slabs of consecutive chunks, which are contiguous
// in memory.  A slab belongs to a team: one warp (32 chunks) whenever no scale
// group spans more than a warp's chunks, otherwise the whole CTA (128 threads).
// A warp team synchronises with __syncwarp only, so warps never wait on each
// other.  Slabs are dealt round-robin over all teams of the grid, so at any
// moment the grid works on one compact window of memory.
//
// Each slab is staged through shared memory:
//   load   16-byte cp.async copies, consecutive lanes on consecutive 16-byte
//          pieces (fully coalesced), into chunk slots padded to 272 bytes so
//          that a thread reading its own chunk row-wise is bank-conflict free.
//          Two stages per team: the next slab streams in while this one is
//          computed.
//   store  each thread writes its results back into its own slot; after a
//          team barrier the team copies them out with coalesced 16-byte
//          stores (they too are contiguous in memory).
//
// Scale groups: G = 2^g with 8 <= G <= 128 reduce inside the thread; groups of
// gpc = G/128 chunks reduce with lane shuffles (warp team, gpc divides 32) or
// one shared-memory max per slab (CTA team); a slab always holds whole groups.
#pragma once

#include <type_traits>

#include "hadq_common.cuh"

namespace hadq {

constexpr int kCK = 128;     // elements per chunk (one thread)
constexpr int kCT = 128;     // threads per CTA
constexpr int kCPad = 272;   // bytes per chunk slot in shared memory (256 + 16)

struct ChunkArgs {
  const uint16_t* x;         // forward input (bf16)
  const uint8_t* codes_in;   // inverse input
  const float* scales_in;
  const int8_t* signs;
  uint8_t* codes;
  float* scales;
  float* rot;                // forward: optional fp32 y; inverse: fp32 output
  uint16_t* out_bf16;
  int64_t nchunks;           // rows * dim / 128
  int cpr;                   // chunks per row
  int slab_chunks;           // chunks per slab: 32 (warp team) or <= 128, a multiple of gpc
  int G;
  int log_g;                 // log2(G) when G <= 128, else -1
  int gpc;                   // chunks per group when G > 128, else 1
  int dim;
  float scale_mul;
  float rsqrt_b;
};

// Arguments of the kept-token (mixed-precision) variants.  Rows are
// [heads, keep_tokens]; token t is kept when keep_slot[t] is in [0, n_keep),
// and its rows live as bf16 in kept[head][keep_slot[t]][dim].  The plain
// kernels take the ChunkArgs base alone.
struct ChunkKeepArgs : ChunkArgs {
  const int32_t* keep_slot;
  uint16_t* kept;
  int64_t keep_tokens;
  int n_keep;
};
template <bool KEEP>
using ChunkArgsT = typename std::conditional<KEEP, ChunkKeepArgs, ChunkArgs>::type;

// Keep-table entry of the token of chunk `ch` (kept-token calls have fewer
// than 2^31 chunks).  Loaded one slab ahead of its use.
__device__ __forceinline__ int kept_slot_of(const ChunkKeepArgs& a, int64_t ch) {
  const uint32_t row = static_cast<uint32_t>(ch) / static_cast<uint32_t>(a.cpr);
  return __ldg(a.keep_slot + row % static_cast<uint32_t>(a.keep_tokens));
}

// Element offset into `kept` of chunk `ch` whose token has keep-table entry
// `s`, or -1 when the token is not kept.
__device__ __forceinline__ int64_t kept_offset(const ChunkKeepArgs& a, int64_t ch, int s) {
  if (s < 0 || s >= a.n_keep) return -1;
  const uint32_t c32 = static_cast<uint32_t>(ch);
  const uint32_t row = c32 / static_cast<uint32_t>(a.cpr);
  const uint32_t head = row / static_cast<uint32_t>(a.keep_tokens);
  return (int64_t(head) * a.n_keep + s) * a.dim + int64_t(c32 - row * uint32_t(a.cpr)) * kCK;
}

// Shared-memory layout shared by host and device:
//   [two stages of kCT slots][sign table, sign bits (SIGNS)][group max (CTA teams)]
// The sign vector is kept as packed bits (one per column) plus a 256-entry
// table mapping a byte of 8 sign bits to the four XOR masks of its bf16 pairs,
// so the layout stays near 74 KB for any width (three CTAs per SM).
__host__ __device__ constexpr int chunk_stage_bytes() { return kCT * kCPad; }
constexpr int kSignTabBytes = 256 * 16;
__host__ __device__ inline int sign_bits_bytes(int dim) { return ((dim / 8) + 15) & ~15; }
__host__ __device__ inline size_t chunk_smem_bytes(int dim, bool signs, bool cta_team) {
  return size_t(2) * chunk_stage_bytes() + (signs ? size_t(kSignTabBytes + sign_bits_bytes(dim)) : 0) +
         (cta_team ? size_t(2 * kCT * sizeof(uint32_t)) : 0);
}

// Builds the sign table and the packed sign bits of one row (all threads; the
// caller synchronises).  Bit b of word w is set when signs[32 w + b] < 0.
__device__ __forceinline__ void load_sign_tables(const int8_t* signs, int dim, uint4* s_tab, uint32_t* s_bits) {
  for (int e = threadIdx.x; e < 256; e += blockDim.x) {
    uint32_t m[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) m[k] = (((uint32_t)e >> (2 * k)) & 1u) << 15 | (((uint32_t)e >> (2 * k + 1)) & 1u) << 31;
    s_tab[e] = make_uint4(m[0], m[1], m[2], m[3]);
  }
  for (int w = threadIdx.x; w < dim / 32; w += blockDim.x) {
    uint32_t b = 0;
    for (int i = 0; i < 32; ++i) b |= (uint32_t)(signs[32 * w + i] < 0) << i;
    s_bits[w] = b;
  }
}

// XOR masks of the 4 bf16 pairs of 8-column vector p of a chunk whose 128 sign
// bits are `sb`.
__device__ __forceinline__ uint4 sign_masks8(const uint4* s_tab, const uint4& sb, int p) {
  const uint32_t w = (p >> 2) == 0 ? sb.x : (p >> 2) == 1 ? sb.y : (p >> 2) == 2 ? sb.z : sb.w;
  return s_tab[__byte_perm(w, 0, 0x4440 + (p & 3))];
}

// A team of TEAM threads (32: one warp, 128: the CTA) owning one slab at a time.
template <int TEAM>
struct Team {
  static_assert(TEAM == 32 || TEAM == kCT, "warp or CTA teams");
  static constexpr int PER_CTA = kCT / TEAM;
  __device__ static int index() { return TEAM == 32 ? (int)(threadIdx.x >> 5) : 0; }
  __device__ static int tid() { return (int)threadIdx.x & (TEAM - 1); }
  __device__ static void sync() {
    if constexpr (TEAM == 32) __syncwarp(); else __syncthreads();
  }
  // this team's two stages of TEAM slots
  __device__ static uint8_t* stage(uint8_t* smem, int s) { return smem + (index() * 2 + s) * TEAM * kCPad; }
  __device__ static int64_t first() { return (int64_t)blockIdx.x * PER_CTA + index(); }
  __device__ static int64_t stride() { return (int64_t)gridDim.x * PER_CTA; }
};

// Copies `nch` chunks of 16 * PPC bytes starting at `src` into padded slots of
// `dst`.  Consecutive team threads take consecutive 16-byte pieces, so every
// warp reads 512 contiguous bytes per instruction.  Full slabs use a fully
// unrolled loop with constant strides.
template <int PPC, int TEAM>
__device__ __forceinline__ void chunk_load(const uint8_t* src, int nch, uint8_t* dst, int tt) {
  if (nch == TEAM) {
    constexpr int STEP = TEAM / PPC;  // chunks covered by one pass of the team
    const uint8_t* s0 = src + 16 * tt;
    uint8_t* d0 = dst + (tt / PPC) * kCPad + 16 * (tt % PPC);
#pragma unroll
    for (int i = 0; i < PPC; ++i) cp_async16(d0 + i * STEP * kCPad, s0 + i * 16 * TEAM);
  } else {
    for (int g = tt; g < nch * PPC; g += TEAM) cp_async16(dst + (g / PPC) * kCPad + 16 * (g % PPC), src + 16 * g);
  }
}

// Copies `nch` chunk results of 16 * PPC bytes from padded slots to `dst`.
template <int PPC, int TEAM>
__device__ __forceinline__ void chunk_store(const uint8_t* src, int nch, uint8_t* dst, int tt) {
  if (nch == TEAM) {
    constexpr int STEP = TEAM / PPC;
    const uint8_t* s0 = src + (tt / PPC) * kCPad + 16 * (tt % PPC);
    uint8_t* d0 = dst + 16 * tt;
#pragma unroll
    for (int i = 0; i < PPC; ++i)
      *reinterpret_cast<uint4*>(d0 + i * 16 * TEAM) = *reinterpret_cast<const uint4*>(s0 + i * STEP * kCPad);
  } else {
    for (int g = tt; g < nch * PPC; g += TEAM)
      *reinterpret_cast<uint4*>(dst + 16 * g) = *reinterpret_cast<const uint4*>(src + (g / PPC) * kCPad + 16 * (g % PPC));
  }
}

// Chunks of the slab starting at chunk c (the last slab may be short).
__device__ __forceinline__ int slab_count(int64_t c, int64_t nchunks, int slab_chunks) {
  const int64_t left = nchunks - c;
  return left < slab_chunks ? (int)left : slab_chunks;
}

// Codes of the 128 values of one chunk into its shared-memory slot: vector p
// (8 values) uses multiplier inv[p] (all equal when the group covers the chunk).
template <int BITS>
__device__ __forceinline__ void chunk_codes(const float (&v)[kCK], const float (&inv)[16], uint8_t* slot) {
#pragma unroll
  for (int p = 0; p < 16; p += 2) {
    uint32_t c[16];
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      magic_code2(v[8 * p + k], v[8 * p + k + 1], inv[p], c[k], c[k + 1]);
      magic_code2(v[8 * p + 8 + k], v[8 * p + 9 + k], inv[p + 1], c[8 + k], c[9 + k]);
    }
    if constexpr (BITS == 8) {
      *reinterpret_cast<uint4*>(slot + 8 * p) =
          make_uint4(pack_i8x4(c[0], c[1], c[2], c[3]), pack_i8x4(c[4], c[5], c[6], c[7]),
                     pack_i8x4(c[8], c[9], c[10], c[11]), pack_i8x4(c[12], c[13], c[14], c[15]));
    } else {
      const uint32_t a0[8] = {c[0], c[1], c[2], c[3], c[4], c[5], c[6], c[7]};
      const uint32_t a1[8] = {c[8], c[9], c[10], c[11], c[12], c[13], c[14], c[15]};
      *reinterpret_cast<uint2*>(slot + 4 * p) = make_uint2(pack_i4x8(a0), pack_i4x8(a1));
    }
  }
}

// Forward: bf16 -> signs -> H_B (B = 2^LOG_B, 8..128) -> group max -> codes.
// WIDE_G: the scale group covers whole chunks (G >= 128); otherwise 8 <= G < 128.
// TEAM: 32 (warp teams; groups of at most 32 chunks, gpc dividing 32) or 128.
// KEEP: rows of kept tokens (ChunkArgs.keep_slot) are copied out as bf16 and
// get codes 0 and scale 0.
template <int LOG_B, int BITS, bool SIGNS, bool WIDE_G, int TEAM, bool KEEP = false>
__global__ void __launch_bounds__(kCT, 3) rq_chunk_kernel(ChunkArgsT<KEEP> a) {
  using T = Team<TEAM>;
  constexpr float QMAX = (float)((1 << (BITS - 1)) - 1);
  constexpr int CB = BITS == 8 ? 128 : 64;  // code bytes per chunk
  extern __shared__ __align__(16) uint8_t smem[];
  uint4* s_tab = reinterpret_cast<uint4*>(smem + 2 * chunk_stage_bytes());
  uint32_t* s_bits = reinterpret_cast<uint32_t*>(smem + 2 * chunk_stage_bytes() + kSignTabBytes);
  uint32_t* s_gmax = reinterpret_cast<uint32_t*>(smem + 2 * chunk_stage_bytes() +
                                                 (SIGNS ? kSignTabBytes + sign_bits_bytes(a.dim) : 0));  // [2][kCT], CTA teams
  const int tt = T::tid();
  const int G = a.G;
  const bool multi = WIDE_G && G > kCK;  // groups spanning several chunks

  if constexpr (SIGNS) load_sign_tables(a.signs, a.dim, s_tab, s_bits);
  if constexpr (TEAM == kCT) {
    for (int i = threadIdx.x; i < 2 * kCT; i += kCT) s_gmax[i] = 0u;
  }
  __syncthreads();  // masks and group-max area ready (the only CTA-wide barrier of warp teams)

  const uint8_t* xsrc = reinterpret_cast<const uint8_t*>(a.x);
  const int64_t nslabs = (a.nchunks + a.slab_chunks - 1) / a.slab_chunks;
  // Column chunk of this thread's chunk, advanced from slab to slab (sign
  // masks only); group bookkeeping for groups spanning several chunks.
  int colc = SIGNS ? (int)((T::first() * a.slab_chunks + tt) % a.cpr) : 0;
  const int col_step = SIGNS ? (int)((T::stride() * a.slab_chunks) % a.cpr) : 0;
  const int gslot = multi ? tt / a.gpc : 0;         // group of this chunk inside its slab
  const bool glead = multi ? (tt - gslot * a.gpc) == 0 : true;
  const int groups_per_slab = multi ? a.slab_chunks / a.gpc : 0;
  uint8_t* st0 = T::stage(smem, 0);
  uint8_t* st1 = T::stage(smem, 1);

  int64_t slab = T::first();
  int kslot_next = -1;  // KEEP: keep-table entry of this thread's chunk in the next slab
  if (slab < nslabs) {
    chunk_load<16, TEAM>(xsrc + slab * a.slab_chunks * 256, slab_count(slab * a.slab_chunks, a.nchunks, a.slab_chunks), st0, tt);
    if constexpr (KEEP)
      if (slab * a.slab_chunks + tt < a.nchunks) kslot_next = kept_slot_of(a, slab * a.slab_chunks + tt);
  }
  cp_async_commit();
  for (int it = 0; slab < nslabs; ++it, slab += T::stride()) {
    uint8_t* cur = (it & 1) ? st1 : st0;
    const int64_t c = slab * a.slab_chunks;
    const int kslot = kslot_next;
    cp_async_wait<0>();
    T::sync();  // slab data visible; the other stage is free again
    {
      const int64_t nx = slab + T::stride();
      if (nx < nslabs) {
        chunk_load<16, TEAM>(xsrc + nx * a.slab_chunks * 256, slab_count(nx * a.slab_chunks, a.nchunks, a.slab_chunks),
                             (it & 1) ? st0 : st1, tt);
        if constexpr (KEEP)
          kslot_next = nx * a.slab_chunks + tt < a.nchunks ? kept_slot_of(a, nx * a.slab_chunks + tt) : -1;
      }
      cp_async_commit();
    }
    const int nch = slab_count(c, a.nchunks, a.slab_chunks);
    const int64_t ch = c + tt;
    const bool active = tt < nch;
    const int col0 = colc * kCK;
    if constexpr (SIGNS) {
      colc += col_step;
      if (colc >= a.cpr) colc -= a.cpr;
    }
    uint8_t* mine = cur + tt * kCPad;
    // kept row: its bf16 chunk is copied out unchanged; codes and scales are 0
    bool kept_row = false;
    if constexpr (KEEP) {
      const int64_t kofs = active ? kept_offset(a, ch, kslot) : -1;
      kept_row = kofs >= 0;
      if (kept_row) {  // rare: a rolled loop keeps registers free
        uint4* dst = reinterpret_cast<uint4*>(a.kept + kofs);
#pragma unroll 1
        for (int p = 0; p < 16; ++p) dst[p] = *reinterpret_cast<const uint4*>(mine + 16 * p);
      }
    }

    float v[kCK];
    float pm[16];
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
      if constexpr (WIDE_G) {
        // one group covers the chunk: fuse the maximum into the last stage
        reg_fwht_from<kCK, 1, LOG_B - 1>(v);
        pm[0] = reg_stage_absmax<kCK, (1 << (LOG_B - 1))>(v);
#pragma unroll
        for (int p = 1; p < 16; ++p) pm[p] = pm[0];
      } else {
        reg_fwht_from<kCK, 1, LOG_B>(v);
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          float m = fmaxf(fabsf(v[8 * p]), fabsf(v[8 * p + 1]));
#pragma unroll
          for (int k = 2; k < 8; ++k) m = fmaxf(m, fabsf(v[8 * p + k]));
          pm[p] = m;
        }
      }
    } else {
#pragma unroll
      for (int p = 0; p < 16; ++p) pm[p] = 0.0f;
    }

    float gmax = 0.0f;  // WIDE_G: maximum of the whole group
    if constexpr (WIDE_G) {
      gmax = pm[0];
      if constexpr (TEAM == 32) {
        // groups of gpc consecutive lanes (gpc divides 32): butterfly max
        for (int b = 1; b < a.gpc; b <<= 1) gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, b));
      } else {
        if (multi) {
          uint32_t* slot = s_gmax + (it & 1) * kCT + gslot;
          if (active) atomicMax(slot, __float_as_uint(gmax));
          __syncthreads();
          gmax = __uint_as_float(*slot);
          s_gmax[((it + 1) & 1) * kCT + tt] = 0u;  // read two slabs later, after two barriers
        }
      }
    } else {
#pragma unroll
      for (int l = 0; l < 4; ++l) {
        if (G > (8 << l)) {
          float t[16];
#pragma unroll
          for (int p = 0; p < 16; ++p) t[p] = fmaxf(pm[p], pm[p ^ (1 << l)]);
#pragma unroll
          for (int p = 0; p < 16; ++p) pm[p] = t[p];
        }
      }
    }

    if (active) {
      // scale index = (flat element index of the group's first element) / G
      if constexpr (WIDE_G) {
        if (glead) a.scales[multi ? slab * groups_per_slab + gslot : ch] = kept_row ? 0.0f : gmax * a.scale_mul;
      } else {
        const int lg = a.log_g;
#pragma unroll
        for (int p = 0; p < 16; ++p)
          if (((8 * p) & (G - 1)) == 0)
            a.scales[((ch * kCK) >> lg) + ((8 * p) >> lg)] = kept_row ? 0.0f : pm[p] * a.scale_mul;
      }
      if (a.rot) {
        float4* dst = reinterpret_cast<float4*>(a.rot + ch * kCK);
#pragma unroll
        for (int i = 0; i < 32; ++i)
          dst[i] = make_float4(v[4 * i] * a.rsqrt_b, v[4 * i + 1] * a.rsqrt_b, v[4 * i + 2] * a.rsqrt_b,
                               v[4 * i + 3] * a.rsqrt_b);
      }
      // codes into this thread's own slot (its input is already in registers)
      float inv[16];
      bool tiny = false;
      if constexpr (WIDE_G) {
        const QInv q = make_qinv(gmax, QMAX);
        tiny = q.tiny;
#pragma unroll
        for (int p = 0; p < 16; ++p) inv[p] = q.inv;
      } else {
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          const QInv q = make_qinv(pm[p], QMAX);
          inv[p] = q.inv;
          tiny |= q.tiny;
        }
      }
      if (tiny) {  // groups whose maximum is below kTinyMax: codes from v * 2^64 (see make_qinv)
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          const float m = WIDE_G ? gmax : pm[p];
          if (m < kTinyMax) {
#pragma unroll
            for (int k = 0; k < 8; ++k) v[8 * p + k] *= 18446744073709551616.0f;
          }
        }
      }
      if (kept_row) {
#pragma unroll
        for (int p = 0; p < CB / 16; ++p) *reinterpret_cast<uint4*>(mine + 16 * p) = make_uint4(0, 0, 0, 0);
      } else {
        chunk_codes<BITS>(v, inv, mine);
      }
    }
    T::sync();
    chunk_store<CB / 16, TEAM>(cur, nch, a.codes + c * CB, tt);
  }
  cp_async_wait<0>();
}

// Inverse: codes * scale -> H_B -> signs -> bf16 (or fp32), warp teams.
//
// When every Hadamard block lies inside one scale group (G >= B), the
// butterflies run on the integer codes themselves (exact in float32: the sums
// stay at or below 128 * 127) and each vector is scaled once afterwards, by
// scale / sqrt(B).  Otherwise (G < B) the codes are scaled first.  With one
// scale per chunk (G >= 128) the scale of the next slab is loaded one slab
// ahead.
// KEEP: rows of kept tokens return the bf16 values stored in ChunkArgs.kept.
template <int LOG_B, int BITS, bool SIGNS, bool SCALE_FIRST, bool OUT_F32, bool KEEP = false>
__global__ void __launch_bounds__(kCT, 3) dq_chunk_kernel(ChunkArgsT<KEEP> a) {
  using T = Team<32>;
  constexpr int CB = BITS == 8 ? 128 : 64;  // code bytes per chunk
  extern __shared__ __align__(16) uint8_t smem[];
  uint4* s_tab = reinterpret_cast<uint4*>(smem + 2 * chunk_stage_bytes());
  uint32_t* s_bits = reinterpret_cast<uint32_t*>(smem + 2 * chunk_stage_bytes() + kSignTabBytes);
  const int tt = T::tid();
  const int G = a.G;
  const bool one_scale = G >= kCK;

  if constexpr (SIGNS) {
    load_sign_tables(a.signs, a.dim, s_tab, s_bits);
    __syncthreads();
  }
  const int64_t nslabs = (a.nchunks + a.slab_chunks - 1) / a.slab_chunks;
  int colc = SIGNS ? (int)((T::first() * a.slab_chunks + tt) % a.cpr) : 0;
  const int col_step = SIGNS ? (int)((T::stride() * a.slab_chunks) % a.cpr) : 0;
  uint8_t* st0 = T::stage(smem, 0);
  uint8_t* st1 = T::stage(smem, 1);
  auto chunk_scale = [&](int64_t ch) { return __ldg(a.scales_in + (a.gpc == 1 ? ch : ch / a.gpc)); };

  int64_t slab = T::first();
  float sc_next = 0.0f;
  int kslot_next = -1;  // KEEP: keep-table entry of this thread's chunk in the next slab
  if (slab < nslabs) {
    const int64_t c0 = slab * a.slab_chunks;
    chunk_load<CB / 16, 32>(a.codes_in + c0 * CB, slab_count(c0, a.nchunks, a.slab_chunks), st0, tt);
    if (one_scale && c0 + tt < a.nchunks) sc_next = chunk_scale(c0 + tt);
    if constexpr (KEEP)
      if (c0 + tt < a.nchunks) kslot_next = kept_slot_of(a, c0 + tt);
  }
  cp_async_commit();
  for (int it = 0; slab < nslabs; ++it, slab += T::stride()) {
    uint8_t* cur = (it & 1) ? st1 : st0;
    const int64_t c = slab * a.slab_chunks;
    const float sc_cur = sc_next;
    const int kslot = kslot_next;
    cp_async_wait<0>();
    T::sync();
    {
      const int64_t nx = slab + T::stride();
      if (nx < nslabs) {
        const int64_t cn = nx * a.slab_chunks;
        chunk_load<CB / 16, 32>(a.codes_in + cn * CB, slab_count(cn, a.nchunks, a.slab_chunks), (it & 1) ? st0 : st1, tt);
        if (one_scale && cn + tt < a.nchunks) sc_next = chunk_scale(cn + tt);
        if constexpr (KEEP) kslot_next = cn + tt < a.nchunks ? kept_slot_of(a, cn + tt) : -1;
      }
      cp_async_commit();
    }
    const int nch = slab_count(c, a.nchunks, a.slab_chunks);
    const int64_t ch = c + tt;
    const bool active = tt < nch;
    const int col0 = colc * kCK;
    if constexpr (SIGNS) {
      colc += col_step;
      if (colc >= a.cpr) colc -= a.cpr;
    }
    uint8_t* mine = cur + tt * kCPad;

    if (active) {
      // per-vector scale (a group covers >= 8 columns)
      float sc[16];
      if (one_scale) {
#pragma unroll
        for (int p = 0; p < 16; ++p) sc[p] = sc_cur;
      } else {
        const int lg = a.log_g;
#pragma unroll
        for (int p = 0; p < 16; ++p) sc[p] = __ldg(a.scales_in + (((ch * kCK) + 8 * p) >> lg));
      }
      // Scales below 2^-100 would give subnormal factors (scale / sqrt(B)) or
      // butterflies on subnormal values: those take factors at 2^64 scale and
      // one exact 2^-64 rescale at the end.
      bool tiny = false;
#pragma unroll
      for (int p = 0; p < 16; ++p) tiny |= sc[p] < kTinyScale && sc[p] != 0.0f;
      float v[kCK];
#pragma unroll
      for (int q4 = 0; q4 < CB / 16; ++q4) {
        const uint4 r = *reinterpret_cast<const uint4*>(mine + 16 * q4);
        if constexpr (BITS == 8) {  // 16 codes: elements 16 q4 .. 16 q4 + 15
          i8x4_to_float(r.x, v + 16 * q4);
          i8x4_to_float(r.y, v + 16 * q4 + 4);
          i8x4_to_float(r.z, v + 16 * q4 + 8);
          i8x4_to_float(r.w, v + 16 * q4 + 12);
        } else {                    // 32 codes: elements 32 q4 .. 32 q4 + 31
          i4x8_to_float(r.x, v + 32 * q4);
          i4x8_to_float(r.y, v + 32 * q4 + 8);
          i4x8_to_float(r.z, v + 32 * q4 + 16);
          i4x8_to_float(r.w, v + 32 * q4 + 24);
        }
      }
      const float pre = tiny ? kUp64 : 1.0f;
      if constexpr (SCALE_FIRST) {
        // the whole chunk runs at 2^64 scale when any of its scales is tiny
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          const float f = (sc[p] * pre) * a.rsqrt_b;
#pragma unroll
          for (int k = 0; k < 8; k += 2) mul2(v[8 * p + k], v[8 * p + k + 1], f);
        }
        reg_fwht<kCK, LOG_B>(v);
        if (tiny) {
#pragma unroll
          for (int i = 0; i < kCK; i += 2) mul2(v[i], v[i + 1], kDown64);
        }
      } else {
        // butterflies on the integer codes (exact), then one factor per vector
        reg_fwht<kCK, LOG_B>(v);
        if (!tiny) {
#pragma unroll
          for (int p = 0; p < 16; ++p) {
            const float f = sc[p] * a.rsqrt_b;
#pragma unroll
            for (int k = 0; k < 8; k += 2) mul2(v[8 * p + k], v[8 * p + k + 1], f);
          }
        } else {
#pragma unroll
          for (int p = 0; p < 16; ++p) {
            const bool t = sc[p] < kTinyScale;
            const float f = (sc[p] * (t ? kUp64 : 1.0f)) * a.rsqrt_b;
            const float g = t ? kDown64 : 1.0f;
#pragma unroll
            for (int k = 0; k < 8; ++k) v[8 * p + k] = (v[8 * p + k] * f) * g;
          }
        }
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
      // kept row: the stored bf16 values replace the reconstruction
      if constexpr (KEEP) {
        const int64_t kofs = kept_offset(a, ch, kslot);
        if (kofs >= 0) {
          const uint4* src = reinterpret_cast<const uint4*>(a.kept + kofs);
#pragma unroll 1
          for (int p = 0; p < 16; ++p) {
            const uint4 r = __ldg(src + p);
            if constexpr (OUT_F32) {
              float* dst = a.rot + ch * kCK + 8 * p;
              reinterpret_cast<float4*>(dst)[0] =
                  make_float4(bf16lo(r.x), bf16hi(r.x), bf16lo(r.y), bf16hi(r.y));
              reinterpret_cast<float4*>(dst)[1] =
                  make_float4(bf16lo(r.z), bf16hi(r.z), bf16lo(r.w), bf16hi(r.w));
            } else {
              *reinterpret_cast<uint4*>(mine + 16 * p) = r;
            }
          }
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

// Forward for 4096-column Hadamard blocks, one block per warp (one scale per
// block, G = 4096).  Lane c first owns chunk c (block columns 128c..128c+127)
// and runs index bits 0..6 in registers, exactly as in rq_chunk_kernel.  Index
// bits 7..11 are the lane number, so the warp then transposes its block
// through its own shared-memory slots, in two halves of 64 columns per chunk
// (column bit 1 clear, then set) so that it fits in the slab's 32 x 272-byte
// slots.
// Afterwards lane t holds columns 4t + j of every chunk c in register 4c + j:
// bits 7..11 are register bits 2..6, run as five more paired-FP32 stages.  Codes are
// written back into the slots in natural order and leave with the usual
// coalesced copy-out.
template <int BITS, bool SIGNS>
__global__ void __launch_bounds__(kCT, 3) rq_wide4096_kernel(ChunkArgs a) {
  using T = Team<32>;
  constexpr float QMAX = (float)((1 << (BITS - 1)) - 1);
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
  const int64_t nslabs = a.nchunks / 32;  // one 4096-column block per slab
  int colc = SIGNS ? (int)((T::first() * 32 + tt) % a.cpr) : 0;
  const int col_step = SIGNS ? (int)((T::stride() * 32) % a.cpr) : 0;
  uint8_t* st0 = T::stage(smem, 0);
  uint8_t* st1 = T::stage(smem, 1);

  int64_t slab = T::first();
  if (slab < nslabs) chunk_load<16, 32>(xsrc + slab * 32 * 256, 32, st0, tt);
  cp_async_commit();
  for (int it = 0; slab < nslabs; ++it, slab += T::stride()) {
    uint8_t* cur = (it & 1) ? st1 : st0;
    const int64_t c0 = slab * 32;
    cp_async_wait<0>();
    T::sync();
    {
      const int64_t nx = slab + T::stride();
      if (nx < nslabs) chunk_load<16, 32>(xsrc + nx * 32 * 256, 32, (it & 1) ? st0 : st1, tt);
      cp_async_commit();
    }
    const int col0 = colc * kCK;
    if constexpr (SIGNS) {
      colc += col_step;
      if (colc >= a.cpr) colc -= a.cpr;
    }
    uint8_t* mine = cur + tt * kCPad;

    float v[kCK];
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
    reg_fwht_from<kCK, 1, 7>(v);  // index bits 0..6

    // transpose inside the warp: first the columns with bit 1 clear, then those
    // with bit 1 set (64 per chunk, whole register pairs so that the written
    // half frees its registers); afterwards register 4c + j of lane t holds
    // column 4t + j of chunk c
    float u[kCK];
    float* slotf = reinterpret_cast<float*>(cur);  // slot c = 68 floats
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      __syncwarp();  // the slots are free (input read / previous half read)
#pragma unroll
      for (int q = 0; q < 16; ++q)
        *reinterpret_cast<float4*>(slotf + tt * 68 + 4 * q) =
            make_float4(v[8 * q + 2 * h], v[8 * q + 2 * h + 1], v[8 * q + 4 + 2 * h], v[8 * q + 5 + 2 * h]);
      __syncwarp();
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float2 f = *reinterpret_cast<const float2*>(slotf + c * 68 + 2 * tt);  // columns 4t + 2h, + 1
        u[4 * c + 2 * h] = f.x;
        u[4 * c + 2 * h + 1] = f.y;
      }
    }
    // index bits 7..11 = register bits 2..6
    reg_stage<kCK, 4>(u);
    reg_stage<kCK, 8>(u);
    reg_stage<kCK, 16>(u);
    reg_stage<kCK, 32>(u);
    float m = reg_stage_absmax<kCK, 64>(u);
#pragma unroll
    for (int b = 1; b < 32; b <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, b));
    if (tt == 0) a.scales[slab] = m * a.scale_mul;
    if (a.rot) {
      float* rr = a.rot + c0 * kCK + 4 * tt;
#pragma unroll
      for (int c = 0; c < 32; ++c)
        *reinterpret_cast<float4*>(rr + c * kCK) =
            make_float4(u[4 * c] * a.rsqrt_b, u[4 * c + 1] * a.rsqrt_b, u[4 * c + 2] * a.rsqrt_b, u[4 * c + 3] * a.rsqrt_b);
    }
    const QInv q = make_qinv(m, QMAX);
    if (q.tiny) {
#pragma unroll
      for (int i = 0; i < kCK; ++i) u[i] *= 18446744073709551616.0f;
    }
    __syncwarp();  // every lane has read the second half
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      uint32_t cc[4];
      magic_code2(u[4 * c], u[4 * c + 1], q.inv, cc[0], cc[1]);
      magic_code2(u[4 * c + 2], u[4 * c + 3], q.inv, cc[2], cc[3]);
      const uint32_t b4 = pack_i8x4(cc[0], cc[1], cc[2], cc[3]);  // columns 4t .. 4t + 3
      if constexpr (BITS == 8) {
        *reinterpret_cast<uint32_t*>(cur + c * kCPad + 4 * tt) = b4;
      } else {
        const uint32_t e = __byte_perm(b4, 0, 0x0020);  // columns 4t, 4t + 2
        const uint32_t o = __byte_perm(b4, 0, 0x0031);  // columns 4t + 1, 4t + 3
        *reinterpret_cast<uint16_t*>(cur + c * kCPad + 2 * tt) = (uint16_t)((e & 0x0f0fu) | ((o << 4) & 0xf0f0u));
      }
    }
    T::sync();
    chunk_store<CB / 16, 32>(cur, 32, a.codes + c0 * CB, tt);
  }
  cp_async_wait<0>();
}

}  // namespace hadq
