// Forward 128-point Hadamard blocks with one scale per block (G = B = 128),
// optionally preceded by a +-1 sign vector, with the first 16-point stage on
// tensor cores.
//
// H_128 = H_8 (x) H_16 on the index split j = 16 p + q of a block.  The bf16
// input is exact in bf16 and H_16 holds only +-1, so the transform along q is
// a bf16 GEMM with exact products and float32 accumulation.  One MMA tile
// takes row p (16 elements) of 16 different blocks: D[block][n] = sum_q
// x[block][p][q] H_16[q][n].  A lane then holds, for its two blocks (MMA rows
// g and g + 8), the outputs of all eight p in its own registers, so the
// remaining three stages (along p) need no exchange at all.  The columns of
// H_16 are permuted in the B fragments so that lane t4 receives the four
// consecutive outputs n = 4 t4 .. 4 t4 + 3: its codes leave as whole words.
//
// Per slab of 16 consecutive blocks (one warp per slab, staged in shared
// memory by cp.async into slots of 272 bytes; the slab after next is
// prefetched into L2 so that the staging copy hits L2):
//   1. 8 tiles: ldmatrix.x4 (the eight rows of an 8x8 load are eight blocks,
//      272 bytes apart: conflict-free), two MMAs;
//   2. three paired-FP32 stages over p;
//   3. per block: maximum over the lane's 32 outputs and a two-step shuffle
//      over the block's four lanes, scale, codes into the block's slot;
//   4. a coalesced copy-out of the codes (the slab's codes are contiguous).
//
// Signs.  The sign of an element flips the sign bit of its bf16 value, so it
// is an XOR on the A fragments before the MMA (the products stay exact).  A
// lane's fragments of tile row p hold columns 16 p + 2 t4 (+1) and 16 p + 8 +
// 2 t4 (+1) of its two blocks; over the eight p those are 32 sign bits per
// block and lane quarter t4.  A per-CTA table keeps them as two words per
// (column block, t4), bit 15 - p and bit 31 - p holding the pair of tile row
// p, so the mask of a fragment register is (word << p) & 0x80008000: a shift
// and one three-input logic operation.  Each lane reads the two table
// entries of its blocks once per slab; the blocks of a slab span rows, so a
// block's column position is its block index modulo the blocks per row, and
// the table repeats its first 16 entries after the last so that the slab's
// start column plus the block offset indexes it directly.
#pragma once

#include "hadq_chunk.cuh"
#include "hadq_mma.cuh"

namespace hadq {

// Shared-memory bytes of the sign-word table: one uint2 per (entry, t4), with
// entries for the column blocks 0 .. cpr - 1 followed by 16 more that repeat
// them (entry e holds column block e mod cpr), so that a slab's column
// positions colc + b (colc < cpr, b < 16) index it without a modulo.
__host__ __device__ inline size_t chunk_mma_sign_bytes(int dim) { return size_t(dim / 128 + 16) * 4 * sizeof(uint2); }

// Sign-word table of one row (all threads; the caller synchronises): entry
// (cb, t4) = {W0, W1}, W0 bit 15 - p / 31 - p = sign of column 16 p + 2 t4 /
// + 1 of column block cb mod cpr negative, W1 the same for columns 16 p + 8 +
// 2 t4 / + 1; cb runs over cpr + 16 entries.
__device__ __forceinline__ void load_mma_sign_words(const int8_t* signs, int cpr, uint2* sw) {
  for (int e = threadIdx.x; e < (cpr + 16) * 4; e += blockDim.x) {
    const int8_t* s = signs + ((e >> 2) % cpr) * 128 + 2 * (e & 3);
    uint32_t w0 = 0, w1 = 0;
    for (int p = 0; p < 8; ++p) {
      w0 |= (uint32_t)(s[16 * p] < 0) << (15 - p) | (uint32_t)(s[16 * p + 1] < 0) << (31 - p);
      w1 |= (uint32_t)(s[16 * p + 8] < 0) << (15 - p) | (uint32_t)(s[16 * p + 9] < 0) << (31 - p);
    }
    sw[e] = make_uint2(w0, w1);
  }
}

// Blocks per slab: one warp owns one slab of kMmaSlab consecutive blocks (one
// MMA tile of 16 rows), staged twice (the next slab streams in while this one
// is computed).  16 blocks keep a lane at 64 values and a warp at 8.7 KB of
// staging, so five CTAs of four warps fit per SM.
constexpr int kMmaSlab = 16;
constexpr int kMmaWarps = 4;
constexpr int kMmaStageBytes = kMmaSlab * kCPad;

__host__ __device__ inline size_t chunk_mma_stage_bytes() { return size_t(2) * kMmaWarps * kMmaStageBytes; }

// Copies `nch` blocks of 16 * PPC bytes at `src` into slots of `dst` (pitch
// kCPad); consecutive lanes take consecutive 16-byte pieces.
template <int PPC>
__device__ __forceinline__ void mma_slab_load(const uint8_t* src, int nch, uint8_t* dst, int lane) {
  if (nch == kMmaSlab) {
#pragma unroll
    for (int i = 0; i < kMmaSlab * PPC / 32; ++i) {
      const int p = lane + 32 * i;
      cp_async16(dst + (p / PPC) * kCPad + 16 * (p % PPC), src + 16 * p);
    }
  } else {
    for (int p = lane; p < nch * PPC; p += 32) cp_async16(dst + (p / PPC) * kCPad + 16 * (p % PPC), src + 16 * p);
  }
}

// Copies `nch` results of 16 * PPC bytes from the slots of `src` to `dst`.
template <int PPC>
__device__ __forceinline__ void mma_slab_store(const uint8_t* src, int nch, uint8_t* dst, int lane) {
  if (nch == kMmaSlab) {
#pragma unroll
    for (int i = 0; i < kMmaSlab * PPC / 32; ++i) {
      const int p = lane + 32 * i;
      *reinterpret_cast<uint4*>(dst + 16 * p) = *reinterpret_cast<const uint4*>(src + (p / PPC) * kCPad + 16 * (p % PPC));
    }
  } else {
    for (int p = lane; p < nch * PPC; p += 32)
      *reinterpret_cast<uint4*>(dst + 16 * p) = *reinterpret_cast<const uint4*>(src + (p / PPC) * kCPad + 16 * (p % PPC));
  }
}

__host__ __device__ inline size_t chunk_mma_smem_bytes(int dim, bool signs) {
  return chunk_mma_stage_bytes() + (signs ? chunk_mma_sign_bytes(dim) : 0);
}

// ROT: also write the rotated float32 values (a.rot); a separate instance so
// that the codes-only kernel carries no registers for them.
// KEEP: kept-token rows (the keep table of ChunkKeepArgs) leave as bf16 copies
// in a.kept, with codes and scale 0; each lane looks up the keep-table entries
// of its two blocks one slab ahead.
// Four CTAs per SM (112 registers): with the five-CTA cap (95 registers) the
// compiler recomputed masks and addresses in every slab, 50 more
// instructions per slab, and the kernel ran 2-5 % slower.
template <int BITS, bool SIGNS, bool ROT, bool KEEP = false>
__global__ void __launch_bounds__(kMmaWarps * 32, 4) rq_chunk_mma_kernel(ChunkArgsT<KEEP> a) {
  static_assert(!(ROT && KEEP), "kept-token calls write no rotated values");
  constexpr float QMAX = (float)((1 << (BITS - 1)) - 1);
  constexpr int CB = BITS == 8 ? 128 : 64;  // code bytes per block
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const uint2* s_sw = reinterpret_cast<const uint2*>(smem + chunk_mma_stage_bytes());
  // Slab and chunk indices are 32-bit: the host takes this kernel only for
  // fewer than 2^30 chunks (a 256 GiB input), so every index below, including
  // the slab after next, stays under 2^31.  Byte offsets are widened.
  const int wstride = int(gridDim.x) * kMmaWarps;
  int slab = int(blockIdx.x) * kMmaWarps + wid;
  const uint8_t* xsrc = reinterpret_cast<const uint8_t*>(a.x);
  const int nslabs = int((a.nchunks + kMmaSlab - 1) / kMmaSlab);
  uint8_t* st0 = smem + (2 * wid) * kMmaStageBytes;
  uint8_t* st1 = st0 + kMmaStageBytes;
  constexpr int SB = kMmaSlab * 256;  // input bytes per slab

  // the first slab is in flight while the CTA builds its sign table
  if (slab < nslabs) mma_slab_load<16>(xsrc + size_t(slab) * SB, slab_count(slab * kMmaSlab, a.nchunks, kMmaSlab), st0, lane);
  cp_async_commit();
  // KEEP: keep-table entries of blocks g, g + 8 of the slab staged next.  The
  // token (row mod tokens) and the block's place in its row are carried from
  // slab to slab with adds, so that no division runs in the loop.
  int ks_next[2] = {-1, -1};
  int k_tok[2] = {0, 0}, k_col[2] = {0, 0};
  int k_dr = 0, k_dt = 0;  // advance per slab step: blocks within a row, tokens
  if constexpr (KEEP) {
    const uint32_t cpr = uint32_t(a.cpr), toks = uint32_t(a.keep_tokens), step = uint32_t(wstride) * kMmaSlab;
    k_dr = int(step % cpr);
    k_dt = int((step / cpr) % toks);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const uint32_t ch = uint32_t(slab * kMmaSlab + g + 8 * r);
      k_col[r] = int(ch % cpr);
      k_tok[r] = int((ch / cpr) % toks);
      if (slab < nslabs && int(ch) < a.nchunks) ks_next[r] = __ldg(a.keep_slot + k_tok[r]);
    }
  }
  if constexpr (SIGNS) {
    load_mma_sign_words(a.signs, a.cpr, reinterpret_cast<uint2*>(smem + chunk_mma_stage_bytes()));
    __syncthreads();
  }
  // column block of this warp's slab start, advanced from slab to slab
  int colc = SIGNS ? (int)((slab * kMmaSlab) % a.cpr) : 0;
  const int col_step = SIGNS ? (int)((wstride * kMmaSlab) % a.cpr) : 0;

  // B fragments of H_16 (bf16 +-1) with permuted columns: in n-tile nt,
  // column g holds output n = 4 (g >> 1) + 2 nt + (g & 1); k = 2 t4 + 8 kh
  uint32_t hb[2][2];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
    for (int kh = 0; kh < 2; ++kh) {
      const int k = 2 * t4 + 8 * kh, n = 4 * (g >> 1) + 2 * nt + (g & 1);
      const uint32_t lo = (__popc(k & n) & 1) ? 0xBF80u : 0x3F80u;
      const uint32_t hi = (__popc((k + 1) & n) & 1) ? 0xBF80u : 0x3F80u;
      hb[nt][kh] = lo | (hi << 16);
    }
  }
  // ldmatrix row of this lane: block (lane & 7) + 8 ((lane >> 3) & 1), column
  // half lane >> 4; tile row p adds 32 bytes
  const uint32_t lm_off = uint32_t(((lane & 7) + 8 * ((lane >> 3) & 1)) * kCPad + (lane >> 4) * 16);

  for (int it = 0; slab < nslabs; ++it, slab += wstride) {
    uint8_t* cur = (it & 1) ? st1 : st0;
    const int c = slab * kMmaSlab;
    const int ks[2] = {ks_next[0], ks_next[1]};
    cp_async_wait<0>();
    __syncwarp();
    {
      const int nx = slab + wstride;
      if (nx < nslabs) mma_slab_load<16>(xsrc + size_t(nx) * SB, slab_count(nx * kMmaSlab, a.nchunks, kMmaSlab), (it & 1) ? st0 : st1, lane);
      cp_async_commit();
      if constexpr (KEEP) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          k_col[r] += k_dr;
          const int carry = k_col[r] >= a.cpr;
          if (carry) k_col[r] -= a.cpr;
          k_tok[r] += k_dt + carry;
          if (k_tok[r] >= a.keep_tokens) k_tok[r] -= int(a.keep_tokens);
          const int ch = nx * kMmaSlab + g + 8 * r;
          ks_next[r] = (nx < nslabs && ch < a.nchunks) ? __ldg(a.keep_slot + k_tok[r]) : -1;
        }
      }
      const int n2 = nx + wstride;  // the slab after: into L2 now, staged next iteration
      if (lane == 0 && n2 < nslabs)
        prefetch_l2_bulk(xsrc + size_t(n2) * SB, uint32_t(slab_count(n2 * kMmaSlab, a.nchunks, kMmaSlab)) * 256u);
    }
    const int nch = slab_count(c, a.nchunks, kMmaSlab);  // blocks beyond nch hold stale data: computed, never stored
    // sign words of this lane's blocks g + 8 r
    uint2 sgw[2];
    if constexpr (SIGNS) {
#pragma unroll
      for (int r = 0; r < 2; ++r) sgw[r] = s_sw[(colc + g + 8 * r) * 4 + t4];  // colc + g + 8 r < cpr + 16
      colc += col_step;
      if (colc >= a.cpr) colc -= a.cpr;
    }

    // 1. H_16 along q: u[8 p + 4 r + e] = output n = 4 t4 + e of row p of block g + 8 r
    float u[64];
    const uint32_t cur_s = static_cast<uint32_t>(__cvta_generic_to_shared(cur));
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(cur_s + lm_off + uint32_t(p * 32), a0, a1, a2, a3);
      if constexpr (SIGNS) {  // a0 / a2: block g, a1 / a3: block g + 8
        a0 ^= (sgw[0].x << p) & 0x80008000u;
        a1 ^= (sgw[1].x << p) & 0x80008000u;
        a2 ^= (sgw[0].y << p) & 0x80008000u;
        a3 ^= (sgw[1].y << p) & 0x80008000u;
      }
      float d0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, d1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      mma_bf16_k16(d0, a0, a1, a2, a3, hb[0][0], hb[0][1]);
      mma_bf16_k16(d1, a0, a1, a2, a3, hb[1][0], hb[1][1]);
      float* o = u + 8 * p;
      o[0] = d0[0];
      o[1] = d0[1];
      o[2] = d1[0];
      o[3] = d1[1];
      o[4] = d0[2];
      o[5] = d0[3];
      o[6] = d1[2];
      o[7] = d1[3];
    }
    // 2. H_8 along p
    reg_stage<64, 8>(u);
    reg_stage<64, 16>(u);
    reg_stage<64, 32>(u);
    // KEEP: a kept block's staged bf16 input goes out unchanged, 64 bytes per
    // lane of its four, before its slot takes the codes
    bool kept[2] = {false, false};
    if constexpr (KEEP) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int b = g + 8 * r;
        const int64_t kofs = b < nch ? kept_offset(a, c + b, ks[r]) : -1;
        if (kofs >= 0) {
          kept[r] = true;
          const uint4* src = reinterpret_cast<const uint4*>(cur + b * kCPad + 64 * t4);
          uint4* dst = reinterpret_cast<uint4*>(a.kept + kofs + 32 * t4);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = src[i];
        }
      }
    }
    __syncwarp();  // every lane has loaded its fragments: the slots take the codes

    // 3. per block: maximum, scale, codes
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float* v = u + 4 * r;  // v[8 p + e]
      float m0 = 0.0f, m1 = 0.0f;
#pragma unroll
      for (int p = 0; p < 8; p += 2) {
        m0 = max3(m0, fabsf(v[8 * p]), fabsf(v[8 * p + 1]));
        m1 = max3(m1, fabsf(v[8 * p + 2]), fabsf(v[8 * p + 3]));
        m0 = max3(m0, fabsf(v[8 * p + 8]), fabsf(v[8 * p + 9]));
        m1 = max3(m1, fabsf(v[8 * p + 10]), fabsf(v[8 * p + 11]));
      }
      float m = fmaxf(m0, m1);
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      if constexpr (KEEP)
        if (kept[r]) m = 0.0f;  // scale 0
      const int b = g + 8 * r;
      const bool live = b < nch;
      if (t4 == 0 && live) a.scales[c + b] = m * a.scale_mul;
      if constexpr (ROT) {
        if (live) {
          float* rr = a.rot + size_t(c + b) * kCK + 4 * t4;
#pragma unroll
          for (int p = 0; p < 8; ++p)
            *reinterpret_cast<float4*>(rr + 16 * p) = make_float4(v[8 * p] * a.rsqrt_b, v[8 * p + 1] * a.rsqrt_b,
                                                                  v[8 * p + 2] * a.rsqrt_b, v[8 * p + 3] * a.rsqrt_b);
        }
      }
      const QInv q = make_qinv(m, QMAX);
      if (q.tiny) {
#pragma unroll
        for (int p = 0; p < 8; ++p)
#pragma unroll
          for (int e = 0; e < 4; ++e) v[8 * p + e] *= 18446744073709551616.0f;
      }
      uint8_t* slot = cur + b * kCPad;
      if constexpr (BITS == 8) {
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          uint32_t c0, c1, c2, c3;
          magic_code2(v[8 * p], v[8 * p + 1], q.inv, c0, c1);
          magic_code2(v[8 * p + 2], v[8 * p + 3], q.inv, c2, c3);
          const uint32_t wd = (KEEP && kept[r]) ? 0u : pack_i8x4(c0, c1, c2, c3);
          *reinterpret_cast<uint32_t*>(slot + 16 * p + 4 * t4) = wd;  // outputs 16 p + 4 t4 .. + 3
        }
      } else {
        // rows p and p + 1 in one word: its low half holds outputs 16 p + 4 t4 .. + 3, the high half those of p + 1
#pragma unroll
        for (int p = 0; p < 8; p += 2) {
          uint32_t cc[8];
          magic_code2(v[8 * p], v[8 * p + 1], q.inv, cc[0], cc[1]);
          magic_code2(v[8 * p + 2], v[8 * p + 3], q.inv, cc[2], cc[3]);
          magic_code2(v[8 * p + 8], v[8 * p + 9], q.inv, cc[4], cc[5]);
          magic_code2(v[8 * p + 10], v[8 * p + 11], q.inv, cc[6], cc[7]);
          const uint32_t wd = (KEEP && kept[r]) ? 0u : pack_i4x8(cc);
          *reinterpret_cast<uint16_t*>(slot + 8 * p + 2 * t4) = (uint16_t)(wd & 0xffffu);
          *reinterpret_cast<uint16_t*>(slot + 8 * p + 8 + 2 * t4) = (uint16_t)(wd >> 16);
        }
      }
    }
    __syncwarp();
    mma_slab_store<CB / 16>(cur, nch, a.codes + size_t(c) * CB, lane);
  }
  cp_async_wait<0>();
}

}  // namespace hadq
