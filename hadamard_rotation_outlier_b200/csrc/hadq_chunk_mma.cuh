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
// Per slab of 32 blocks (staged in shared memory by cp.async, one warp per
// slab, as in rq_chunk_kernel):
//   1. two groups of 16 blocks x 8 tiles: ldmatrix.x4 (the eight rows of an
//      8x8 load are eight blocks, 272 bytes apart: conflict-free), two MMAs;
//   2. three paired-FP32 stages over p;
//   3. per block: maximum over the lane's 32 outputs and a two-step shuffle
//      over the block's four lanes, scale, codes into the block's slot;
//   4. the usual coalesced copy-out of the codes.
//
// Signs.  The sign of an element flips the sign bit of its bf16 value, so it
// is an XOR on the A fragments before the MMA (the products stay exact).  A
// lane's fragments of tile row p hold columns 16 p + 2 t4 (+1) and 16 p + 8 +
// 2 t4 (+1) of its two blocks; over the eight p those are 32 sign bits per
// block and lane quarter t4.  A per-CTA table keeps them as two words per
// (column block, t4), bit 15 - p and bit 31 - p holding the pair of tile row
// p, so the mask of a fragment register is (word << p) & 0x80008000: a shift
// and one three-input logic operation.  Each lane reads the four table
// entries of its blocks once per slab; the blocks of a slab span rows, so a
// block's column position is its chunk index modulo the chunks per row.
#pragma once

#include "hadq_chunk.cuh"
#include "hadq_mma.cuh"

namespace hadq {

// Shared-memory bytes of the sign-word table: one uint2 per (column block, t4).
__host__ __device__ inline size_t chunk_mma_sign_bytes(int dim) { return size_t(dim / 128) * 4 * sizeof(uint2); }
__host__ __device__ inline size_t chunk_mma_smem_bytes(int dim, bool signs) {
  return size_t(2) * chunk_stage_bytes() + (signs ? chunk_mma_sign_bytes(dim) : 0);
}

// Sign-word table of one row (all threads; the caller synchronises): entry
// (cb, t4) = {W0, W1}, W0 bit 15 - p / 31 - p = sign of column 16 p + 2 t4 /
// + 1 of block cb negative, W1 the same for columns 16 p + 8 + 2 t4 / + 1.
__device__ __forceinline__ void load_mma_sign_words(const int8_t* signs, int cpr, uint2* sw) {
  for (int e = threadIdx.x; e < cpr * 4; e += blockDim.x) {
    const int8_t* s = signs + (e >> 2) * 128 + 2 * (e & 3);
    uint32_t w0 = 0, w1 = 0;
    for (int p = 0; p < 8; ++p) {
      w0 |= (uint32_t)(s[16 * p] < 0) << (15 - p) | (uint32_t)(s[16 * p + 1] < 0) << (31 - p);
      w1 |= (uint32_t)(s[16 * p + 8] < 0) << (15 - p) | (uint32_t)(s[16 * p + 9] < 0) << (31 - p);
    }
    sw[e] = make_uint2(w0, w1);
  }
}

// ROT: also write the rotated float32 values (a.rot); a separate instance so
// that the codes-only kernel carries no registers for them.
template <int BITS, bool SIGNS, bool ROT>
__global__ void __launch_bounds__(kCT, 3) rq_chunk_mma_kernel(ChunkArgs a) {
  using T = Team<32>;
  constexpr float QMAX = (float)((1 << (BITS - 1)) - 1);
  constexpr int CB = BITS == 8 ? 128 : 64;  // code bytes per block
  extern __shared__ __align__(16) uint8_t smem[];
  const int tt = T::tid();
  const int g = tt >> 2, t4 = tt & 3;
  const uint2* s_sw = reinterpret_cast<const uint2*>(smem + 2 * chunk_stage_bytes());
  if constexpr (SIGNS) {
    load_mma_sign_words(a.signs, a.cpr, reinterpret_cast<uint2*>(smem + 2 * chunk_stage_bytes()));
    __syncthreads();
  }
  // column block of this warp's first slab block, advanced from slab to slab
  int colc = SIGNS ? (int)((T::first() * 32) % a.cpr) : 0;
  const int col_step = SIGNS ? (int)((T::stride() * 32) % a.cpr) : 0;

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
  // ldmatrix row of this lane: block (tt & 7) + 8 ((tt >> 3) & 1) of the
  // group, column half tt >> 4; tile p adds 32 bytes, group 1 adds 16 slots
  const uint32_t lm_off = uint32_t(((tt & 7) + 8 * ((tt >> 3) & 1)) * kCPad + (tt >> 4) * 16);

  const uint8_t* xsrc = reinterpret_cast<const uint8_t*>(a.x);
  const int64_t nslabs = (a.nchunks + 31) / 32;
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
      const int64_t n2 = nx + T::stride();  // the slab after: into L2 now, staged next iteration
      if (tt == 0 && n2 < nslabs) prefetch_l2_bulk(xsrc + n2 * 32 * 256, uint32_t(slab_count(n2 * 32, a.nchunks, 32)) * 256u);
    }
    const int nch = slab_count(c, a.nchunks, 32);  // blocks beyond nch hold stale data: computed, never stored
    // sign words of this lane's blocks g + 8 r + 16 grp (index 2 grp + r)
    uint2 sgw[4];
    if constexpr (SIGNS) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t cb = (uint32_t)(colc + g + 8 * i);  // i = 2 grp + r: block offset 16 grp + 8 r
        cb = a.cpr >= 32 ? (cb >= (uint32_t)a.cpr ? cb - a.cpr : cb) : cb % (uint32_t)a.cpr;
        sgw[i] = s_sw[cb * 4 + t4];
      }
      colc += col_step;
      if (colc >= a.cpr) colc -= a.cpr;
    }

    // 1. H_16 along q: u[64 grp + 8 p + 4 r + e] = output n = 4 t4 + e of row
    // p of block 16 grp + g + 8 r
    float u[128];
    const uint32_t cur_s = static_cast<uint32_t>(__cvta_generic_to_shared(cur));
#pragma unroll
    for (int grp = 0; grp < 2; ++grp) {
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(cur_s + lm_off + uint32_t(grp * 16 * kCPad + p * 32), a0, a1, a2, a3);
        if constexpr (SIGNS) {  // a0 / a2: block g (+16 grp), a1 / a3: block g + 8
          a0 ^= (sgw[2 * grp].x << p) & 0x80008000u;
          a1 ^= (sgw[2 * grp + 1].x << p) & 0x80008000u;
          a2 ^= (sgw[2 * grp].y << p) & 0x80008000u;
          a3 ^= (sgw[2 * grp + 1].y << p) & 0x80008000u;
        }
        float d0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, d1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        mma_bf16_k16(d0, a0, a1, a2, a3, hb[0][0], hb[0][1]);
        mma_bf16_k16(d1, a0, a1, a2, a3, hb[1][0], hb[1][1]);
        float* o = u + 64 * grp + 8 * p;
        o[0] = d0[0];
        o[1] = d0[1];
        o[2] = d1[0];
        o[3] = d1[1];
        o[4] = d0[2];
        o[5] = d0[3];
        o[6] = d1[2];
        o[7] = d1[3];
      }
    }
    // 2. H_8 along p
    reg_stage<128, 8>(u);
    reg_stage<128, 16>(u);
    reg_stage<128, 32>(u);
    __syncwarp();  // every lane has loaded its fragments: the slots take the codes

    // 3. per block: maximum, scale, codes
#pragma unroll
    for (int grp = 0; grp < 2; ++grp) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float* v = u + 64 * grp + 4 * r;  // v[8 p + e]
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
        const int b = 16 * grp + g + 8 * r;
        const bool live = b < nch;
        if (t4 == 0 && live) a.scales[c + b] = m * a.scale_mul;
        if constexpr (ROT) {
          if (live) {
            float* rr = a.rot + (c + b) * kCK + 4 * t4;
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
            *reinterpret_cast<uint32_t*>(slot + 16 * p + 4 * t4) = pack_i8x4(c0, c1, c2, c3);  // outputs 16 p + 4 t4 .. + 3
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
            const uint32_t wd = pack_i4x8(cc);
            *reinterpret_cast<uint16_t*>(slot + 8 * p + 2 * t4) = (uint16_t)(wd & 0xffffu);
            *reinterpret_cast<uint16_t*>(slot + 8 * p + 8 + 2 * t4) = (uint16_t)(wd >> 16);
          }
        }
      }
    }
    __syncwarp();
    chunk_store<CB / 16, 32>(cur, nch, a.codes + c * CB, tt);
  }
  cp_async_wait<0>();
}

}  // namespace hadq
