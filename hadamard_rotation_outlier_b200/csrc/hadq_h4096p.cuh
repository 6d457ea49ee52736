// Forward 4096-point Hadamard blocks (one scale per block) on warp pairs:
// two warps per block, 64 values per lane, the first 16-point stage on tensor
// cores.
//
// Element j of a block has 12 index bits.  Tile T = j >> 8 (bits 8-11) holds
// 256 consecutive elements; warp w of the pair takes the tiles with T bit 3 =
// w (j11), so a lane owns eight tiles t = T & 7 (bits 8-10).
//
// 1. Load.  A lane copies 16 bytes per tile into the pair's staging buffer
//    (cp.async) and reads them back into registers: elements o = 8 lane + e
//    (e = 0..7) of the tile, o = 32 g + 8 t4 + e.  Those 8 bf16 values are
//    exactly the lane's A fragment of one
//    m16n8k16 MMA when the tile is a 16 x 16 matrix with rows m = g + 8 e2 and
//    columns k = 2 t4 + e0 + 8 e1: bits j0, j1, j3, j4 are the MMA's k (the
//    "q" bits it transforms), j2 and j5-j7 its rows.  A lane stages only its
//    own pieces, so the staging needs no barrier: the next block's copy is
//    issued as soon as this block's pieces went through the MMAs, and the
//    block after that is prefetched into L2 with one bulk prefetch.
// 2. Signs.  The element signs flip bf16 sign bits: an XOR on the fragments
//    (the products stay exact).  Each lane's 64 sign bits are two words built
//    once per CTA; the mask of register r of tile t is (word << i) &
//    0x80008000 with i = 4 (t & 3) + r.
// 3. H_16 over the q bits: two MMAs against +-1 B fragments whose rows and
//    columns are ordered so that lane (g, t4) receives outputs j0, j1 in its
//    registers and j3, j4 = t4.  Values: u[8 t + 4 j2 + 2 j1 + j0].
// 4. Register stages over j2, j8, j9, j10.
// 5. Transpose through the pair's 16 KB float buffer: each lane writes its
//    values as 16-byte runs (j0, j1) at position j, reads back 16-byte runs
//    with lane bits = (j2, j3, j4, j8, j9), warp = j10 and registers =
//    (j5, j6, j7, j11); the 16-byte unit index is swizzled (bit 0 ^= j5) so
//    both sides are free of bank conflicts.  One pair barrier.
// 6. Register stages over j5, j6, j7, j11, the last fused with max |y|; warp
//    maximum by shuffles, pair maximum through shared memory (second pair
//    barrier, which also frees the buffer for the next block).
// 7. Codes: four consecutive outputs per run, INT8 as one 32-bit store per
//    run, INT4 as one 16-bit store per run (the L2 merges the runs of a
//    sector).
#pragma once

#include "hadq_chunk.cuh"
#include "hadq_mma.cuh"

namespace hadq {

constexpr int kH4PairsPerCta = 2;              // warp pairs (blocks in flight) per CTA
constexpr int kH4PairFloats = 4096 + 8 + 2048;  // transpose buffer, two pairs of max slots, staging (8 KB)

__host__ __device__ inline size_t h4096p_smem_bytes() { return size_t(kH4PairsPerCta) * kH4PairFloats * sizeof(float); }

__device__ __forceinline__ void pair_sync(int id) { asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory"); }

// k-slot and output-column Q values (Q bits j0, j1, j3, j4, lowest first):
// slot k = 2 t4 + 8 kh + pair holds j0 = pair, j1 = kh, (j3, j4) = t4;
// column n = 8 nt + 2 t4 + e holds j0 = e, j1 = nt, (j3, j4) = t4.
__device__ __forceinline__ int h4p_qin(int k) { return (k & 1) | (((k >> 3) & 1) << 1) | (((k >> 1) & 3) << 2); }
__device__ __forceinline__ int h4p_qout(int n) { return (n & 1) | (((n >> 3) & 1) << 1) | (((n >> 1) & 3) << 2); }

template <int BITS, bool SIGNS, bool ROT>
__global__ void __launch_bounds__(kH4PairsPerCta * 64, 4) rq_h4096_pair_kernel(ChunkArgs a) {
  constexpr float QMAX = (float)((1 << (BITS - 1)) - 1);
  extern __shared__ __align__(16) float psm[];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int pair = wid >> 1, w = wid & 1;
  const int g = lane >> 2, t4 = lane & 3;
  float* buf = psm + pair * kH4PairFloats;
  float* pmax = buf + 4096;  // [parity][warp]
  const int bar = 1 + pair;

  // sign words: word h covers tiles t = 4 h .. 4 h + 3; register r of tile t
  // (a0: e 0-1, a1: e 4-5, a2: e 2-3, a3: e 6-7) at i = 4 (t & 3) + r
  uint32_t sw[2] = {0u, 0u};
  if constexpr (SIGNS) {
#pragma unroll 1
    for (int t = 0; t < 8; ++t) {
      const int jt = 256 * (8 * w + t) + 8 * lane;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int e = r == 0 ? 0 : r == 1 ? 4 : r == 2 ? 2 : 6;
        const int i = 4 * (t & 3) + r;
        sw[t >> 2] |= (uint32_t)(a.signs[jt + e] < 0) << (15 - i) | (uint32_t)(a.signs[jt + e + 1] < 0) << (31 - i);
      }
    }
  }
  // B fragments: +-1 (bf16) entries between slot and column Q values
  uint32_t hb[2][2];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
    for (int kh = 0; kh < 2; ++kh) {
      const int k = 2 * t4 + 8 * kh, n = g + 8 * nt;
      const uint32_t lo = (__popc(h4p_qin(k) & h4p_qout(n)) & 1) ? 0xBF80u : 0x3F80u;
      const uint32_t hi = (__popc(h4p_qin(k + 1) & h4p_qout(n)) & 1) ? 0xBF80u : 0x3F80u;
      hb[nt][kh] = lo | (hi << 16);
    }
  }
  // transpose addresses (floats): write run (t, j2) of this lane at
  // 4 (j2 ^ j5) + 8 t4 + 32 g + 256 t + 2048 w with j5 = g & 1; read run r =
  // (j5, j6, j7, j11) at 4 (l0 ^ j5) + 8 l1 + 16 l2 + 256 l3 + 512 l4 + 1024 w
  // + 32 j5 + 64 j6 + 128 j7 + 2048 j11 (lane bits l0..l4)
  const int wr_base = 8 * t4 + 32 * g + 2048 * w;
  const int wr_sw = 4 * (g & 1);
  const int l0 = lane & 1;
  const int rd_base = 8 * ((lane >> 1) & 1) + 16 * ((lane >> 2) & 1) + 256 * ((lane >> 3) & 1) + 512 * (lane >> 4) + 1024 * w;
  // this lane's output runs after the transpose: j = 4 l0 + rd_base + 32 j5 + ... (no swizzle)
  const int out_base = 4 * l0 + rd_base;

  const int64_t nblk = a.nchunks / 32;  // 4096-column blocks
  const int64_t pstride = int64_t(gridDim.x) * kH4PairsPerCta;
  const uint16_t* x = a.x;
  int parity = 0;
  int64_t blk = int64_t(blockIdx.x) * kH4PairsPerCta + pair;
  // staging: a lane's 16-byte piece of tile t of the pair's block sits at
  // uint4 index 256 w + 32 t + lane (the piece's own offset in the block);
  // each lane copies in and reads back only its own pieces, so no barrier
  uint4* stg = reinterpret_cast<uint4*>(buf + 4096 + 8) + 256 * w + lane;
  auto stage_in = [&](int64_t k) {
    const uint4* src = reinterpret_cast<const uint4*>(x + k * 4096 + 2048 * w) + lane;
#pragma unroll
    for (int t = 0; t < 8; ++t) cp_async16(stg + 32 * t, src + 32 * t);
  };
  if (blk < nblk) stage_in(blk);
  cp_async_commit();
  if (w == 0 && lane == 0 && blk + pstride < nblk) prefetch_l2_bulk(x + (blk + pstride) * 4096, 8192);
  for (; blk < nblk; blk += pstride, parity ^= 1) {
    // the block after the next one into L2 (it is staged during the next block)
    if (w == 0 && lane == 0 && blk + 2 * pstride < nblk) prefetch_l2_bulk(x + (blk + 2 * pstride) * 4096, 8192);
    cp_async_wait<0>();
    // 1-3. signs, H_16 on tensor cores
    float u[64];
    {
      uint4 f[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) f[t] = stg[32 * t];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        uint32_t a0 = f[t].x, a2 = f[t].y, a1 = f[t].z, a3 = f[t].w;
        if constexpr (SIGNS) {
          const uint32_t s = sw[t >> 2];
          const int i = 4 * (t & 3);
          a0 ^= (s << i) & 0x80008000u;
          a1 ^= (s << (i + 1)) & 0x80008000u;
          a2 ^= (s << (i + 2)) & 0x80008000u;
          a3 ^= (s << (i + 3)) & 0x80008000u;
        }
        float d0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, d1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        mma_bf16_k16(d0, a0, a1, a2, a3, hb[0][0], hb[0][1]);
        mma_bf16_k16(d1, a0, a1, a2, a3, hb[1][0], hb[1][1]);
        u[8 * t + 0] = d0[0];
        u[8 * t + 1] = d0[1];
        u[8 * t + 2] = d1[0];
        u[8 * t + 3] = d1[1];
        u[8 * t + 4] = d0[2];
        u[8 * t + 5] = d0[3];
        u[8 * t + 6] = d1[2];
        u[8 * t + 7] = d1[3];
      }
    }
    // the MMAs have consumed this lane's pieces: its slots take the next block
    if (blk + pstride < nblk) stage_in(blk + pstride);
    cp_async_commit();
    // 4. j2, j8, j9, j10
    reg_stage<64, 4>(u);
    reg_stage<64, 8>(u);
    reg_stage<64, 16>(u);
    reg_stage<64, 32>(u);
    // 5. transpose through the pair's buffer
#pragma unroll
    for (int t = 0; t < 8; ++t) {
#pragma unroll
      for (int j2 = 0; j2 < 2; ++j2)
        *reinterpret_cast<float4*>(buf + ((4 * j2) ^ wr_sw) + wr_base + 256 * t) =
            make_float4(u[8 * t + 4 * j2], u[8 * t + 4 * j2 + 1], u[8 * t + 4 * j2 + 2], u[8 * t + 4 * j2 + 3]);
    }
    pair_sync(bar);
    float v[64];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      const int j5 = r & 1;
      const float4 q = *reinterpret_cast<const float4*>(buf + ((4 * l0) ^ (4 * j5)) + rd_base + 32 * (r & 7) +
                                                        2048 * (r >> 3));
      v[4 * r] = q.x;
      v[4 * r + 1] = q.y;
      v[4 * r + 2] = q.z;
      v[4 * r + 3] = q.w;
    }
    // 6. j5, j6, j7, j11; block maximum
    reg_stage<64, 4>(v);
    reg_stage<64, 8>(v);
    reg_stage<64, 16>(v);
    float m = reg_stage_absmax<64, 32>(v);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) pmax[2 * parity + w] = m;
    pair_sync(bar);
    m = fmaxf(pmax[2 * parity], pmax[2 * parity + 1]);
    if (w == 0 && lane == 0) a.scales[blk] = m * a.scale_mul;
    // 7. codes
    const QInv q = make_qinv(m, QMAX);
    float pre = 1.0f;  // blocks with a tiny maximum take their codes at 2^64 scale (exact)
    if (q.tiny) {
      pre = 18446744073709551616.0f;
#pragma unroll
      for (int i = 0; i < 64; ++i) v[i] *= pre;
    }
#pragma unroll
    for (int r = 0; r < 16; r += 2) {
      // runs r and r + 1 (j5 = 0, 1): first outputs j = out_base + 32 (r & 7) + 2048 (r >> 3)
      const int ja = out_base + 32 * (r & 7) + 2048 * (r >> 3);
      const int jb = ja + 32;
      uint32_t cc[8];
      magic_code2(v[4 * r], v[4 * r + 1], q.inv, cc[0], cc[1]);
      magic_code2(v[4 * r + 2], v[4 * r + 3], q.inv, cc[2], cc[3]);
      magic_code2(v[4 * r + 4], v[4 * r + 5], q.inv, cc[4], cc[5]);
      magic_code2(v[4 * r + 6], v[4 * r + 7], q.inv, cc[6], cc[7]);
      if constexpr (ROT) {
        const float s = a.rsqrt_b / pre;
        float* rr = a.rot + blk * 4096;
        *reinterpret_cast<float4*>(rr + ja) = make_float4(v[4 * r] * s, v[4 * r + 1] * s, v[4 * r + 2] * s, v[4 * r + 3] * s);
        *reinterpret_cast<float4*>(rr + jb) =
            make_float4(v[4 * r + 4] * s, v[4 * r + 5] * s, v[4 * r + 6] * s, v[4 * r + 7] * s);
      }
      if constexpr (BITS == 8) {
        uint8_t* cdst = a.codes + blk * 4096;
        *reinterpret_cast<uint32_t*>(cdst + ja) = pack_i8x4(cc[0], cc[1], cc[2], cc[3]);
        *reinterpret_cast<uint32_t*>(cdst + jb) = pack_i8x4(cc[4], cc[5], cc[6], cc[7]);
      } else {
        const uint32_t wd = pack_i4x8(cc);  // low half: run r, high half: run r + 1
        uint8_t* cdst = a.codes + blk * 2048;
        *reinterpret_cast<uint16_t*>(cdst + ja / 2) = (uint16_t)(wd & 0xffffu);
        *reinterpret_cast<uint16_t*>(cdst + jb / 2) = (uint16_t)(wd >> 16);
      }
    }
  }
}

}  // namespace hadq
