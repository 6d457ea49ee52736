// Forward 4096-point Hadamard blocks (one scale per block) with the first
// 16-point stage on tensor cores.
//
// H_4096 = H_16 (x) H_256 on the index split j = 16 p + q.  The signed bf16
// input is exact in bf16, and H_16 holds only +-1, so the transform along q
// is a bf16 GEMM with exact products: D[p][n] = sum_q x[p][q] H_16[q][n],
// one m16n8k16 mma.sync per 16 x 8 output tile with float32 accumulation.
// The remaining eight stages (along p) run as paired FP32 butterflies.
//
// One warp owns one 4096-column block (a slab of 32 chunks of 128 columns,
// staged in shared memory by cp.async as in the chunk kernels).  Per block:
//   1. 16 tiles of 16 p-rows: ldmatrix.x4 gives the A fragments (rows picked
//      so that the eight rows of every 8x8 load fall in different banks), the
//      sign vector is an XOR on the fragments (masks from a per-CTA table),
//      and two MMAs with H_16 give 8 outputs per lane and tile.  Lane (g, t4)
//      then holds output j' = 16 p + n with n bits 1-2 = t4, p bits 0, 1, 3 =
//      g, and the register index covering n bits 0 and 3, p bit 2 and the tile
//      (p bits 4-7): register u[8 T + 4 p2 + 2 n3 + n0].
//   2. Five register stages: output bits 6 and 8-11.
//   3. One transpose through the slab's shared memory, in two halves (output
//      bit 3 clear / set): each lane writes its 64 values of the half as one
//      row of 68 floats (128-bit stores), and reads 64-bit pairs across the
//      rows; both sides are conflict-free with one base address per lane.
//      Afterwards lane L holds bits 6 (L bit 0) and 8-11 (L bits 1-4) fixed
//      and register w[e + 8 c + 32 b7 + 64 h] for output bits 0-2 = e,
//      4-5 = c, 7 = b7, 3 = h.
//   4. Three register stages (output bits 4, 5, 7), the last fused with the
//      absolute maximum; a warp reduction gives the block maximum.
//   5. Codes of 4 (INT8) or 8 (INT4) consecutive outputs per word, written
//      into per-lane rows of the slab (odd pitch), then copied out in natural
//      order with coalesced 32-bit stores.
#pragma once

#include "hadq_chunk.cuh"
#include "hadq_mma.cuh"

namespace hadq {

constexpr int kH4096Warps = 6;                   // warps (blocks in flight) per CTA
constexpr int kH4096SignBytes = 16 * 32 * 16;    // sign masks: [tile][lane] x 4 words

__host__ __device__ inline size_t h4096_smem_bytes(bool signs) {
  return size_t(2) * kH4096Warps * 32 * kCPad + (signs ? size_t(kH4096SignBytes) : 0);
}

// p-row of MMA row m (0..15) in tile T: rows 0-7 take p = 16 T + {0, 1, 2, 3,
// 8, 9, 10, 11} and rows 8-15 the same + 4, so that the eight 32-byte rows of
// one 8x8 load span two chunk slots and eight different 16-byte bank groups.
__host__ __device__ inline int h4096_p(int T, int m) { return 16 * T + (m & 3) + 8 * ((m >> 2) & 1) + 4 * (m >> 3); }

// Eight rotated outputs (normalised by rsqrt_b) to global memory.
__device__ __forceinline__ void rot_run8(float* d, const float* s, float r) {
  reinterpret_cast<float4*>(d)[0] = make_float4(s[0] * r, s[1] * r, s[2] * r, s[3] * r);
  reinterpret_cast<float4*>(d)[1] = make_float4(s[4] * r, s[5] * r, s[6] * r, s[7] * r);
}

// ROT: also write the rotated float32 values (a.rot); a separate instance so
// that the codes-only kernel carries no registers for them.
template <int BITS, bool SIGNS, bool ROT>
__global__ void __launch_bounds__(kH4096Warps * 32, 2) rq_h4096_mma_kernel(ChunkArgs a) {
  constexpr float QMAX = (float)((1 << (BITS - 1)) - 1);
  extern __shared__ __align__(16) uint8_t smem[];
  uint4* s_sm = reinterpret_cast<uint4*>(smem + size_t(2) * kH4096Warps * 32 * kCPad);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int g = lane >> 2, t4 = lane & 3;

  if constexpr (SIGNS) {
    // mask words of lane l's four A registers in tile T: pairs at columns
    // 2 t4 (+1) and 2 t4 + 8 (+1) of p-rows h4096_p(T, g) and h4096_p(T, g + 8)
    for (int e = threadIdx.x; e < 16 * 32; e += blockDim.x) {
      const int tile = e >> 5, l = e & 31, gg = l >> 2, c = 2 * (l & 3);
      const int j0 = 16 * h4096_p(tile, gg) + c, j1 = 16 * h4096_p(tile, gg + 8) + c;
      auto mk = [&](int j) {
        return (a.signs[j] < 0 ? 0x8000u : 0u) | (a.signs[j + 1] < 0 ? 0x80000000u : 0u);
      };
      s_sm[e] = make_uint4(mk(j0), mk(j1), mk(j0 + 8), mk(j1 + 8));
    }
    __syncthreads();
  }

  // B fragments of H_16 (bf16 +-1): n-tile nt, k half kh: {H[k][n], H[k + 1][n]}
  // with k = 2 t4 + 8 kh, n = g + 8 nt
  uint32_t hb[2][2];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
    for (int kh = 0; kh < 2; ++kh) {
      const int k = 2 * t4 + 8 * kh, n = g + 8 * nt;
      const uint32_t lo = (__popc(k & n) & 1) ? 0xBF80u : 0x3F80u;
      const uint32_t hi = (__popc((k + 1) & n) & 1) ? 0xBF80u : 0x3F80u;
      hb[nt][kh] = lo | (hi << 16);
    }
  }

  // this lane's ldmatrix row inside tile 0 (tile T adds 2 T chunk slots)
  const int lmi = lane >> 3, lr = lane & 7;
  const int lp = h4096_p(0, lr + 8 * (lmi & 1));
  const uint32_t lm_off = uint32_t((lp >> 3) * kCPad + (lp & 7) * 32 + (lmi >> 1) * 16);
  // this lane's fixed output bits after the transpose
  const int b6 = lane & 1, tp = lane >> 1;

  const uint8_t* xsrc = reinterpret_cast<const uint8_t*>(a.x);
  const int64_t nslabs = a.nchunks / 32;
  uint8_t* st0 = smem + (wid * 2 + 0) * 32 * kCPad;
  uint8_t* st1 = smem + (wid * 2 + 1) * 32 * kCPad;
  const int64_t wstride = int64_t(gridDim.x) * (blockDim.x >> 5);

  int64_t slab = int64_t(blockIdx.x) * (blockDim.x >> 5) + wid;
  if (slab < nslabs) chunk_load<16, 32>(xsrc + slab * 32 * 256, 32, st0, lane);
  cp_async_commit();
  for (int it = 0; slab < nslabs; ++it, slab += wstride) {
    uint8_t* cur = (it & 1) ? st1 : st0;
    cp_async_wait<0>();
    __syncwarp();
    {
      const int64_t nx = slab + wstride;
      if (nx < nslabs) chunk_load<16, 32>(xsrc + nx * 32 * 256, 32, (it & 1) ? st0 : st1, lane);
      cp_async_commit();
      const int64_t n2 = nx + wstride;  // the block after: into L2 now, staged next iteration
      if (lane == 0 && n2 < nslabs) prefetch_l2_bulk(xsrc + n2 * 32 * 256, 8192u);
    }

    // 1. H_16 along q on tensor cores
    float u[128];
    const uint32_t cur_s = static_cast<uint32_t>(__cvta_generic_to_shared(cur));
#pragma unroll
    for (int T = 0; T < 16; ++T) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(cur_s + lm_off + uint32_t(T * 2 * kCPad), a0, a1, a2, a3);
      if constexpr (SIGNS) {
        const uint4 sm = s_sm[T * 32 + lane];
        a0 ^= sm.x;
        a1 ^= sm.y;
        a2 ^= sm.z;
        a3 ^= sm.w;
      }
      float d0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, d1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      mma_bf16_k16(d0, a0, a1, a2, a3, hb[0][0], hb[0][1]);
      mma_bf16_k16(d1, a0, a1, a2, a3, hb[1][0], hb[1][1]);
      u[8 * T + 0] = d0[0];
      u[8 * T + 1] = d0[1];
      u[8 * T + 4] = d0[2];
      u[8 * T + 5] = d0[3];
      u[8 * T + 2] = d1[0];
      u[8 * T + 3] = d1[1];
      u[8 * T + 6] = d1[2];
      u[8 * T + 7] = d1[3];
    }
    // 2. output bits 6 (p2) and 8-11 (tile)
    reg_stage<128, 4>(u);
    reg_stage<128, 8>(u);
    reg_stage<128, 16>(u);
    reg_stage<128, 32>(u);
    reg_stage<128, 64>(u);

    // 3. transpose through the slab, output bit 3 clear, then set.  Writer
    // lane (t4, g) puts register (n0, p2, T) at row lane, column n0 + 2 p2 +
    // 4 T; the value of output (e, c, b7, b6, tp) sits in row (e >> 1) + 4 c +
    // 16 b7, column (e & 1) + 2 b6 + 4 tp.
    float w[128];
    float* xs = reinterpret_cast<float*>(cur);
    float* wrow = xs + lane * 68;
    const float* rcol = xs + 2 * b6 + 4 * tp;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      __syncwarp();  // the slab is free (fragments loaded / previous half read)
#pragma unroll
      for (int T = 0; T < 16; ++T)
        *reinterpret_cast<float4*>(wrow + 4 * T) =
            make_float4(u[8 * T + 2 * h], u[8 * T + 2 * h + 1], u[8 * T + 4 + 2 * h], u[8 * T + 5 + 2 * h]);
      __syncwarp();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int b7 = 0; b7 < 2; ++b7) {
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const float2 f = *reinterpret_cast<const float2*>(rcol + (e2 + 4 * c + 16 * b7) * 68);
            w[2 * e2 + 8 * c + 32 * b7 + 64 * h] = f.x;
            w[2 * e2 + 1 + 8 * c + 32 * b7 + 64 * h] = f.y;
          }
        }
      }
    }
    __syncwarp();  // every lane has read the transpose: the slab now takes the codes
    // 4. output bits 4, 5 and 7, then the block maximum
    reg_stage<128, 8>(w);
    reg_stage<128, 16>(w);
    float m = reg_stage_absmax<128, 32>(w);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) a.scales[slab] = m * a.scale_mul;
    // 5. codes of runs of 8 consecutive outputs (register block w + 8 c +
    // 32 b7 + 64 h) into per-lane rows, then out in natural order
    const QInv q = make_qinv(m, QMAX);
    float* rr = ROT ? a.rot + slab * 4096 + 64 * b6 + 256 * tp : nullptr;
    float pre = 1.0f;  // blocks with a tiny maximum take their codes at 2^64 scale (exact)
    if (q.tiny) {
      pre = 18446744073709551616.0f;
#pragma unroll
      for (int i = 0; i < 128; ++i) w[i] *= pre;
    }
    uint32_t* cw = reinterpret_cast<uint32_t*>(cur);
    if constexpr (BITS == 8) {
      // word r = (e >> 2) + 2 h + 4 c + 16 b7 of lane L: row L, pitch 33;
      // natural word index (e >> 2) + 2 h + 4 c + 16 b6 + 32 b7 + 64 tp
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int b7 = 0; b7 < 2; ++b7) {
            const float* s = w + 8 * c + 32 * b7 + 64 * h;
            if constexpr (ROT) rot_run8(rr + 8 * h + 16 * c + 128 * b7, s, a.rsqrt_b / pre);
            uint32_t cc[8];
            magic_code2(s[0], s[1], q.inv, cc[0], cc[1]);
            magic_code2(s[2], s[3], q.inv, cc[2], cc[3]);
            magic_code2(s[4], s[5], q.inv, cc[4], cc[5]);
            magic_code2(s[6], s[7], q.inv, cc[6], cc[7]);
            cw[lane * 33 + 2 * h + 4 * c + 16 * b7] = pack_i8x4(cc[0], cc[1], cc[2], cc[3]);
            cw[lane * 33 + 1 + 2 * h + 4 * c + 16 * b7] = pack_i8x4(cc[4], cc[5], cc[6], cc[7]);
          }
      __syncwarp();
      uint32_t* dst = reinterpret_cast<uint32_t*>(a.codes + slab * 4096);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int wi = lane + 32 * i;
        const int L = ((wi >> 4) & 1) + 2 * (wi >> 6), r = (wi & 15) + 16 * ((wi >> 5) & 1);
        dst[wi] = cw[L * 33 + r];
      }
    } else {
      // word r = h + 2 c + 8 b7 of lane L: row L, pitch 17; natural word index
      // h + 2 c + 8 b6 + 16 b7 + 32 tp
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int b7 = 0; b7 < 2; ++b7) {
            const float* s = w + 8 * c + 32 * b7 + 64 * h;
            if constexpr (ROT) rot_run8(rr + 8 * h + 16 * c + 128 * b7, s, a.rsqrt_b / pre);
            uint32_t cc[8];
            magic_code2(s[0], s[1], q.inv, cc[0], cc[1]);
            magic_code2(s[2], s[3], q.inv, cc[2], cc[3]);
            magic_code2(s[4], s[5], q.inv, cc[4], cc[5]);
            magic_code2(s[6], s[7], q.inv, cc[6], cc[7]);
            cw[lane * 17 + h + 2 * c + 8 * b7] = pack_i4x8(cc);
          }
      __syncwarp();
      uint32_t* dst = reinterpret_cast<uint32_t*>(a.codes + slab * 2048);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int wi = lane + 32 * i;
        const int L = ((wi >> 3) & 1) + 2 * (wi >> 5), r = (wi & 7) + 8 * ((wi >> 4) & 1);
        dst[wi] = cw[L * 17 + r];
      }
    }
  }
  cp_async_wait<0>();
}

}  // namespace hadq
