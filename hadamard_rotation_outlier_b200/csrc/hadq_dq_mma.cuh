// Inverse of 128-point Hadamard blocks (dequantise + inverse rotation) with
// the first 16-point stage on tensor cores: blocks of B = 128 whose scale
// group covers whole blocks (G a multiple of 128), INT4 or INT8 codes.
//
// The codes are integers, and an f16 value 1024 + u (0 <= u < 1024) has the
// bit pattern 0x6400 | u, so a biased code becomes an exact f16 operand with
// one three-input logic operation.  H_128 = H_8 (x) H_16 on a split of the
// code index into four "q" bits (transformed by one m16n8k16 f16 MMA with
// float32 accumulation: integer products and sums, exact) and three "p" bits
// (three register stages, still on integers).  The scale is applied once at
// the end, as in the chunk dequantiser, so the results are the same numbers.
//
// One MMA tile takes 16 blocks of a slab (rows) and the 16 q-values of one
// p-value (columns).  The codes of a slab (32 consecutive blocks) are staged
// in shared memory by cp.async, three stages per warp, and the slab after the
// last staged one is prefetched into L2; ldmatrix.x4 over 16-byte segments of the code
// rows hands each lane 4 bytes of a segment of two blocks, and the choice of
// which code bits are q bits follows what a lane receives:
//
//   INT4 (32 codes per segment): a lane (g, t4) holds codes
//        j = 32 s + 8 t4 + 2 i + nib of blocks g and g + 8.  Register
//        (word & 0x000F000F) pairs bytes 0 and 2 (low nibbles), (word &
//        0x00F000F0) the high nibbles at 16 times their value, and the same
//        for bytes 1 and 3 after a shift: q bits j2 (pair), j3, j4 (t4) and
//        j0 (nibble, rows of B scaled by 1/16); p bits j1 and j5, j6.
//   INT8 (16 codes per segment): codes j = 16 s + 4 t4 + i; a byte permute
//        makes pairs (i = 0, 1) and (2, 3): q bits j0 (pair), j2, j3 (t4), j1;
//        p bits j4..j6.
//
// The codes enter with a bias (u = code + 2^(b-1), plus 1024 from the f16
// pattern); its contribution to the MMA is a constant per output column,
// taken out by starting the accumulators at minus that constant.  The columns
// of H_16 in the B fragments are ordered so that a lane ends up with runs of
// consecutive outputs (8 for INT4, 4 for INT8): with the three p stages in
// registers, each run is converted to bf16, gets its signs, and goes to a
// per-warp staging area laid out as the slab is in global memory (8 KB of
// bf16 rows), which leaves with one bulk asynchronous copy issued by one lane
// (no per-lane copy-out; the copy engine reads the staging while the warp
// computes the next slab, and the lane waits for that read before the rows
// are written again).
#pragma once

#include "hadq_chunk.cuh"
#include "hadq_mma.cuh"

namespace hadq {

template <int BITS>
struct DqMmaLayout {
  static constexpr int CB = BITS == 8 ? 128 : 64;    // code bytes per block
  static constexpr int CP = CB + 16;                 // code row pitch (ldmatrix rows conflict-free)
  static constexpr int OP = 256;                     // bf16 output rows: the slab's global layout
  static constexpr int NS = 3;                       // code stages per warp (plus the L2 prefetch)
  static constexpr int WARP_BYTES = NS * 32 * CP + 32 * OP;
};

__host__ __device__ inline size_t dq_mma_smem_bytes(int bits, int dim, bool signs) {
  const size_t w = bits == 8 ? DqMmaLayout<8>::WARP_BYTES : DqMmaLayout<4>::WARP_BYTES;
  return (kCT / 32) * w + (signs ? size_t(kSignTabBytes + sign_bits_bytes(dim)) : 0);
}

__device__ __forceinline__ void mma_f16_k16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Q-space value (bits in the order of the q bits listed above, lowest first)
// of MMA k-slot k and of output column n.  INT4: Q = (j0, j2, j3, j4), k bit
// 0 -> j2, bits 1-2 -> j3, j4, bit 3 -> j0.  INT8: Q = (j0, j1, j2, j3), k bit 0
// -> j0, bits 1-2 -> j2, j3, bit 3 -> j1.  Column n = 8 nt + 2 t4 + e carries
// Q value e + 2 nt + 4 t4 (both widths).
template <int BITS>
__device__ __forceinline__ int dq_qin(int k) {
  const int k0 = k & 1, k12 = (k >> 1) & 3, k3 = (k >> 3) & 1;
  return BITS == 4 ? (k3 | (k0 << 1) | (k12 << 2)) : (k0 | (k3 << 1) | (k12 << 2));
}
__device__ __forceinline__ int dq_qout(int n) { return (n & 1) | (((n >> 3) & 1) << 1) | (((n >> 1) & 3) << 2); }

// Bias of output column n: sum over k of (operand bias of k-slot k) x B[k][n],
// with operand 1024 + u = 1024 + 2^(b-1) + code; INT4 rows of the high nibble
// carry 16 (1024 + u) at weight 1/16.
template <int BITS>
__device__ __forceinline__ float dq_bias(int n) {
  float b = 0.0f;
  const int qo = dq_qout(n);
#pragma unroll 1
  for (int k = 0; k < 16; ++k) {
    const float h = (__popc(dq_qin<BITS>(k) & qo) & 1) ? -1.0f : 1.0f;
    const float off = BITS == 4 ? ((k >> 3) ? 64.0f + 8.0f : 1024.0f + 8.0f) : 1024.0f + 128.0f;
    b += off * h;
  }
  return b;
}

// Codes of `nch` blocks from global memory into code rows of pitch CP.
template <int BITS>
__device__ __forceinline__ void dq_mma_load(const uint8_t* src, int nch, uint8_t* dst, int lane) {
  using L = DqMmaLayout<BITS>;
  constexpr int PPC = L::CB / 16;
  if (nch == 32) {
#pragma unroll
    for (int i = 0; i < PPC; ++i) {
      const int p = lane + 32 * i;
      cp_async16(dst + (p / PPC) * L::CP + 16 * (p % PPC), src + 16 * p);
    }
  } else {
    for (int p = lane; p < nch * PPC; p += 32) cp_async16(dst + (p / PPC) * L::CP + 16 * (p % PPC), src + 16 * p);
  }
}

template <int BITS, bool SIGNS, bool OUT_F32>
__global__ void __launch_bounds__(kCT, 3) dq_chunk_mma_kernel(ChunkArgs a) {
  using L = DqMmaLayout<BITS>;
  constexpr int RUN = BITS == 4 ? 8 : 4;      // consecutive outputs per lane and p
  constexpr int NP = BITS == 4 ? 4 : 8;       // runs (segment positions) per block
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  uint8_t* wbase = smem + size_t(wid) * L::WARP_BYTES;
  uint8_t* ostage = wbase + L::NS * 32 * L::CP;
  uint4* s_tab = reinterpret_cast<uint4*>(smem + (kCT / 32) * L::WARP_BYTES);
  const uint8_t* s_bytes = smem + (kCT / 32) * L::WARP_BYTES + kSignTabBytes;

  // B fragments: H_16 entries between k-slot and column Q values (INT4:
  // high-nibble rows at 1/16), as f16 pairs {B[k][n], B[k + 1][n]} with
  // k = 2 t4 + 8 kh, n = g + 8 nt; accumulators start at minus the bias.
  uint32_t hb[2][2];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const int n = g + 8 * nt;
#pragma unroll
    for (int kh = 0; kh < 2; ++kh) {
      const int k = 2 * t4 + 8 * kh;
      const uint32_t mag = (BITS == 4 && kh) ? 0x2C00u : 0x3C00u;  // 1/16 or 1
      const uint32_t lo = mag | ((__popc(dq_qin<BITS>(k) & dq_qout(n)) & 1) << 15);
      const uint32_t hi = mag | ((__popc(dq_qin<BITS>(k + 1) & dq_qout(n)) & 1) << 15);
      hb[nt][kh] = lo | (hi << 16);
    }
  }
  // accumulator start values: minus the bias of this lane's columns 8 nt + 2 t4 + e
  const float nb00 = -dq_bias<BITS>(2 * t4), nb01 = -dq_bias<BITS>(2 * t4 + 1);
  const float nb10 = -dq_bias<BITS>(8 + 2 * t4), nb11 = -dq_bias<BITS>(8 + 2 * t4 + 1);

  // ldmatrix row of this lane: block (lane & 7) + 8 ((lane >> 3) & 1) of a
  // group of 16, segment + (lane >> 4)
  const uint32_t lm_off = uint32_t(((lane & 7) + 8 * ((lane >> 3) & 1)) * L::CP + (lane >> 4) * 16);

  // Slab and chunk indices are 32-bit: the host takes this kernel only for
  // fewer than 2^30 chunks, so every index below, including the slabs staged
  // ahead, stays under 2^31.  Byte offsets are widened.
  const int nslabs = int((a.nchunks + 31) / 32);
  const int wstride = int(gridDim.x) * (kCT / 32);
  int slab = int(blockIdx.x) * (kCT / 32) + wid;
  int colc = SIGNS ? (int)((slab * 32) % a.cpr) : 0;
  const int col_step = SIGNS ? (int)((wstride * 32) % a.cpr) : 0;
  auto block_scale = [&](int blk) {
    return blk < a.nchunks ? __ldg(a.scales_in + (a.gpc == 1 ? blk : blk / a.gpc)) : 0.0f;
  };
  // prologue: the first NS - 1 slabs of this warp in flight, the scales of the first
#pragma unroll
  for (int k = 0; k < L::NS - 1; ++k) {
    const int sk = slab + k * wstride;
    if (sk < nslabs) dq_mma_load<BITS>(a.codes_in + size_t(sk) * (32 * L::CB), slab_count(sk * 32, a.nchunks, 32), wbase + k * 32 * L::CP, lane);
    cp_async_commit();
  }
  // the sign tables are built while those copies are in flight
  if constexpr (SIGNS) {
    load_sign_tables(a.signs, a.dim, s_tab, reinterpret_cast<uint32_t*>(smem + (kCT / 32) * L::WARP_BYTES + kSignTabBytes));
    __syncthreads();
  }
  float sc_next[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) sc_next[i] = slab < nslabs ? block_scale(slab * 32 + g + 8 * i) : 0.0f;
  for (int it = 0; slab < nslabs; ++it, slab += wstride) {
    uint8_t* cur = wbase + (it % L::NS) * 32 * L::CP;
    const int c = slab * 32;
    float sc[4];  // scales of this lane's blocks g + 8 i (i = 2 grp + r)
#pragma unroll
    for (int i = 0; i < 4; ++i) sc[i] = sc_next[i];
    cp_async_wait<L::NS - 2>();  // this slab's group has landed (one group per slab, empty ones included)
    __syncwarp();
    {
      // the stage read in the previous iteration takes the slab NS - 1 ahead
      const int nf = slab + (L::NS - 1) * wstride;
      if (nf < nslabs)
        dq_mma_load<BITS>(a.codes_in + size_t(nf) * (32 * L::CB), slab_count(nf * 32, a.nchunks, 32),
                          wbase + ((it + L::NS - 1) % L::NS) * 32 * L::CP, lane);
      cp_async_commit();
      const int n2 = nf + wstride;  // the slab after: into L2 now, staged next iteration
      if (lane == 0 && n2 < nslabs)
        prefetch_l2_bulk(a.codes_in + size_t(n2) * (32 * L::CB), uint32_t(slab_count(n2 * 32, a.nchunks, 32)) * L::CB);
      const int nx = slab + wstride;
#pragma unroll
      for (int i = 0; i < 4; ++i) sc_next[i] = nx < nslabs ? block_scale(nx * 32 + g + 8 * i) : 0.0f;
    }
    const int nch = slab_count(c, a.nchunks, 32);

    // Per group of 16 blocks (lane blocks g + 16 grp and g + 8 + 16 grp):
    // 1. the q bits on tensor cores: u[32 r + RUN s + local], local = position
    //    inside the lane's run of outputs at segment s;
    // 2. the p bits in registers (exact integer sums);
    // 3. scale, signs, bf16 runs into the staging rows (or float32 out).
#pragma unroll 1
    for (int grp = 0; grp < 2; ++grp) {
      float u[64];
      const uint32_t cur_s = static_cast<uint32_t>(__cvta_generic_to_shared(cur));
#pragma unroll
      for (int sp = 0; sp < NP; sp += 2) {
        uint32_t r0, r1, r2, r3;  // blocks g / g + 8 at segments sp, sp + 1
        ldsm_x4(cur_s + lm_off + uint32_t(grp * 16 * L::CP + sp * 16), r0, r1, r2, r3);
        const uint32_t rr[2][2] = {{r0, r1}, {r2, r3}};  // [segment][row half]
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int s = sp + h;
          if constexpr (BITS == 4) {
#pragma unroll
            for (int pb = 0; pb < 2; ++pb) {
              const uint32_t wg = pb ? (rr[h][0] >> 8) : rr[h][0];
              const uint32_t w8 = pb ? (rr[h][1] >> 8) : rr[h][1];
              // per bit: mask ? (c ? ~y : y) : c (three-input function 0x6A), i.e.
              // the masked nibbles with their bias bit flipped (code + 8) under
              // the f16 pattern 0x6400 of c
              uint32_t a0, a1, a2, a3;
              asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(a0) : "r"(wg), "r"(0x000F000Fu), "r"(0x64086408u));
              asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(a1) : "r"(w8), "r"(0x000F000Fu), "r"(0x64086408u));
              asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(a2) : "r"(wg), "r"(0x00F000F0u), "r"(0x64806480u));
              asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(a3) : "r"(w8), "r"(0x00F000F0u), "r"(0x64806480u));
              float d0[4] = {nb00, nb01, nb00, nb01}, d1[4] = {nb10, nb11, nb10, nb11};
              mma_f16_k16(d0, a0, a1, a2, a3, hb[0][0], hb[0][1]);
              mma_f16_k16(d1, a0, a1, a2, a3, hb[1][0], hb[1][1]);
              // local = e + 2 pb + 4 nt; rows g (d[0], d[1]) and g + 8 (d[2], d[3])
              float* o0 = u + RUN * s + 2 * pb;
              float* o1 = u + 32 + RUN * s + 2 * pb;
              o0[0] = d0[0];
              o0[1] = d0[1];
              o0[4] = d1[0];
              o0[5] = d1[1];
              o1[0] = d0[2];
              o1[1] = d0[3];
              o1[4] = d1[2];
              o1[5] = d1[3];
            }
          } else {
            const uint32_t wg = rr[h][0] ^ 0x80808080u, w8 = rr[h][1] ^ 0x80808080u;
            const uint32_t a0 = __byte_perm(wg, 0x64646464u, 0x4140);  // codes i = 0, 1 of block g
            const uint32_t a1 = __byte_perm(w8, 0x64646464u, 0x4140);
            const uint32_t a2 = __byte_perm(wg, 0x64646464u, 0x4342);  // i = 2, 3
            const uint32_t a3 = __byte_perm(w8, 0x64646464u, 0x4342);
            float d0[4] = {nb00, nb01, nb00, nb01}, d1[4] = {nb10, nb11, nb10, nb11};
            mma_f16_k16(d0, a0, a1, a2, a3, hb[0][0], hb[0][1]);
            mma_f16_k16(d1, a0, a1, a2, a3, hb[1][0], hb[1][1]);
            // local = e + 2 nt
            float* o0 = u + RUN * s;
            float* o1 = u + 32 + RUN * s;
            o0[0] = d0[0];
            o0[1] = d0[1];
            o0[2] = d1[0];
            o0[3] = d1[1];
            o1[0] = d0[2];
            o1[1] = d0[3];
            o1[2] = d1[2];
            o1[3] = d1[3];
          }
        }
      }
      // INT4: local bit 1 (j1) and segment bits (j5, j6); INT8: segment bits (j4..j6)
      if constexpr (BITS == 4) {
        reg_stage<64, 2>(u);
        reg_stage<64, 8>(u);
        reg_stage<64, 16>(u);
      } else {
        reg_stage<64, 4>(u);
        reg_stage<64, 8>(u);
        reg_stage<64, 16>(u);
      }
      if (!OUT_F32 && grp == 0) {  // the previous slab's bulk copy has read the staging rows
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int b = g + 8 * r + 16 * grp;  // block in the slab
        float* v = u + 32 * r;
        const float s0 = sc[2 * grp + r];
        const bool tiny = s0 < kTinyScale && s0 != 0.0f;
        const float f = (tiny ? s0 * kUp64 : s0) * a.rsqrt_b;
#pragma unroll
        for (int k = 0; k < 32; k += 2) mul2(v[k], v[k + 1], f);
        if (tiny) {
#pragma unroll
          for (int k = 0; k < 32; k += 2) mul2(v[k], v[k + 1], kDown64);
        }
        uint4 sb = make_uint4(0, 0, 0, 0);
        if constexpr (SIGNS) {
          uint32_t cb = (uint32_t)(colc + b);
          cb = a.cpr >= 32 ? (cb >= (uint32_t)a.cpr ? cb - a.cpr : cb) : cb % (uint32_t)a.cpr;
          sb = *reinterpret_cast<const uint4*>(s_bytes + cb * 16);
        }
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          const float* w = v + RUN * p;
          const int j0 = BITS == 4 ? 32 * p + 8 * t4 : 16 * p + 4 * t4;  // first output of the run
          uint4 m4 = make_uint4(0, 0, 0, 0);
          if constexpr (SIGNS) {
            const uint32_t wsel = (j0 >> 5) == 0 ? sb.x : (j0 >> 5) == 1 ? sb.y : (j0 >> 5) == 2 ? sb.z : sb.w;
            m4 = s_tab[__byte_perm(wsel, 0, 0x4440 + ((j0 >> 3) & 3))];
            if (BITS == 8 && (j0 & 4)) m4 = make_uint4(m4.z, m4.w, 0, 0);
          }
          if constexpr (OUT_F32) {
            if (b < nch) {
              float* dst = a.rot + size_t(c + b) * kCK + j0;
              const uint32_t mm[4] = {m4.x, m4.y, m4.z, m4.w};
              uint32_t o[8];
#pragma unroll
              for (int k = 0; k < RUN / 2; ++k) {
                o[2 * k] = __float_as_uint(w[2 * k]) ^ (mm[k] << 16);
                o[2 * k + 1] = __float_as_uint(w[2 * k + 1]) ^ (mm[k] & 0x80000000u);
              }
              reinterpret_cast<uint4*>(dst)[0] = make_uint4(o[0], o[1], o[2], o[3]);
              if constexpr (RUN == 8) reinterpret_cast<uint4*>(dst)[1] = make_uint4(o[4], o[5], o[6], o[7]);
            }
          } else {
            uint32_t o[4];
#pragma unroll
            for (int k = 0; k < RUN / 2; ++k) {
              uint32_t rcv;
              asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(rcv) : "f"(w[2 * k + 1]), "f"(w[2 * k]));
              o[k] = rcv;
            }
            if constexpr (SIGNS) {
              o[0] ^= m4.x;
              o[1] ^= m4.y;
              if constexpr (RUN == 8) {
                o[2] ^= m4.z;
                o[3] ^= m4.w;
              }
            }
            uint8_t* dst = ostage + b * L::OP + 2 * j0;
            if constexpr (RUN == 8)
              *reinterpret_cast<uint4*>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
            else
              *reinterpret_cast<uint2*>(dst) = make_uint2(o[0], o[1]);
          }
        }
      }
    }
    if constexpr (SIGNS) {
      colc += col_step;
      if (colc >= a.cpr) colc -= a.cpr;
    }
    if constexpr (!OUT_F32) {
      fence_async_shared();  // the run stores are visible to the copy engine
      __syncwarp();
      if (lane == 0) {
        bulk_store_s2g(reinterpret_cast<uint8_t*>(a.out_bf16) + size_t(c) * 256, ostage, uint32_t(nch) * 256u);
        bulk_commit();
      }
    }
  }
  cp_async_wait<0>();
  if (!OUT_F32 && lane == 0) bulk_wait_all();  // the staging stays valid until the last copy is done
}

}  // namespace hadq
