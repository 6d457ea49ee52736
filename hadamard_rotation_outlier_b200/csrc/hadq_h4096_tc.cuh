// Forward 4096-point Hadamard blocks (one scale per block) on the fifth-
// generation tensor cores (tcgen05, TMEM accumulators, TMA loads).
//
// H_4096 = H_128 (x) H_32 on the index split j = 32 h + l (h: index bits
// 5-11, l: bits 0-4).  The bf16 input (times the +-1 signs, still exact in
// bf16) and H_128 (+-1) make the transform along h a bf16 GEMM with exact
// products and float32 accumulation,
//     D[h'][(r, l)] = sum_h H_128[h'][h] X_r[h][l],
// over the four blocks r of a tile: M = 128 (h'), N = 4 x 32 (r, l), K = 128
// (h).  The five remaining stages act along l inside one thread: TMEM lane h'
// holds block r's 32 values at l = 0..31, and after the butterflies these are
// the outputs 32 h' + l', so each thread writes 32 consecutive codes (16
// bytes for INT4, 32 for INT8) with no transpose.
//
// Roles (one CTA per SM, persistent over tiles of four blocks):
//  * producer (one thread): one TMA copy per tile, 3-D tensor map
//    [block][h][l] with a 64-byte swizzle, into one of kTcStages 32 KB stages;
//  * signs (four warps, signed calls only): XOR the sign masks into the
//    stage.  The four 8 KB block images of a tile share one swizzled layout,
//    so each thread keeps the masks of its four 16-byte pieces in registers;
//  * MMA (one thread): eight tcgen05.mma (K = 16 each) per tile into one of
//    kTcAcc TMEM accumulators of 128 columns.  A = H_128 from shared memory
//    (K-major, 128-byte swizzle, written once per CTA); B = the stage
//    (MN-major, 64-byte swizzle, as the TMA left it).  Commits release the
//    stage and hand the accumulator on;
//  * epilogue (one warpgroup per block of a tile, so the four work on the
//    same tile at once): tcgen05.ld of the block's 32 columns, five butterfly
//    stages, the block maximum by warp reduction and one named barrier,
//    codes and scales to global memory.
// Every mbarrier wait gives up after about a second: the kernel then records
// a fault (hadq_device_status reads it), every role leaves its loop, copies
// still in flight are awaited (bounded), and the CTA frees its TMEM.
#pragma once

#include <cuda.h>

#include <cstddef>

#include "hadq_common.cuh"
#include "hadq_tc.cuh"

namespace hadq {

// Shape constants (the defaults are the measured best on the 16384 x 4096
// workload; other values build for comparison).
#ifndef HADQ_TC_TILE
#define HADQ_TC_TILE 4
#endif
#ifndef HADQ_TC_STAGES
#define HADQ_TC_STAGES (20 / HADQ_TC_TILE)
#endif
constexpr int kTcTileBlocks = HADQ_TC_TILE;        // 4096-point blocks per tile (N = 32 per block)
constexpr int kTcStages = HADQ_TC_STAGES;          // input stages of one tile each
constexpr int kTcAcc = 16 / kTcTileBlocks;         // TMEM accumulators (512 columns in all)
constexpr int kTcEpiWG = kTcTileBlocks;            // epilogue warpgroups: one per block of a tile
static_assert(kTcTileBlocks == 2 || kTcTileBlocks == 4, "tiles of 2 or 4 blocks");
constexpr int kTcStageBytes = kTcTileBlocks * 8192;
constexpr int kTcABytes = 128 * 128 * 2;           // H_128 in bf16
#ifndef HADQ_TC_SIGNW
#define HADQ_TC_SIGNW 4
#endif
constexpr int kTcSignWarps = HADQ_TC_SIGNW;        // warps applying the signs
constexpr int kTcSignPieces = 512 / (32 * kTcSignWarps);  // 16-byte pieces per thread and block image
static_assert(kTcSignPieces * 32 * kTcSignWarps == 512, "sign pieces cover a block image");
constexpr int kTcSignWarp0 = 4 * kTcEpiWG;         // warps 0 .. 4 kTcEpiWG - 1: epilogue
constexpr int kTcProdWarp = kTcSignWarp0 + kTcSignWarps;  // then the sign warps, the producer
constexpr int kTcMmaWarp = kTcProdWarp + 1;        // and the MMA warp (also allocates TMEM)
constexpr int kTcThreads = (kTcMmaWarp + 1) * 32;
constexpr int kTcAccCols = 32 * kTcTileBlocks;    // N of the MMA
constexpr uint32_t kTcTmemCols = kTcAcc * kTcAccCols;
// Instruction descriptor: M = 128, N = 32 x blocks per tile, B MN-major.
constexpr uint32_t kTcIdesc = tc_idesc_bf16(128, kTcAccCols, true);

struct TcTail {
  uint64_t full[kTcStages];    // TMA bytes landed
  uint64_t signd[kTcStages];   // signs applied (signed calls)
  uint64_t empty[kTcStages];   // MMAs done reading the stage
  uint64_t tfull[kTcAcc];      // accumulator written
  uint64_t tempty[kTcAcc];     // accumulator read by every epilogue warp
  alignas(16) uint32_t red[kTcEpiWG][2][4];  // [group][parity][warp]: max bits, read back as
                                             // 16-byte vectors
  uint32_t tmem_base;
  uint32_t abort;
};

static_assert(offsetof(TcTail, red) % 16 == 0, "the maxima are read as 16-byte vectors");
static_assert(offsetof(TcTail, full) % 8 == 0, "mbarriers are 8-byte aligned");

__host__ __device__ constexpr size_t h4096_tc_smem_bytes() {
  return 1024 + size_t(kTcStages) * kTcStageBytes + kTcABytes + sizeof(TcTail);
}

struct TcArgs {
  int64_t nblocks;        // rows * dim / 4096
  int64_t ntiles;         // ceil(nblocks / 4)
  const int8_t* signs;    // 4096 entries (signed calls have dim = 4096)
  uint8_t* codes;
  float* scales;
  float scale_mul;        // 1 / (64 * qmax)
  unsigned* fault;        // set to 1 when a bounded wait ran out
  int stall_tile;         // -1; else the producer stops before this local tile
                          // (self-test: the waits for it run out)
};

// Codes of one block's 32 consecutive outputs against the block maximum m,
// stored at dst (16 bytes for INT4, 32 for INT8).
template <int BITS>
__device__ __forceinline__ void tc_store_codes(float (&v)[32], float m, uint8_t* dst) {
  constexpr float QMAX = BITS == 8 ? 127.0f : 7.0f;
  const QInv q = make_qinv(m, QMAX);
  if (q.tiny) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] *= 18446744073709551616.0f;  // 2^64, exact
  }
  uint32_t c[32];
#pragma unroll
  for (int i = 0; i < 32; i += 2) magic_code2(v[i], v[i + 1], q.inv, c[i], c[i + 1]);
  if constexpr (BITS == 8) {
    uint4* d = reinterpret_cast<uint4*>(dst);
    d[0] = make_uint4(pack_i8x4(c[0], c[1], c[2], c[3]), pack_i8x4(c[4], c[5], c[6], c[7]),
                      pack_i8x4(c[8], c[9], c[10], c[11]), pack_i8x4(c[12], c[13], c[14], c[15]));
    d[1] = make_uint4(pack_i8x4(c[16], c[17], c[18], c[19]), pack_i8x4(c[20], c[21], c[22], c[23]),
                      pack_i8x4(c[24], c[25], c[26], c[27]), pack_i8x4(c[28], c[29], c[30], c[31]));
  } else {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t (&ck)[8] = *reinterpret_cast<const uint32_t(*)[8]>(c + 8 * k);
      w[k] = pack_i4x8(ck);
    }
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Five butterfly stages over a block's 32 values (along l), the last fused
// with the block-local maximum of |y|.
__device__ __forceinline__ float tc_h32_absmax(float (&v)[32]) {
  reg_stage<32, 1>(v);
  reg_stage<32, 2>(v);
  reg_stage<32, 4>(v);
  reg_stage<32, 8>(v);
  return reg_stage_absmax<32, 16>(v);
}

template <int BITS, bool SIGNS>
__global__ void __launch_bounds__(kTcThreads, 1) rq_h4096_tc_kernel(const __grid_constant__ CUtensorMap tmap, TcArgs a) {
  extern __shared__ uint8_t tc_smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = base;
  uint8_t* amat = base + kTcStages * kTcStageBytes;
  TcTail* tl = reinterpret_cast<TcTail*>(amat + kTcABytes);
  const volatile uint32_t* abort = &tl->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  write_h128_kmajor(amat, kTcThreads);  // H_128 as the A operand
  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&tl->full[s], 1);
      mbar_init(&tl->signd[s], kTcSignWarps);
      mbar_init(&tl->empty[s], 1);
    }
    for (int c = 0; c < kTcAcc; ++c) {
      mbar_init(&tl->tfull[c], 1);
      mbar_init(&tl->tempty[c], 4 * kTcEpiWG);
    }
    tl->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kTcMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&tl->tmem_base)),
                 "r"(kTcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_async_shared();  // H_128 (generic writes) is read by the tensor cores
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tl->tmem_base;
  const int64_t first = blockIdx.x, step = gridDim.x;

  if (warp == kTcProdWarp) {
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap)) : "memory");
      int issued = 0;
      for (int64_t t = first; t < a.ntiles; t += step, ++issued) {
        if (issued == a.stall_tile) break;
        const int s = issued % kTcStages;
        const uint32_t ph = (issued / kTcStages) & 1;
        if (!mbar_wait(&tl->empty[s], ph ^ 1u, abort)) {
          tc_give_up(&tl->abort, a.fault);
          break;
        }
        mbar_expect_tx(&tl->full[s], kTcStageBytes);
        tma_load_3d(stages + s * kTcStageBytes, &tmap, &tl->full[s], 0, 0, int(t * kTcTileBlocks));
      }
      // Every copy this thread issued has landed before the CTA can exit (on
      // the normal path these waits pass at once).
      for (int j = issued > kTcStages ? issued - kTcStages : 0; j < issued; ++j)
        (void)mbar_wait(&tl->full[j % kTcStages], (j / kTcStages) & 1, nullptr);
    }
  } else if (warp == kTcMmaWarp) {
    if (lane == 0) {
      const uint32_t abase = smem_addr(amat);
      int issued = 0;
      for (int64_t t = first; t < a.ntiles; t += step, ++issued) {
        const int s = issued % kTcStages, c = issued % kTcAcc;
        const uint32_t ph = (issued / kTcStages) & 1, cph = (issued / kTcAcc) & 1;
        if (!mbar_wait(SIGNS ? &tl->signd[s] : &tl->full[s], ph, abort) ||
            !mbar_wait(&tl->tempty[c], cph ^ 1u, abort)) {
          tc_give_up(&tl->abort, a.fault);
          break;
        }
        tc_fence_after();
        const uint32_t bbase = smem_addr(stages + s * kTcStageBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = smem_desc(abase + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, 2);
          const uint64_t bd = smem_desc(bbase + kk * 1024, 8192, 512, 4);
          tc_mma(tmem + uint32_t(c * kTcAccCols), ad, bd, kTcIdesc, kk > 0 ? 1u : 0u);
        }
        tc_commit(&tl->empty[s]);
        tc_commit(&tl->tfull[c]);
      }
      // The MMAs are complete before TMEM is freed (passes at once normally).
      if (issued > 0) {
        const int j = issued - 1;
        (void)mbar_wait(&tl->tfull[j % kTcAcc], (j / kTcAcc) & 1, nullptr);
      }
    }
  } else if (warp >= kTcSignWarp0) {
    if constexpr (SIGNS) {
      // Thread st owns the 16-byte pieces st + 32 kTcSignWarps c of every 8 KB
      // block image.  Piece P holds h = P / 4 and the 8 values l = 8 ((P % 4)
      // XOR (h / 2) % 4) + e (the 64-byte swizzle).
      const int st = threadIdx.x - kTcSignWarp0 * 32;
      constexpr int PS = 32 * kTcSignWarps;  // piece stride between a thread's pieces
      uint4 mask[kTcSignPieces];
#pragma unroll
      for (int c = 0; c < kTcSignPieces; ++c) {
        const int P = st + PS * c, h = P >> 2, l0 = 8 * ((P & 3) ^ ((h >> 1) & 3));
        const int8_t* sg = a.signs + 32 * h + l0;
        mask[c] = make_uint4(pair_sign_mask(sg[0], sg[1]), pair_sign_mask(sg[2], sg[3]), pair_sign_mask(sg[4], sg[5]),
                             pair_sign_mask(sg[6], sg[7]));
      }
      int it = 0;
      for (int64_t t = first; t < a.ntiles; t += step, ++it) {
        const int s = it % kTcStages;
        const uint32_t ph = (it / kTcStages) & 1;
        if (!mbar_wait(&tl->full[s], ph, abort)) {
          tc_give_up(&tl->abort, a.fault);
          break;
        }
        uint4* p = reinterpret_cast<uint4*>(stages + s * kTcStageBytes) + st;
#pragma unroll
        for (int r = 0; r < kTcTileBlocks; ++r)
#pragma unroll
          for (int c = 0; c < kTcSignPieces; ++c) {
            uint4 v = p[512 * r + PS * c];
            v.x ^= mask[c].x;
            v.y ^= mask[c].y;
            v.z ^= mask[c].z;
            v.w ^= mask[c].w;
            p[512 * r + PS * c] = v;
          }
        fence_async_shared();  // the tensor cores read what this thread wrote
        __syncwarp();
        if (lane == 0) mbar_arrive(&tl->signd[s]);
      }
    }
  } else {
    // Epilogue warpgroup g takes block g of every tile; its warp q = warp % 4
    // reads TMEM lanes 32 q .. 32 q + 31.
    const int g = warp >> 2, q = warp & 3, h = 32 * q + lane;
    constexpr int CODE_BYTES = BITS == 8 ? 32 : 16;
    uint32_t par = 0;
    int it = 0;
    for (int64_t t = first; t < a.ntiles; t += step, ++it) {
      const int c = it % kTcAcc;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tl->tfull[c], (it / kTcAcc) & 1, abort));
      tc_fence_after();
      // A warp that gave up still reads its accumulator (allocated TMEM, so
      // the read is safe); its values are never stored.
      float v[32];
      tmem_ld32(tmem + (uint32_t(32 * q) << 16) + uint32_t(c * kTcAccCols + 32 * g), v);
      tc_fence_before();  // this warp's part of the accumulator has been read
      __syncwarp();
      if (lane == 0) mbar_arrive(&tl->tempty[c]);
      // non-negative floats order as their bit patterns; a warp that gave up
      // votes ~0, which no |y| can reach
      const float m = tc_h32_absmax(v);
      const uint32_t mb = __reduce_max_sync(0xffffffffu, ok ? __float_as_uint(m) : ~0u);
      if (lane == 0) tl->red[g][par][q] = mb;
      named_bar_sync(1 + g, 128);
      const uint4 r = *reinterpret_cast<const uint4*>(tl->red[g][par]);  // after the barrier
      const uint32_t M = max(max(r.x, r.y), max(r.z, r.w));
      par ^= 1u;
      if (M == ~0u) {
        if (h == 0) tc_give_up(&tl->abort, a.fault);
        break;
      }
      const int64_t blk = t * kTcTileBlocks + g;
      if (blk < a.nblocks) {
        const float mf = __uint_as_float(M);
        if (h == 0) a.scales[blk] = mf * a.scale_mul;
        tc_store_codes<BITS>(v, mf, a.codes + blk * (4096 * BITS / 8) + h * CODE_BYTES);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kTcMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols) : "memory");
  }
}

}  // namespace hadq
