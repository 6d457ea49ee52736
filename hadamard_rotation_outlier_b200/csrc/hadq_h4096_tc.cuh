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
//  * epilogue (kTcEpiWG warpgroups, taking tiles in turn): tcgen05.ld of two
//    blocks (64 columns) at a time, five butterfly stages, block maxima by
//    warp reduction and one named barrier per pair of blocks, codes and
//    scales to global memory.
// Every mbarrier wait gives up after about a second: the kernel then records
// a fault (hadq_device_status reads it), every role leaves its loop, copies
// still in flight are awaited (bounded), and the CTA frees its TMEM.
#pragma once

#include <cuda.h>

#include <cstddef>

#include "hadq_common.cuh"

namespace hadq {

// Shape constants (the defaults are the measured best on the 16384 x 4096
// workload; other values build for comparison).
#ifndef HADQ_TC_EPI_WG
#define HADQ_TC_EPI_WG 4
#endif
#ifndef HADQ_TC_BPP
#define HADQ_TC_BPP 1
#endif
#ifndef HADQ_TC_TILE
#define HADQ_TC_TILE 4
#endif
#ifndef HADQ_TC_STAGES
#define HADQ_TC_STAGES (20 / HADQ_TC_TILE)
#endif
constexpr int kTcTileBlocks = HADQ_TC_TILE;        // 4096-point blocks per tile (N = 32 per block)
constexpr int kTcStages = HADQ_TC_STAGES;          // input stages of one tile each
constexpr int kTcAcc = 16 / kTcTileBlocks;         // TMEM accumulators (512 columns in all)
constexpr int kTcEpiWG = HADQ_TC_EPI_WG;           // epilogue warpgroups
constexpr int kTcBpp = HADQ_TC_BPP;                // blocks per epilogue pass (one barrier each)
static_assert(kTcTileBlocks == 2 || kTcTileBlocks == 4, "tiles of 2 or 4 blocks");
static_assert(kTcTileBlocks % kTcBpp == 0, "passes cover a tile");
static_assert(kTcBpp == 1 || kTcBpp == 2 || kTcBpp == 4, "blocks per pass");
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
constexpr unsigned long long kTcWaitNs = 1000000000ull;  // about one second per wait

struct TcTail {
  uint64_t full[kTcStages];    // TMA bytes landed
  uint64_t signd[kTcStages];   // signs applied (signed calls)
  uint64_t empty[kTcStages];   // MMAs done reading the stage
  uint64_t tfull[kTcAcc];      // accumulator written
  uint64_t tempty[kTcAcc];     // accumulator read by its warpgroup
  alignas(16) uint32_t red[kTcEpiWG][2][kTcBpp][4];  // [group][parity][block of the pass][warp]:
                                                     // max bits, read back as 16-byte vectors
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

// ------------------------------------------------------------- PTX wrappers

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(b)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_addr(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait for the phase of `parity` to complete.  False after kTcWaitNs, or as
// soon as another role has given up (abort set; a null abort waits out the
// time limit, for copies and MMAs still in flight).
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, const volatile uint32_t* abort) {
  if (mbar_test(b, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
    if (mbar_test(b, parity)) return true;
    if (abort && *abort) return false;
    if (global_ns() - t0 > kTcWaitNs) return false;
  }
}
__device__ __forceinline__ void tc_give_up(TcTail* tl, unsigned* fault) {
  atomicOr(fault, 1u);
  *reinterpret_cast<volatile uint32_t*>(&tl->abort) = 1u;
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: start address, leading and stride byte
// offsets (16-byte units), the fixed version field, the swizzle mode
// (2 = 128-byte, 4 = 64-byte).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t swizzle) {
  return uint64_t((addr & 0x3FFFFu) >> 4) | (uint64_t(lbo >> 4) << 16) | (uint64_t(sbo >> 4) << 32) | (1ull << 46) |
         (uint64_t(swizzle) << 61);
}
// Instruction descriptor of kind::f16: D float32, A and B bf16, A K-major,
// B MN-major, N = 32 x blocks per tile, M = 128.
constexpr uint32_t kTcIdesc =
    (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t(kTcAccCols) >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kTcIdesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// 32 lanes x 64 columns of 32 bits from TMEM (lane = thread, register j =
// column + j), waited for inside the same statement so that no use of the
// registers can be scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&a)[32], float (&b)[32]) {
  uint32_t r[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, "
      "%38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, "
      "%60, %61, %62, %63}, [%64];\n"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]),
        "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]),
        "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]),
        "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]),
        "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    a[j] = __uint_as_float(r[j]);
    b[j] = __uint_as_float(r[32 + j]);
  }
}

// 32 lanes x 32 columns (one block), waited for in the same statement.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&a)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int j = 0; j < 32; ++j) a[j] = __uint_as_float(r[j]);
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

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

  // H_128 as the A operand, K-major with the 128-byte swizzle: element (m, k)
  // at (k / 64) * 16384 + (m / 8) * 1024 + (m % 8) * 128 + 16 * ((k % 64) / 8
  // XOR m % 8) + 2 * (k % 8); one 16-byte piece (8 k) per iteration.
  for (int i = threadIdx.x; i < 128 * 16; i += kTcThreads) {
    const int m = i >> 4, kc = i & 15;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int k = 8 * kc + 2 * e;
      const uint32_t lo = (__popc(m & k) & 1) ? 0xBF80u : 0x3F80u;
      const uint32_t hi = (__popc(m & (k + 1)) & 1) ? 0xBF80u : 0x3F80u;
      w[e] = lo | (hi << 16);
    }
    const int off = (kc >> 3) * 16384 + (m >> 3) * 1024 + (m & 7) * 128 + (((kc & 7) ^ (m & 7)) << 4);
    *reinterpret_cast<uint4*>(amat + off) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&tl->full[s], 1);
      mbar_init(&tl->signd[s], kTcSignWarps);
      mbar_init(&tl->empty[s], 1);
    }
    for (int c = 0; c < kTcAcc; ++c) {
      mbar_init(&tl->tfull[c], 1);
      mbar_init(&tl->tempty[c], 4);
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
          tc_give_up(tl, a.fault);
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
          tc_give_up(tl, a.fault);
          break;
        }
        tc_fence_after();
        const uint32_t bbase = smem_addr(stages + s * kTcStageBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = smem_desc(abase + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, 2);
          const uint64_t bd = smem_desc(bbase + kk * 1024, 8192, 512, 4);
          tc_mma(tmem + uint32_t(c * kTcAccCols), ad, bd, kk > 0 ? 1u : 0u);
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
          tc_give_up(tl, a.fault);
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
    // Epilogue warpgroup g: warp q = warp % 4 reads TMEM lanes 32 q .. 32 q + 31.
    const int g = warp >> 2, q = warp & 3, h = 32 * q + lane;
    constexpr int CODE_BYTES = BITS == 8 ? 32 : 16;
    uint32_t par = 0;
    int it = 0;
    for (int64_t t = first; t < a.ntiles; t += step, ++it) {
      if (it % kTcEpiWG != g) continue;
      const int c = it % kTcAcc;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tl->tfull[c], (it / kTcAcc) & 1, abort));
      tc_fence_after();
      bool stop = false;
#pragma unroll 1
      for (int pr = 0; pr < kTcTileBlocks / kTcBpp; ++pr) {
        float v[kTcBpp][32];
        if (ok) {
          const uint32_t ta = tmem + (uint32_t(32 * q) << 16) + uint32_t(c * kTcAccCols + 32 * kTcBpp * pr);
          if constexpr (kTcBpp == 2) {
            tmem_ld64(ta, v[0], v[1]);
          } else {
#pragma unroll
            for (int b = 0; b < kTcBpp; ++b) tmem_ld32(ta + 32 * b, v[b]);
          }
        } else {
#pragma unroll
          for (int b = 0; b < kTcBpp; ++b)
#pragma unroll
            for (int j = 0; j < 32; ++j) v[b][j] = 0.0f;
        }
        if (pr == kTcTileBlocks / kTcBpp - 1) {  // the accumulator has been read
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tl->tempty[c]);
        }
        // non-negative floats order as their bit patterns; a warp that gave up
        // votes ~0, which no |y| can reach
#pragma unroll
        for (int b = 0; b < kTcBpp; ++b) {
          const float m = tc_h32_absmax(v[b]);
          const uint32_t mb = __reduce_max_sync(0xffffffffu, ok ? __float_as_uint(m) : ~0u);
          if (lane == 0) tl->red[g][par][b][q] = mb;
        }
        named_bar_sync(1 + g, 128);
        uint32_t M[kTcBpp];
#pragma unroll
        for (int b = 0; b < kTcBpp; ++b) {
          const uint4 r = *reinterpret_cast<const uint4*>(tl->red[g][par][b]);  // after the barrier
          M[b] = max(max(r.x, r.y), max(r.z, r.w));
          if (M[b] == ~0u) stop = true;
        }
        par ^= 1u;
        if (stop) break;
#pragma unroll
        for (int b = 0; b < kTcBpp; ++b) {
          const int64_t blk = t * kTcTileBlocks + kTcBpp * pr + b;
          if (blk < a.nblocks) {
            const float m = __uint_as_float(M[b]);
            if (h == 0) a.scales[blk] = m * a.scale_mul;
            tc_store_codes<BITS>(v[b], m, a.codes + blk * (4096 * BITS / 8) + h * CODE_BYTES);
          }
        }
      }
      if (stop) {
        if (h == 0) tc_give_up(tl, a.fault);
        break;
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
