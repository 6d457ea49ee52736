// C ABI of libhadq: argument checks, kernel choice and launches.
//
// Every entry point validates its arguments on the host, picks a kernel
// family, launches one kernel on the caller's stream and returns.  Nothing here
// allocates device memory, and only hadq_device_status synchronises.
#include <cmath>
#include <cstdint>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>
#include <string>
#include <unordered_map>
#include <vector>

#include "../../include/hadq.h"
#include "hadq_asym.cuh"
#include "hadq_attn.cuh"
#include "hadq_blocked.cuh"
#include "hadq_chunk.cuh"
#include "hadq_chunk_mma.cuh"
#include "hadq_dq_mma.cuh"
#include "hadq_full4096.cuh"
#include "hadq_generic.cuh"
#include "hadq_h4096.cuh"
#include "hadq_h4096_tc.cuh"
#include "hadq_kron.cuh"
#include "hadq_kernels.h"

namespace {

thread_local std::string g_last_error;
std::atomic<int64_t> g_launches{0};

hadq_status fail(hadq_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
hadq_status fail(hadq_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }
int ilog2(int64_t v) {
  int r = 0;
  while ((int64_t(1) << r) < v) ++r;
  return r;
}
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

struct Shape {
  int64_t rows;
  int dim, B, G, bits;
  bool has_signs;
};

// Size checks shared by both directions.  On success fills B and G.
hadq_status check_sizes(int64_t rows, int32_t dim, int32_t block, int32_t bits, int32_t group,
                        Shape* s) {
  if (rows < 0) return fail(HADQ_ERR_INVALID_ARG, "rows must be >= 0 (got %lld)", (long long)rows);
  if (dim < 1 || dim > HADQ_MAX_DIM)
    return fail(HADQ_ERR_INVALID_ARG, "dim must be in [1, %d] (got %d)", HADQ_MAX_DIM, dim);
  if (bits != 4 && bits != 8) return fail(HADQ_ERR_INVALID_ARG, "bits must be 4 or 8 (got %d)", bits);
  if (bits == 4 && (dim & 1))
    return fail(HADQ_ERR_INVALID_ARG, "INT4 packs two codes per byte: dim must be even (got %d)", dim);
  int B;
  if (block == -1) {
    if (!is_pow2(dim))
      return fail(HADQ_ERR_INVALID_ARG, "block -1 (whole row) needs a power-of-two dim (got %d)", dim);
    B = dim;
  } else {
    if (!is_pow2(block)) return fail(HADQ_ERR_INVALID_ARG, "block must be -1 or a power of two (got %d)", block);
    if (dim % block) return fail(HADQ_ERR_INVALID_ARG, "block %d does not divide dim %d", block, dim);
    B = block;
  }
  int G;
  if (group == -1) {
    G = dim;
  } else {
    if (group < 1) return fail(HADQ_ERR_INVALID_ARG, "group must be -1 or >= 1 (got %d)", group);
    if (dim % group) return fail(HADQ_ERR_INVALID_ARG, "group %d does not divide dim %d", group, dim);
    G = group;
  }
  s->rows = rows;
  s->dim = dim;
  s->B = B;
  s->G = G;
  s->bits = bits;
  return HADQ_OK;
}

bool blocked_group_ok(int G, int B) { return (is_pow2(G) && G >= 8 && G <= B) || (G % B == 0); }

bool chunk_ok(int direction, const Shape& s) {
  (void)direction;
  if (s.B < 8 || s.B > 128 || s.dim % 128) return false;
  if (is_pow2(s.G) && s.G >= 8 && s.G <= 128) return true;
  return s.G % 128 == 0 && s.dim <= 128 * hadq::kCT;  // a slab holds whole rows
}

hadq_path choose_path(int direction, const Shape& s, bool aligned16) {
  if (s.rows == 0) return HADQ_PATH_NONE;
  // the tensor-core 128-point kernels index chunks with 32-bit integers
  const bool mma_size_ok = s.rows * (s.dim / 128) < (int64_t(1) << 30);
  if (aligned16 && direction == 0 && s.B == 128 && s.G == 128 && s.dim % 128 == 0 && mma_size_ok)
    return HADQ_PATH_CHUNK_MMA;
  if (aligned16 && direction == 1 && s.B == 128 && s.G % 128 == 0 && s.dim % 128 == 0 && mma_size_ok)
    return HADQ_PATH_CHUNK_MMA;
  if (aligned16 && chunk_ok(direction, s)) return HADQ_PATH_CHUNK;
  if (aligned16 && direction == 0 && s.B == 4096 && s.dim % 4096 == 0 && s.G == 4096) {
    if (s.dim != 4096 && s.has_signs) return HADQ_PATH_WIDE4096;
    // tile coordinates of the tcgen05 kernel are 32-bit
    return s.rows * (s.dim / 4096) < (int64_t(1) << 30) ? HADQ_PATH_H4096_TC : HADQ_PATH_WIDE4096_MMA;
  }
  if (aligned16 && (s.B == 32 || s.B == 64 || s.B == 128 || s.B == 256) && s.dim % 32 == 0 &&
      s.dim <= 16384 && blocked_group_ok(s.G, s.B))
    return HADQ_PATH_BLOCKED;
  if (direction == 0 && aligned16 && s.B == 4096 && s.dim == 4096 && is_pow2(s.G) && s.G >= 64)
    return HADQ_PATH_FULL4096;
  return HADQ_PATH_GENERIC;
}

int sm_count() {
  static std::mutex mu;
  static std::unordered_map<int, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(dev);
  if (it != cache.end()) return it->second;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  cache[dev] = n;
  return n;
}

// One launch configuration per (device, kernel, block size, dynamic shared
// memory): the resident CTAs per SM are read once; later calls only find the
// entry.  The dynamic shared-memory limit is an attribute of the kernel, not
// of a launch, so it is raised to the largest size any call has needed (a
// smaller launch of the same kernel stays valid under a larger limit).
struct LaunchEntry {
  int dev;
  const void* fn;
  int threads;
  size_t smem;
  int resident;
};
struct SmemLimit {
  int dev;
  const void* fn;
  size_t smem;
};
std::mutex g_launch_mu;
std::vector<LaunchEntry> g_launch_cache;
std::vector<SmemLimit> g_smem_limits;

hadq_status prepare(const void* fn, int threads, size_t smem, const char* what, int* resident_out) {
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(g_launch_mu);
  for (const LaunchEntry& e : g_launch_cache)
    if (e.dev == dev && e.fn == fn && e.threads == threads && e.smem == smem) {
      *resident_out = e.resident;
      return HADQ_OK;
    }
  if (smem > 48 * 1024) {
    SmemLimit* lim = nullptr;
    for (SmemLimit& l : g_smem_limits)
      if (l.dev == dev && l.fn == fn) lim = &l;
    if (!lim || lim->smem < smem) {
      cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(HADQ_ERR_CUDA, "%s: cannot reserve %zu bytes of shared memory: %s", what, smem,
                    cudaGetErrorString(e));
      }
      if (lim)
        lim->smem = smem;
      else
        g_smem_limits.push_back({dev, fn, smem});
    }
  }
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, smem) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = 1;
  }
  g_launch_cache.push_back({dev, fn, threads, smem, n});
  *resident_out = n;
  return HADQ_OK;
}

hadq_status after_launch(const char* what) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(HADQ_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(e));
  return HADQ_OK;
}

// ----------------------------------------------------------------- blocked

struct BlockedPlan {
  int threads, rpi, tpr;
  int64_t nslabs;
  size_t smem;
};

BlockedPlan blocked_plan(const Shape& s) {
  BlockedPlan p;
  p.tpr = s.dim / 32;
  p.rpi = p.tpr <= 256 ? 256 / p.tpr : 1;
  const int t = p.rpi * p.tpr;
  p.threads = (t + 31) / 32 * 32;
  p.nslabs = (s.rows + p.rpi - 1) / p.rpi;
  p.smem = s.G > s.B ? size_t(3) * p.rpi * (s.dim / s.G) * sizeof(uint32_t) : 0;
  return p;
}

hadq_status launch_blocked(int direction, const Shape& s, hadq::BlockedArgs a, bool f32,
                           cudaStream_t stream) {
  const BlockedPlan p = blocked_plan(s);
  a.rows = s.rows;
  a.nslabs = p.nslabs;
  a.dim = s.dim;
  a.group = s.G;
  a.rpi = p.rpi;
  a.tpr = p.tpr;
  const void* fn = hadq::blocked_kernel_ptr(direction, s.bits, s.B, s.has_signs, f32, p.threads);
  const size_t smem = direction == 0 ? p.smem : 0;
  int res = 1;
  const hadq_status pst = prepare(fn, p.threads, smem, "blocked kernel", &res);
  if (pst != HADQ_OK) return pst;
  const int64_t cap = int64_t(res) * sm_count();
  const unsigned grid = (unsigned)(p.nslabs < cap ? p.nslabs : cap);
  void* args[] = {&a};
  cudaError_t e = cudaLaunchKernel(fn, dim3(grid), dim3(p.threads), args, smem, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return fail(HADQ_ERR_CUDA, "blocked kernel launch failed: %s", cudaGetErrorString(e));
  }
  return after_launch("blocked kernel");
}

// ----------------------------------------------------------------- chunk

// `ka` carries the kept-token table when `keep`; the plain kernels read only
// its ChunkArgs base (the first bytes of the struct).
hadq_status launch_chunk_args(int direction, const Shape& s, hadq::ChunkKeepArgs ka, bool keep, bool f32,
                              cudaStream_t stream) {
  hadq::ChunkArgs& a = ka;
  a.cpr = s.dim / hadq::kCK;
  a.nchunks = s.rows * a.cpr;
  a.G = s.G;
  a.dim = s.dim;
  a.log_g = s.G <= hadq::kCK ? ilog2(s.G) : -1;
  a.gpc = s.G > hadq::kCK ? s.G / hadq::kCK : 1;
  // Warp teams (slabs of 32 chunks) unless a scale group spans a chunk count
  // that does not divide 32; the dequantiser needs no group reduction.
  const int team = (direction == 1 || (32 % a.gpc) == 0) ? 32 : hadq::kCT;
  a.slab_chunks = team == 32 ? 32 : (hadq::kCT / a.gpc) * a.gpc;  // a slab never splits a group
  const void* fn;
  if (keep)  // kept tokens: groups of >= 128 columns on warp teams (checked by the caller)
    fn = direction == 0 ? hadq::keep_chunk_kernel_ptr(s.bits, s.B, s.has_signs)
                        : hadq::keep_dq_chunk_kernel_ptr(s.bits, s.B, s.has_signs, f32);
  else
    fn = direction == 0 ? hadq::chunk_kernel_ptr(s.bits, s.B, s.has_signs, s.G >= hadq::kCK, team)
                        : hadq::dq_chunk_kernel_ptr(s.bits, s.B, s.has_signs, s.G < s.B, f32);
  const size_t smem = hadq::chunk_smem_bytes(s.dim, s.has_signs, direction == 0 && team != 32);
  int res = 1;
  const hadq_status pst = prepare(fn, hadq::kCT, smem, "chunk kernel", &res);
  if (pst != HADQ_OK) return pst;
  const int64_t cap = int64_t(res) * sm_count();
  cudaError_t e;
  const int64_t teams = team == 32 ? hadq::kCT / 32 : 1;
  const int64_t want = ((a.nchunks + a.slab_chunks - 1) / a.slab_chunks + teams - 1) / teams;  // CTAs for one slab per team
  const unsigned grid = (unsigned)(want < cap ? want : cap);
  void* args[] = {&ka};
  e = cudaLaunchKernel(fn, dim3(grid), dim3(hadq::kCT), args, smem, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return fail(HADQ_ERR_CUDA, "chunk kernel launch failed: %s", cudaGetErrorString(e));
  }
  return after_launch("chunk kernel");
}

hadq_status launch_chunk(int direction, const Shape& s, hadq::ChunkArgs a, bool f32, cudaStream_t stream) {
  hadq::ChunkKeepArgs ka{};
  static_cast<hadq::ChunkArgs&>(ka) = a;
  return launch_chunk_args(direction, s, ka, false, f32, stream);
}

// `ka` carries the kept-token table when `keep`; the plain kernels read only
// its ChunkArgs base.
hadq_status launch_chunk_mma_args(const Shape& s, hadq::ChunkKeepArgs ka, bool keep, cudaStream_t stream) {
  hadq::ChunkArgs& a = ka;
  a.cpr = s.dim / hadq::kCK;
  a.nchunks = s.rows * a.cpr;
  a.slab_chunks = hadq::kMmaSlab;
  a.G = s.G;
  a.dim = s.dim;
  a.log_g = 7;
  a.gpc = 1;
  const void* fn = keep ? hadq::keep_chunk_mma_kernel_ptr(s.bits, s.has_signs)
                        : hadq::chunk_mma_kernel_ptr(s.bits, s.has_signs, a.rot != nullptr);
  const size_t smem = hadq::chunk_mma_smem_bytes(s.dim, s.has_signs);
  const int threads = hadq::kMmaWarps * 32;
  int res = 1;
  const hadq_status pst = prepare(fn, threads, smem, "128-block tensor-core kernel", &res);
  if (pst != HADQ_OK) return pst;
  const int64_t cap = int64_t(res) * sm_count();
  cudaError_t e;
  const int64_t slabs = (a.nchunks + hadq::kMmaSlab - 1) / hadq::kMmaSlab;
  const int64_t want = (slabs + hadq::kMmaWarps - 1) / hadq::kMmaWarps;  // one slab per warp
  const unsigned grid = (unsigned)(want < cap ? want : cap);
  void* args[] = {&ka};
  e = cudaLaunchKernel(fn, dim3(grid), dim3(threads), args, smem, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return fail(HADQ_ERR_CUDA, "128-block tensor-core kernel launch failed: %s", cudaGetErrorString(e));
  }
  return after_launch("128-block tensor-core kernel");
}

hadq_status launch_chunk_mma(const Shape& s, hadq::ChunkArgs a, cudaStream_t stream) {
  hadq::ChunkKeepArgs ka{};
  static_cast<hadq::ChunkArgs&>(ka) = a;
  return launch_chunk_mma_args(s, ka, false, stream);
}

hadq_status launch_dq_chunk_mma(const Shape& s, hadq::ChunkArgs a, bool f32, cudaStream_t stream) {
  a.cpr = s.dim / hadq::kCK;
  a.nchunks = s.rows * a.cpr;
  a.slab_chunks = 32;
  a.G = s.G;
  a.dim = s.dim;
  a.log_g = -1;
  a.gpc = s.G / hadq::kCK;
  const void* fn = hadq::dq_chunk_mma_kernel_ptr(s.bits, s.has_signs, f32);
  const size_t smem = hadq::dq_mma_smem_bytes(s.bits, s.dim, s.has_signs);
  int res = 1;
  const hadq_status pst = prepare(fn, hadq::kCT, smem, "128-block tensor-core inverse", &res);
  if (pst != HADQ_OK) return pst;
  const int64_t cap = int64_t(res) * sm_count();
  const int64_t want = ((a.nchunks + 31) / 32 + 3) / 4;  // one slab of 32 blocks per warp
  const unsigned grid = (unsigned)(want < cap ? want : cap);
  void* args[] = {&a};
  cudaError_t e = cudaLaunchKernel(fn, dim3(grid), dim3(hadq::kCT), args, smem, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return fail(HADQ_ERR_CUDA, "128-block tensor-core inverse launch failed: %s", cudaGetErrorString(e));
  }
  return after_launch("128-block tensor-core inverse");
}

// One persistent CTA per SM (the kernel holds all 512 TMEM columns and most
// of the shared memory), over tiles of four 4096-point blocks.
hadq_status launch_h4096_tc(const Shape& s, const void* x, const int8_t* signs, uint8_t* codes, float* scales,
                            float scale_mul, cudaStream_t stream, int stall_tile = -1) {
  hadq::TcArgs a{};
  a.stall_tile = stall_tile;
  a.nblocks = s.rows * (s.dim / 4096);
  a.ntiles = (a.nblocks + hadq::kTcTileBlocks - 1) / hadq::kTcTileBlocks;
  a.signs = signs;
  a.codes = codes;
  a.scales = scales;
  a.scale_mul = scale_mul;
  a.fault = hadq::tc_fault_word();
  if (!a.fault) return fail(HADQ_ERR_CUDA, "tcgen05 4096-block kernel: the fault word has no device address");
  CUtensorMap map;
  if (!hadq::h4096_tc_encode_map(&map, x, a.nblocks))
    return fail(HADQ_ERR_CUDA, "tcgen05 4096-block kernel: cuTensorMapEncodeTiled failed");
  const void* fn = hadq::h4096_tc_kernel_ptr(s.bits, s.has_signs);
  const size_t smem = hadq::h4096_tc_smem();
  const int threads = hadq::h4096_tc_threads();
  int res = 1;
  const hadq_status pst = prepare(fn, threads, smem, "tcgen05 4096-block kernel", &res);
  if (pst != HADQ_OK) return pst;
  const int64_t cap = sm_count();
  const unsigned grid = (unsigned)(a.ntiles < cap ? a.ntiles : cap);
  void* args[] = {&map, &a};
  const cudaError_t e = cudaLaunchKernel(fn, dim3(grid), dim3(threads), args, smem, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return fail(HADQ_ERR_CUDA, "tcgen05 4096-block kernel launch failed: %s", cudaGetErrorString(e));
  }
  return after_launch("tcgen05 4096-block kernel");
}

hadq_status launch_wide4096(const Shape& s, hadq::ChunkArgs a, cudaStream_t stream, bool mma) {
  a.cpr = s.dim / hadq::kCK;
  a.nchunks = s.rows * a.cpr;
  a.slab_chunks = 32;
  a.G = s.G;
  a.dim = s.dim;
  a.log_g = -1;
  a.gpc = 32;
  const void* fn = mma ? hadq::h4096_mma_kernel_ptr(s.bits, s.has_signs, a.rot != nullptr) : hadq::wide4096_kernel_ptr(s.bits, s.has_signs);
  const size_t smem = mma ? hadq::h4096_smem_bytes(s.has_signs) : hadq::chunk_smem_bytes(s.dim, s.has_signs, false);
  const int threads = mma ? hadq::kH4096Warps * 32 : hadq::kCT;
  int res = 1;
  const hadq_status pst = prepare(fn, threads, smem, "4096-block kernel", &res);
  if (pst != HADQ_OK) return pst;
  const int64_t cap = int64_t(res) * sm_count();
  cudaError_t e;
  const int64_t want = (a.nchunks / 32 + threads / 32 - 1) / (threads / 32);  // one block per warp
  const unsigned grid = (unsigned)(want < cap ? want : cap);
  void* args[] = {&a};
  e = cudaLaunchKernel(fn, dim3(grid), dim3(threads), args, smem, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return fail(HADQ_ERR_CUDA, "4096-block kernel launch failed: %s", cudaGetErrorString(e));
  }
  return after_launch("4096-block kernel");
}

// ------------------------------------------------------------------ 4096

hadq_status launch_full4096(const Shape& s, hadq::FullArgs a, cudaStream_t stream) {
  a.rows = s.rows;
  const int lg = ilog2(s.G);
  const void* fn = hadq::full4096_kernel_ptr(s.bits, s.has_signs, lg);
  int res = 1;
  const hadq_status pst = prepare(fn, 64, 0, "4096-point kernel", &res);
  if (pst != HADQ_OK) return pst;
  const int64_t cap = int64_t(res) * sm_count();
  const unsigned grid = (unsigned)(s.rows < cap ? s.rows : cap);
  void* args[] = {&a};
  cudaError_t e = cudaLaunchKernel(fn, dim3(grid), dim3(64), args, 0, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return fail(HADQ_ERR_CUDA, "4096-point kernel launch failed: %s", cudaGetErrorString(e));
  }
  return after_launch("4096-point kernel");
}

// --------------------------------------------------------------- generic

hadq_status launch_generic(int direction, const Shape& s, hadq::GenericArgs a, bool f32,
                           cudaStream_t stream) {
  a.rows = s.rows;
  a.dim = s.dim;
  a.block = s.B;
  a.group = s.G;
  const void* fn;
  size_t smem;
  if (direction == 0) {
    fn = hadq::generic_kernel_ptr(0, s.bits);
    smem = size_t(s.dim) * 4 + ((size_t(s.dim) + 15) & ~size_t(15));
  } else {
    fn = hadq::generic_kernel_ptr(1, s.bits);
    smem = size_t(s.dim) * 4 + ((size_t(s.dim / s.B) + 15) & ~size_t(15));
  }
  int res = 1;
  const hadq_status pst = prepare(fn, 256, smem, "generic kernel", &res);
  if (pst != HADQ_OK) return pst;
  const int64_t cap = int64_t(res) * sm_count();
  const unsigned grid = (unsigned)(s.rows < cap ? s.rows : cap);
  cudaError_t e;
  if (direction == 0) {
    void* args[] = {&a};
    e = cudaLaunchKernel(fn, dim3(grid), dim3(256), args, smem, stream);
  } else {
    bool out_f32 = f32;
    void* args[] = {&a, &out_f32};
    e = cudaLaunchKernel(fn, dim3(grid), dim3(256), args, smem, stream);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return fail(HADQ_ERR_CUDA, "generic kernel launch failed: %s", cudaGetErrorString(e));
  }
  return after_launch("generic kernel");
}

// ------------------------------------------------------ decode attention

struct AttnShape {
  int64_t groups;  // batch * n_kv_heads * query-head groups of 4
  int hgroups;
  int max_splits;  // upper bound used for the workspace size
};

hadq_status attn_check(int32_t batch, int32_t nqh, int32_t nkv, int64_t tokens, AttnShape* s) {
  if (batch < 0) return fail(HADQ_ERR_INVALID_ARG, "batch must be >= 0 (got %d)", batch);
  if (nqh < 1 || nkv < 1)
    return fail(HADQ_ERR_INVALID_ARG, "n_q_heads and n_kv_heads must be >= 1 (got %d, %d)", nqh, nkv);
  if (nqh % nkv)
    return fail(HADQ_ERR_INVALID_ARG, "n_q_heads %d is not a multiple of n_kv_heads %d", nqh, nkv);
  if (tokens < 1) return fail(HADQ_ERR_INVALID_ARG, "tokens must be >= 1 (got %lld)", (long long)tokens);
  if (tokens > (int64_t(1) << 30))
    return fail(HADQ_ERR_UNSUPPORTED, "tokens must be at most 2^30 (got %lld)", (long long)tokens);
  const int g = nqh / nkv;
  s->hgroups = (g + hadq::kAttnHeads - 1) / hadq::kAttnHeads;
  s->groups = int64_t(batch) * nkv * s->hgroups;
  if (s->groups > 65535)
    return fail(HADQ_ERR_UNSUPPORTED, "batch * n_kv_heads * ceil(group/4) = %lld exceeds 65535",
                (long long)s->groups);
  const int64_t by_tokens = (tokens + 63) / 64;
  s->max_splits = int(by_tokens < hadq::kAttnMaxSplits ? by_tokens : hadq::kAttnMaxSplits);
  return HADQ_OK;
}

size_t round256(size_t v) { return (v + 255) & ~size_t(255); }

// Workspace layout: counters [groups], then (m, l) [groups][splits][4][2],
// then O [groups][splits][4][128], each part 256-byte aligned.
size_t attn_ws_bytes(int64_t groups, int splits, size_t* off_ml, size_t* off_o) {
  const size_t c = round256(size_t(groups) * sizeof(unsigned));
  const size_t ml = round256(size_t(groups) * splits * hadq::kAttnHeads * 2 * sizeof(float));
  const size_t o = size_t(groups) * splits * hadq::kAttnHeads * hadq::kAttnDim * sizeof(float);
  if (off_ml) *off_ml = c;
  if (off_o) *off_o = c + ml;
  return c + ml + o;
}

hadq_status attn_call(const void* q, const void* k_codes, const float* k_scales, const void* v_codes,
                      const float* v_scales, int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                      int64_t tokens, int64_t token_stride, int32_t dim, int32_t block, const int8_t* signs,
                      int32_t bits, int32_t group, float softmax_scale, void* out, hadq_out_dtype out_dtype,
                      void* workspace, size_t workspace_bytes, bool static_scratch, hadq_stream_t stream) {
  AttnShape as;
  hadq_status st = attn_check(batch, n_q_heads, n_kv_heads, tokens, &as);
  if (st != HADQ_OK) return st;
  if (token_stride < tokens)
    return fail(HADQ_ERR_INVALID_ARG, "token_stride %lld is below tokens %lld", (long long)token_stride,
                (long long)tokens);
  Shape s;
  st = check_sizes(int64_t(batch) * n_q_heads, dim, block, bits, group, &s);
  if (st != HADQ_OK) return st;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    return fail(HADQ_ERR_INVALID_ARG, "softmax_scale must be positive and finite");
  if (out_dtype != HADQ_OUT_BF16 && out_dtype != HADQ_OUT_F32)
    return fail(HADQ_ERR_INVALID_ARG, "out_dtype must be HADQ_OUT_BF16 or HADQ_OUT_F32");
  if (dim != hadq::kAttnDim || s.B != hadq::kAttnDim || (s.G != 128 && s.G != 64 && s.G != 32))
    return fail(HADQ_ERR_UNSUPPORTED,
                "decode attention supports dim 128, block 128, group 128, 64 or 32 (got %d, %d, %d)", dim, s.B,
                s.G);
  const int ng = hadq::kAttnDim / s.G;  // scales per cached row
  if (batch == 0) return HADQ_OK;
  if (!q || !k_codes || !k_scales || !v_codes || !v_scales || !out || (!workspace && !static_scratch))
    return fail(HADQ_ERR_INVALID_ARG, "q, codes, scales, out and workspace must not be NULL");
  const bool f32 = out_dtype == HADQ_OUT_F32;
  if (!aligned(q, 8)) return fail(HADQ_ERR_MISALIGNED, "q must be 8-byte aligned");
  if (!aligned(k_codes, 16) || !aligned(v_codes, 16))
    return fail(HADQ_ERR_MISALIGNED, "k_codes and v_codes must be 16-byte aligned");
  if (!aligned(k_scales, 4) || !aligned(v_scales, 4))
    return fail(HADQ_ERR_MISALIGNED, "k_scales and v_scales must be 4-byte aligned");
  if (ng > 1 && (!aligned(k_scales, 16) || !aligned(v_scales, 16) || (token_stride * ng) % 4 != 0))
    return fail(HADQ_ERR_MISALIGNED,
                "with groups below 128 the scale arrays must be 16-byte aligned and token_stride * 128 / group "
                "a multiple of 4");
  if (signs && !aligned(signs, 4)) return fail(HADQ_ERR_MISALIGNED, "signs must be 4-byte aligned");
  if (!aligned(out, f32 ? 16 : 8))
    return fail(HADQ_ERR_MISALIGNED, "out must be %d-byte aligned", f32 ? 16 : 8);
  if (!static_scratch && !aligned(workspace, 256))
    return fail(HADQ_ERR_MISALIGNED, "workspace must be 256-byte aligned");

  const void* fn = hadq::kv_decode_attn_kernel_ptr(ng, bits);
  const size_t smem = hadq::kv_decode_attn_smem(ng, bits);
  // One wave of CTAs: split the tokens of each head group so that all CTAs
  // are resident at once (a CTA beyond the wave would run alone afterwards);
  // at least 64 tokens (a tile per warp) per split.
  int res = 1;
  const hadq_status pst = prepare(fn, hadq::kAttnThreads, smem, "decode attention kernel", &res);
  if (pst != HADQ_OK) return pst;
  const int64_t wave = int64_t(res) * sm_count();
  int64_t splits = wave / as.groups;
  if (splits > as.max_splits) splits = as.max_splits;
  if (splits < 1) splits = 1;
  int64_t chunk = (tokens + splits - 1) / splits;
  chunk = (chunk + hadq::kAttnTile - 1) / hadq::kAttnTile * hadq::kAttnTile;
  splits = (tokens + chunk - 1) / chunk;
  size_t off_ml = 0, off_o = 0;
  const size_t need = attn_ws_bytes(as.groups, int(splits), &off_ml, &off_o);
  if (static_scratch) {
    if (need > workspace_bytes)
      return fail(HADQ_ERR_UNSUPPORTED, "these sizes need %zu bytes of scratch, above the %zu bytes the library holds",
                  need, workspace_bytes);
    workspace = hadq::attn_static_scratch();
    if (!workspace) return fail(HADQ_ERR_CUDA, "cannot resolve the library's static scratch on this device");
  } else if (workspace_bytes < need) {
    return fail(HADQ_ERR_INVALID_ARG, "workspace of %zu bytes is below the %zu bytes needed", workspace_bytes,
                need);
  }

  hadq::AttnArgs a{};
  a.q = static_cast<const uint16_t*>(q);
  a.k_codes = static_cast<const uint8_t*>(k_codes);
  a.k_scales = k_scales;
  a.v_codes = static_cast<const uint8_t*>(v_codes);
  a.v_scales = v_scales;
  a.signs = signs;
  a.out = out;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.counters = reinterpret_cast<unsigned*>(ws);
  a.part_ml = reinterpret_cast<float*>(ws + off_ml);
  a.part_o = reinterpret_cast<float*>(ws + off_o);
  a.tokens = tokens;
  a.stride = token_stride;
  a.chunk = chunk;
  a.nqh = n_q_heads;
  a.nkv = n_kv_heads;
  a.g = n_q_heads / n_kv_heads;
  a.hgroups = as.hgroups;
  a.splits = int(splits);
  a.qmul = (float)(double(softmax_scale) * 1.4426950408889634 / std::sqrt(double(hadq::kAttnDim)));
  a.inv_sqrt_dim = (float)(1.0 / std::sqrt(double(hadq::kAttnDim)));
  a.out_f32 = f32 ? 1 : 0;
  a.vmask = bits == 8 ? 0x007F007Fu : 0x000F000Fu;
  a.vmagic = bits == 8 ? 0x43004300u : 0x43084308u;
  a.vsign = 0x00800080u;
  void* args[] = {&a};
  cudaError_t e = cudaLaunchKernel(fn, dim3(unsigned(splits), unsigned(as.groups)), dim3(hadq::kAttnThreads),
                                   args, smem, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    cudaGetLastError();
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return fail(HADQ_ERR_CUDA, "decode attention launch failed: %s", cudaGetErrorString(e));
  }
  return after_launch("decode attention kernel");
}

}  // namespace

extern "C" {

hadq_status hadq_plan(int32_t direction, int64_t rows, int32_t dim, int32_t block, int32_t bits,
                      int32_t group, int32_t has_signs, int32_t aligned16, hadq_path* path) {
  if (direction != 0 && direction != 1)
    return fail(HADQ_ERR_INVALID_ARG, "direction must be 0 or 1 (got %d)", direction);
  Shape s;
  hadq_status st = check_sizes(rows, dim, block, bits, group, &s);
  if (st != HADQ_OK) return st;
  s.has_signs = has_signs != 0;
  if (path) *path = choose_path(direction, s, aligned16 != 0);
  return HADQ_OK;
}

hadq_status hadq_rotate_quantize(const void* x, int64_t rows, int32_t dim, int32_t block,
                                 const int8_t* signs, int32_t bits, int32_t group, void* codes,
                                 float* scales, float* rotated_out, hadq_stream_t stream) {
  g_last_error.clear();
  Shape s;
  hadq_status st = check_sizes(rows, dim, block, bits, group, &s);
  if (st != HADQ_OK) return st;
  s.has_signs = signs != nullptr;
  if (rows == 0) return HADQ_OK;
  if (!x || !codes || !scales)
    return fail(HADQ_ERR_INVALID_ARG, "x, codes and scales must not be NULL");
  if (!aligned(x, 2)) return fail(HADQ_ERR_MISALIGNED, "x must be 2-byte aligned");
  if (!aligned(scales, 4)) return fail(HADQ_ERR_MISALIGNED, "scales must be 4-byte aligned");
  if (rotated_out && !aligned(rotated_out, 4))
    return fail(HADQ_ERR_MISALIGNED, "rotated_out must be 4-byte aligned");
  const bool a16 = aligned(x, 16) && aligned(codes, 16) && (!signs || aligned(signs, 16)) &&
                   (!rotated_out || aligned(rotated_out, 16));
  hadq_path path = choose_path(0, s, a16);
  if (path == HADQ_PATH_H4096_TC && rotated_out) path = HADQ_PATH_WIDE4096_MMA;
  const double qmax = double((1 << (bits - 1)) - 1);
  const float scale_mul = (float)(1.0 / (std::sqrt(double(s.B)) * qmax));
  const float rsqrt_b = (float)(1.0 / std::sqrt(double(s.B)));
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (path == HADQ_PATH_BLOCKED) {
    hadq::BlockedArgs a{};
    a.x = static_cast<const uint16_t*>(x);
    a.signs = signs;
    a.codes = static_cast<uint8_t*>(codes);
    a.scales = scales;
    a.rot = rotated_out;
    a.scale_mul = scale_mul;
    a.rsqrt_b = rsqrt_b;
    return launch_blocked(0, s, a, false, cs);
  }
  if (path == HADQ_PATH_CHUNK) {
    hadq::ChunkArgs a{};
    a.x = static_cast<const uint16_t*>(x);
    a.signs = signs;
    a.codes = static_cast<uint8_t*>(codes);
    a.scales = scales;
    a.rot = rotated_out;
    a.scale_mul = scale_mul;
    a.rsqrt_b = rsqrt_b;
    return launch_chunk(0, s, a, false, cs);
  }
  if (path == HADQ_PATH_CHUNK_MMA) {
    hadq::ChunkArgs a{};
    a.x = static_cast<const uint16_t*>(x);
    a.signs = signs;
    a.codes = static_cast<uint8_t*>(codes);
    a.scales = scales;
    a.rot = rotated_out;
    a.scale_mul = scale_mul;
    a.rsqrt_b = rsqrt_b;
    return launch_chunk_mma(s, a, cs);
  }
  if (path == HADQ_PATH_H4096_TC)
    return launch_h4096_tc(s, x, signs, static_cast<uint8_t*>(codes), scales, scale_mul, cs);
  if (path == HADQ_PATH_WIDE4096 || path == HADQ_PATH_WIDE4096_MMA) {
    hadq::ChunkArgs a{};
    a.x = static_cast<const uint16_t*>(x);
    a.signs = signs;
    a.codes = static_cast<uint8_t*>(codes);
    a.scales = scales;
    a.rot = rotated_out;
    a.scale_mul = scale_mul;
    a.rsqrt_b = rsqrt_b;
    return launch_wide4096(s, a, cs, path == HADQ_PATH_WIDE4096_MMA);
  }
  if (path == HADQ_PATH_FULL4096) {
    hadq::FullArgs a{};
    a.x = static_cast<const uint16_t*>(x);
    a.signs = signs;
    a.codes = static_cast<uint8_t*>(codes);
    a.scales = scales;
    a.rot = rotated_out;
    a.scale_mul = scale_mul;
    a.rsqrt_b = rsqrt_b;
    return launch_full4096(s, a, cs);
  }
  hadq::GenericArgs a{};
  a.x = static_cast<const uint16_t*>(x);
  a.signs = signs;
  a.codes = static_cast<uint8_t*>(codes);
  a.scales = scales;
  a.rot = rotated_out;
  a.scale_mul = scale_mul;
  a.rsqrt_b = rsqrt_b;
  return launch_generic(0, s, a, false, cs);
}

hadq_status hadq_dequant_rotate_inv(const void* codes, const float* scales, int64_t rows,
                                    int32_t dim, int32_t block, const int8_t* signs, int32_t bits,
                                    int32_t group, void* out, hadq_out_dtype out_dtype,
                                    hadq_stream_t stream) {
  g_last_error.clear();
  Shape s;
  hadq_status st = check_sizes(rows, dim, block, bits, group, &s);
  if (st != HADQ_OK) return st;
  if (out_dtype != HADQ_OUT_BF16 && out_dtype != HADQ_OUT_F32)
    return fail(HADQ_ERR_INVALID_ARG, "out_dtype must be HADQ_OUT_BF16 or HADQ_OUT_F32");
  s.has_signs = signs != nullptr;
  if (rows == 0) return HADQ_OK;
  if (!codes || !scales || !out) return fail(HADQ_ERR_INVALID_ARG, "codes, scales and out must not be NULL");
  const bool f32 = out_dtype == HADQ_OUT_F32;
  if (!aligned(scales, 4)) return fail(HADQ_ERR_MISALIGNED, "scales must be 4-byte aligned");
  if (!aligned(out, f32 ? 4 : 2)) return fail(HADQ_ERR_MISALIGNED, "out must be aligned to its element size");
  const bool a16 = aligned(codes, 16) && aligned(out, 16) && (!signs || aligned(signs, 16));
  const hadq_path path = choose_path(1, s, a16);
  const float rsqrt_b = (float)(1.0 / std::sqrt(double(s.B)));
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (path == HADQ_PATH_CHUNK_MMA) {
    hadq::ChunkArgs a{};
    a.codes_in = static_cast<const uint8_t*>(codes);
    a.scales_in = scales;
    a.signs = signs;
    a.rot = f32 ? static_cast<float*>(out) : nullptr;
    a.out_bf16 = f32 ? nullptr : static_cast<uint16_t*>(out);
    a.rsqrt_b = rsqrt_b;
    return launch_dq_chunk_mma(s, a, f32, cs);
  }
  if (path == HADQ_PATH_CHUNK) {
    hadq::ChunkArgs a{};
    a.codes_in = static_cast<const uint8_t*>(codes);
    a.scales_in = scales;
    a.signs = signs;
    a.rot = f32 ? static_cast<float*>(out) : nullptr;
    a.out_bf16 = f32 ? nullptr : static_cast<uint16_t*>(out);
    a.rsqrt_b = rsqrt_b;
    return launch_chunk(1, s, a, f32, cs);
  }
  if (path == HADQ_PATH_BLOCKED) {
    hadq::BlockedArgs a{};
    a.codes_in = static_cast<const uint8_t*>(codes);
    a.scales_in = scales;
    a.signs = signs;
    a.rot = f32 ? static_cast<float*>(out) : nullptr;
    a.out_bf16 = f32 ? nullptr : static_cast<uint16_t*>(out);
    a.rsqrt_b = rsqrt_b;
    return launch_blocked(1, s, a, f32, cs);
  }
  hadq::GenericArgs a{};
  a.codes_in = static_cast<const uint8_t*>(codes);
  a.scales_in = scales;
  a.signs = signs;
  a.rot = f32 ? static_cast<float*>(out) : nullptr;
  a.out_bf16 = f32 ? nullptr : static_cast<uint16_t*>(out);
  a.rsqrt_b = rsqrt_b;
  return launch_generic(1, s, a, f32, cs);
}

hadq_status hadq_kv_decode_workspace_size(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                          int64_t tokens, size_t* bytes) {
  g_last_error.clear();
  AttnShape a;
  hadq_status st = attn_check(batch, n_q_heads, n_kv_heads, tokens, &a);
  if (st != HADQ_OK) return st;
  if (!bytes) return fail(HADQ_ERR_INVALID_ARG, "bytes must not be NULL");
  *bytes = a.groups ? attn_ws_bytes(a.groups, a.max_splits, nullptr, nullptr) : 0;
  return HADQ_OK;
}

hadq_status hadq_kv_decode_attention(const void* q, const void* k_codes, const float* k_scales,
                                     const void* v_codes, const float* v_scales, int32_t batch,
                                     int32_t n_q_heads, int32_t n_kv_heads, int64_t tokens,
                                     int64_t token_stride, int32_t dim, int32_t block,
                                     const int8_t* signs, int32_t bits, int32_t group,
                                     float softmax_scale, void* out, hadq_out_dtype out_dtype,
                                     void* workspace, size_t workspace_bytes, hadq_stream_t stream) {
  g_last_error.clear();
  return attn_call(q, k_codes, k_scales, v_codes, v_scales, batch, n_q_heads, n_kv_heads, tokens, token_stride,
                   dim, block, signs, bits, group, softmax_scale, out, out_dtype, workspace, workspace_bytes,
                   false, stream);
}

hadq_status hadq_kv_decode_attention_noalloc(const void* q, const void* k_codes, const float* k_scales,
                                             const void* v_codes, const float* v_scales, int32_t batch,
                                             int32_t n_q_heads, int32_t n_kv_heads, int64_t tokens,
                                             int64_t token_stride, int32_t dim, int32_t block,
                                             const int8_t* signs, int32_t bits, int32_t group,
                                             float softmax_scale, void* out, hadq_out_dtype out_dtype,
                                             hadq_stream_t stream) {
  g_last_error.clear();
  return attn_call(q, k_codes, k_scales, v_codes, v_scales, batch, n_q_heads, n_kv_heads, tokens, token_stride,
                   dim, block, signs, bits, group, softmax_scale, out, out_dtype, nullptr,
                   hadq::kAttnStaticScratchBytes, true, stream);
}

// Mixed-precision (kept-token) variants: the chunk kernels with a keep table.
static hadq_status keep_check(const Shape& s, int64_t heads, int64_t tokens, const int32_t* keep_slot,
                              int32_t n_keep, const void* kept, bool a16) {
  if (heads < 0 || tokens < 0)
    return fail(HADQ_ERR_INVALID_ARG, "heads and tokens must be >= 0 (got %lld, %lld)", (long long)heads,
                (long long)tokens);
  if (n_keep < 0) return fail(HADQ_ERR_INVALID_ARG, "n_keep must be >= 0 (got %d)", n_keep);
  if (s.rows == 0) return HADQ_OK;
  if (!keep_slot) return fail(HADQ_ERR_INVALID_ARG, "keep_slot must not be NULL");
  if (n_keep > 0 && !kept) return fail(HADQ_ERR_INVALID_ARG, "kept must not be NULL when n_keep > 0");
  if (!aligned(keep_slot, 4)) return fail(HADQ_ERR_MISALIGNED, "keep_slot must be 4-byte aligned");
  if (kept && !aligned(kept, 16)) return fail(HADQ_ERR_MISALIGNED, "kept must be 16-byte aligned");
  const int gpc = s.G >= hadq::kCK ? s.G / hadq::kCK : 0;
  if (!a16 || !chunk_ok(0, s) || s.G % hadq::kCK != 0 || 32 % gpc != 0 ||
      s.rows * (s.dim / hadq::kCK) >= (int64_t(1) << 31))
    return fail(HADQ_ERR_UNSUPPORTED,
                "kept tokens need the chunk kernels with wide groups: dim a multiple of 128, block 8..128, "
                "group 128 x (1, 2, 4, .., 32) columns, fewer than 2^31 chunks of 128, 16-byte-aligned buffers");
  return HADQ_OK;
}

// Kept-token quantise calls that the 128-point tensor-core kernel takes.
static bool keep_mma_ok(const Shape& s) {
  return s.B == 128 && s.G == 128 && s.dim % 128 == 0 && s.rows * (s.dim / 128) < (int64_t(1) << 30);
}

hadq_status hadq_rotate_quantize_keep(const void* x, int64_t heads, int64_t tokens, int32_t dim, int32_t block,
                                      const int8_t* signs, int32_t bits, int32_t group, const int32_t* keep_slot,
                                      int32_t n_keep, void* codes, float* scales, void* kept,
                                      hadq_stream_t stream) {
  g_last_error.clear();
  if (heads < 0 || tokens < 0 || (tokens > 0 && heads > INT64_MAX / tokens))
    return fail(HADQ_ERR_INVALID_ARG, "heads and tokens must be >= 0 (got %lld, %lld)", (long long)heads,
                (long long)tokens);
  Shape s;
  hadq_status st = check_sizes(heads * tokens, dim, block, bits, group, &s);
  if (st != HADQ_OK) return st;
  s.has_signs = signs != nullptr;
  if (s.rows > 0 && (!x || !codes || !scales))
    return fail(HADQ_ERR_INVALID_ARG, "x, codes and scales must not be NULL");
  if (s.rows > 0 && !aligned(scales, 4)) return fail(HADQ_ERR_MISALIGNED, "scales must be 4-byte aligned");
  const bool a16 = aligned(x, 16) && aligned(codes, 16) && (!signs || aligned(signs, 16));
  st = keep_check(s, heads, tokens, keep_slot, n_keep, kept, a16);
  if (st != HADQ_OK || s.rows == 0) return st;
  const double qmax = double((1 << (bits - 1)) - 1);
  hadq::ChunkKeepArgs a{};
  a.x = static_cast<const uint16_t*>(x);
  a.signs = signs;
  a.codes = static_cast<uint8_t*>(codes);
  a.scales = scales;
  a.scale_mul = (float)(1.0 / (std::sqrt(double(s.B)) * qmax));
  a.rsqrt_b = (float)(1.0 / std::sqrt(double(s.B)));
  a.keep_slot = keep_slot;
  a.kept = static_cast<uint16_t*>(kept);
  a.keep_tokens = tokens;
  a.n_keep = n_keep;
  // 128-point blocks with one scale per block take the tensor-core quantiser
  // (32-bit chunk indices), the rest the chunk kernels
  if (keep_mma_ok(s)) return launch_chunk_mma_args(s, a, true, reinterpret_cast<cudaStream_t>(stream));
  return launch_chunk_args(0, s, a, true, false, reinterpret_cast<cudaStream_t>(stream));
}

hadq_status hadq_dequant_rotate_inv_keep(const void* codes, const float* scales, const void* kept,
                                         const int32_t* keep_slot, int32_t n_keep, int64_t heads, int64_t tokens,
                                         int32_t dim, int32_t block, const int8_t* signs, int32_t bits,
                                         int32_t group, void* out, hadq_out_dtype out_dtype,
                                         hadq_stream_t stream) {
  g_last_error.clear();
  if (heads < 0 || tokens < 0 || (tokens > 0 && heads > INT64_MAX / tokens))
    return fail(HADQ_ERR_INVALID_ARG, "heads and tokens must be >= 0 (got %lld, %lld)", (long long)heads,
                (long long)tokens);
  Shape s;
  hadq_status st = check_sizes(heads * tokens, dim, block, bits, group, &s);
  if (st != HADQ_OK) return st;
  if (out_dtype != HADQ_OUT_BF16 && out_dtype != HADQ_OUT_F32)
    return fail(HADQ_ERR_INVALID_ARG, "out_dtype must be HADQ_OUT_BF16 or HADQ_OUT_F32");
  s.has_signs = signs != nullptr;
  if (s.rows > 0 && (!codes || !scales || !out))
    return fail(HADQ_ERR_INVALID_ARG, "codes, scales and out must not be NULL");
  if (s.rows > 0 && !aligned(scales, 4)) return fail(HADQ_ERR_MISALIGNED, "scales must be 4-byte aligned");
  const bool a16 = aligned(codes, 16) && aligned(out, 16) && (!signs || aligned(signs, 16));
  st = keep_check(s, heads, tokens, keep_slot, n_keep, kept, a16);
  if (st != HADQ_OK || s.rows == 0) return st;
  const bool f32 = out_dtype == HADQ_OUT_F32;
  hadq::ChunkKeepArgs a{};
  a.codes_in = static_cast<const uint8_t*>(codes);
  a.scales_in = scales;
  a.signs = signs;
  a.rot = f32 ? static_cast<float*>(out) : nullptr;
  a.out_bf16 = f32 ? nullptr : static_cast<uint16_t*>(out);
  a.rsqrt_b = (float)(1.0 / std::sqrt(double(s.B)));
  a.keep_slot = keep_slot;
  a.kept = static_cast<uint16_t*>(const_cast<void*>(kept));
  a.keep_tokens = tokens;
  a.n_keep = n_keep;
  return launch_chunk_args(1, s, a, true, f32, reinterpret_cast<cudaStream_t>(stream));
}

// Asymmetric (zero-point) variants: the chunk pipeline with range-derived
// scale and zero point.
static hadq_status asym_coverage(const Shape& s, bool a16) {
  const int gpc = s.G >= hadq::kCK ? s.G / hadq::kCK : 0;
  if (!a16 || s.B < 8 || s.B > hadq::kCK || s.dim % hadq::kCK != 0 || s.G % hadq::kCK != 0 || 32 % gpc != 0)
    return fail(HADQ_ERR_UNSUPPORTED,
                "the asymmetric quantiser needs dim a multiple of 128, block 8..128, group 128 x (1, 2, 4, .., "
                "32) columns and 16-byte-aligned x/codes/out/signs");
  return HADQ_OK;
}

static hadq_status launch_asym(int direction, const Shape& s, hadq::ChunkAsymArgs a, bool f32, cudaStream_t stream) {
  a.cpr = s.dim / hadq::kCK;
  a.nchunks = s.rows * a.cpr;
  a.slab_chunks = 32;
  a.G = s.G;
  a.gpc = s.G / hadq::kCK;
  a.dim = s.dim;
  a.log_g = -1;
  const void* fn = direction == 0 ? hadq::asym_chunk_kernel_ptr(s.bits, s.B, s.has_signs)
                                  : hadq::asym_dq_chunk_kernel_ptr(s.bits, s.B, s.has_signs, f32);
  const size_t smem = hadq::chunk_smem_bytes(s.dim, s.has_signs, false);
  int res = 1;
  const hadq_status pst = prepare(fn, hadq::kCT, smem, "asymmetric kernel", &res);
  if (pst != HADQ_OK) return pst;
  const int64_t cap = int64_t(res) * sm_count();
  cudaError_t e;
  const int64_t want = ((a.nchunks + 31) / 32 + 3) / 4;  // one slab per warp
  const unsigned grid = (unsigned)(want < cap ? want : cap);
  void* args[] = {&a};
  e = cudaLaunchKernel(fn, dim3(grid), dim3(hadq::kCT), args, smem, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return fail(HADQ_ERR_CUDA, "asymmetric kernel launch failed: %s", cudaGetErrorString(e));
  }
  return after_launch("asymmetric kernel");
}

hadq_status hadq_rotate_quantize_asym(const void* x, int64_t rows, int32_t dim, int32_t block, const int8_t* signs,
                                      int32_t bits, int32_t group, void* codes, float* scales,
                                      uint8_t* zero_points, hadq_stream_t stream) {
  g_last_error.clear();
  Shape s;
  hadq_status st = check_sizes(rows, dim, block, bits, group, &s);
  if (st != HADQ_OK) return st;
  s.has_signs = signs != nullptr;
  if (rows == 0) return HADQ_OK;
  if (!x || !codes || !scales || !zero_points)
    return fail(HADQ_ERR_INVALID_ARG, "x, codes, scales and zero_points must not be NULL");
  if (!aligned(scales, 4)) return fail(HADQ_ERR_MISALIGNED, "scales must be 4-byte aligned");
  st = asym_coverage(s, aligned(x, 16) && aligned(codes, 16) && (!signs || aligned(signs, 16)));
  if (st != HADQ_OK) return st;
  hadq::ChunkAsymArgs a{};
  a.x = static_cast<const uint16_t*>(x);
  a.signs = signs;
  a.codes = static_cast<uint8_t*>(codes);
  a.scales = scales;
  a.zp = zero_points;
  a.scale_mul = (float)(1.0 / (std::sqrt(double(s.B)) * double((1 << bits) - 1)));
  a.rsqrt_b = (float)(1.0 / std::sqrt(double(s.B)));
  return launch_asym(0, s, a, false, reinterpret_cast<cudaStream_t>(stream));
}

hadq_status hadq_dequant_rotate_inv_asym(const void* codes, const float* scales, const uint8_t* zero_points,
                                         int64_t rows, int32_t dim, int32_t block, const int8_t* signs,
                                         int32_t bits, int32_t group, void* out, hadq_out_dtype out_dtype,
                                         hadq_stream_t stream) {
  g_last_error.clear();
  Shape s;
  hadq_status st = check_sizes(rows, dim, block, bits, group, &s);
  if (st != HADQ_OK) return st;
  if (out_dtype != HADQ_OUT_BF16 && out_dtype != HADQ_OUT_F32)
    return fail(HADQ_ERR_INVALID_ARG, "out_dtype must be HADQ_OUT_BF16 or HADQ_OUT_F32");
  s.has_signs = signs != nullptr;
  if (rows == 0) return HADQ_OK;
  if (!codes || !scales || !zero_points || !out)
    return fail(HADQ_ERR_INVALID_ARG, "codes, scales, zero_points and out must not be NULL");
  if (!aligned(scales, 4)) return fail(HADQ_ERR_MISALIGNED, "scales must be 4-byte aligned");
  st = asym_coverage(s, aligned(codes, 16) && aligned(out, 16) && (!signs || aligned(signs, 16)));
  if (st != HADQ_OK) return st;
  const bool f32 = out_dtype == HADQ_OUT_F32;
  hadq::ChunkAsymArgs a{};
  a.codes_in = static_cast<const uint8_t*>(codes);
  a.scales_in = scales;
  a.zp_in = zero_points;
  a.signs = signs;
  a.rot = f32 ? static_cast<float*>(out) : nullptr;
  a.out_bf16 = f32 ? nullptr : static_cast<uint16_t*>(out);
  a.rsqrt_b = (float)(1.0 / std::sqrt(double(s.B)));
  return launch_asym(1, s, a, f32, reinterpret_cast<cudaStream_t>(stream));
}

// Kronecker rotation F (x) H_b: sizes, pointers and the shared-memory budget.
static hadq_status kron_check(int64_t rows, int32_t a, int32_t b, int32_t bits, int32_t group, Shape* s) {
  if (a < 1 || a > 256) return fail(HADQ_ERR_INVALID_ARG, "a must be in [1, 256] (got %d)", a);
  if (b < 2 || !is_pow2(b)) return fail(HADQ_ERR_INVALID_ARG, "b must be a power of two >= 2 (got %d)", b);
  if (int64_t(a) * b > HADQ_MAX_DIM)
    return fail(HADQ_ERR_INVALID_ARG, "a * b must be at most %d (got %lld)", HADQ_MAX_DIM, (long long)a * b);
  hadq_status st = check_sizes(rows, a * b, b, bits, group, s);
  if (st != HADQ_OK) return st;
  if (hadq::kron_smem_bytes(a * b, a) > size_t(227) * 1024)
    return fail(HADQ_ERR_UNSUPPORTED, "a * b = %d with a = %d needs %zu bytes of shared memory (227 KB max)",
                a * b, a, hadq::kron_smem_bytes(a * b, a));
  return HADQ_OK;
}

// Kernel variants of the Kronecker rotation (see hadq_kron_plan).
static int kron_variant(int direction, const Shape& s, int a, int b, bool a16) {
  if (direction != 0) return HADQ_KRON_SMEM;
  const int G = s.G;
  const bool reg = b >= 16 && b <= 512 && G % 16 == 0 && G <= 512 && (32 % (G / 16)) == 0 && s.dim / 16 <= 1024 &&
                   a16;
  if (!reg) return HADQ_KRON_SMEM;
  if (a <= 32 && s.dim % 512 == 0 && s.dim / 16 <= 512) return HADQ_KRON_MMA;
  return HADQ_KRON_REG16;
}

static hadq_status launch_kron(int direction, const Shape& s, hadq::KronArgs k, bool f32, cudaStream_t stream,
                               int variant = HADQ_KRON_SMEM) {
  const void* fn = variant == HADQ_KRON_MMA     ? hadq::kron_tc_kernel_ptr(s.bits, (k.a + 7) / 8, k.s != nullptr, s.B == 256)
                   : variant == HADQ_KRON_REG16 ? hadq::kron16_kernel_ptr(s.bits)
                                                : hadq::kron_kernel_ptr(direction, s.bits);
  const int threads = variant == HADQ_KRON_SMEM ? 256 : s.dim / 16;
  const size_t smem = variant == HADQ_KRON_MMA ? hadq::kron_tc_smem_bytes(k.a, s.B) : hadq::kron_smem_bytes(s.dim, k.a);
  int res = 1;
  const hadq_status pst = prepare(fn, threads, smem, "Kronecker kernel", &res);
  if (pst != HADQ_OK) return pst;
  const int64_t cap = int64_t(res) * sm_count();
  cudaError_t e;
  const unsigned grid = (unsigned)(s.rows < cap ? s.rows : cap);
  if (direction == 0) {
    void* args[] = {&k};
    e = cudaLaunchKernel(fn, dim3(grid), dim3(threads), args, smem, stream);
  } else {
    bool out_f32 = f32;
    void* args[] = {&k, &out_f32};
    e = cudaLaunchKernel(fn, dim3(grid), dim3(threads), args, smem, stream);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return fail(HADQ_ERR_CUDA, "Kronecker kernel launch failed: %s", cudaGetErrorString(e));
  }
  return after_launch("Kronecker kernel");
}

hadq_status hadq_kron_plan(int32_t direction, int64_t rows, int32_t a, int32_t b, int32_t bits, int32_t group,
                           int32_t aligned16, int32_t* variant) {
  g_last_error.clear();
  if (direction != 0 && direction != 1)
    return fail(HADQ_ERR_INVALID_ARG, "direction must be 0 or 1 (got %d)", direction);
  Shape s;
  hadq_status st = kron_check(rows, a, b, bits, group, &s);
  if (st != HADQ_OK) return st;
  if (variant) *variant = kron_variant(direction, s, a, b, aligned16 != 0);
  return HADQ_OK;
}

// Forward Kronecker call with a float32 factor fa or a +-1 factor sa (one of
// them non-null).
static hadq_status kron_forward(bool pm1, const void* x, int64_t rows, int32_t a, const float* fa,
                                const int8_t* sa, int32_t b, const int8_t* signs, int32_t bits, int32_t group, void* codes,
                                float* scales, float* rotated_out, hadq_stream_t stream) {
  g_last_error.clear();
  Shape s;
  hadq_status st = kron_check(rows, a, b, bits, group, &s);
  if (st != HADQ_OK) return st;
  if (rows == 0) return HADQ_OK;
  if (!x || !(fa || sa) || !codes || !scales)
    return fail(HADQ_ERR_INVALID_ARG, "x, %s, codes and scales must not be NULL", pm1 ? "sa" : "fa");
  if (!aligned(x, 2)) return fail(HADQ_ERR_MISALIGNED, "x must be 2-byte aligned");
  if ((fa && !aligned(fa, 4)) || !aligned(scales, 4) || (rotated_out && !aligned(rotated_out, 4)))
    return fail(HADQ_ERR_MISALIGNED, "fa, scales and rotated_out must be 4-byte aligned");
  const double inv_sqrt_a = sa ? 1.0 / std::sqrt(double(a)) : 1.0;
  hadq::KronArgs k{};
  k.g.x = static_cast<const uint16_t*>(x);
  k.g.signs = signs;
  k.g.codes = static_cast<uint8_t*>(codes);
  k.g.scales = scales;
  k.g.rot = rotated_out;
  k.g.rows = rows;
  k.g.dim = s.dim;
  k.g.block = b;
  k.g.group = s.G;
  k.g.scale_mul = (float)(1.0 / (std::sqrt(double(b)) * double((1 << (bits - 1)) - 1)));
  k.g.rsqrt_b = (float)(1.0 / std::sqrt(double(b)));
  k.f = fa;
  k.s = sa;
  k.s_mul = (float)inv_sqrt_a;
  k.a = a;
  k.ap = (a + hadq::kKronR - 1) / hadq::kKronR * hadq::kKronR;
  const bool a16 = aligned(x, 16) && aligned(codes, 16) && (!signs || aligned(signs, 16)) &&
                   (!rotated_out || aligned(rotated_out, 16));
  const int variant = kron_variant(0, s, a, b, a16);
  if (variant == HADQ_KRON_MMA && sa) {
    // the tensor-core kernel mixes with S itself: 1 / sqrt(a) joins the
    // output multipliers
    k.g.scale_mul = (float)(inv_sqrt_a / (std::sqrt(double(b)) * double((1 << (bits - 1)) - 1)));
    k.g.rsqrt_b = (float)(inv_sqrt_a / std::sqrt(double(b)));
  }
  return launch_kron(0, s, k, false, reinterpret_cast<cudaStream_t>(stream), variant);
}

static hadq_status kron_inverse(bool pm1, const void* codes, const float* scales, int64_t rows, int32_t a,
                                const float* fa, const int8_t* sa, int32_t b, const int8_t* signs, int32_t bits, int32_t group,
                                void* out, hadq_out_dtype out_dtype, hadq_stream_t stream) {
  g_last_error.clear();
  Shape s;
  hadq_status st = kron_check(rows, a, b, bits, group, &s);
  if (st != HADQ_OK) return st;
  if (out_dtype != HADQ_OUT_BF16 && out_dtype != HADQ_OUT_F32)
    return fail(HADQ_ERR_INVALID_ARG, "out_dtype must be HADQ_OUT_BF16 or HADQ_OUT_F32");
  if (rows == 0) return HADQ_OK;
  if (!codes || !scales || !(fa || sa) || !out)
    return fail(HADQ_ERR_INVALID_ARG, "codes, scales, %s and out must not be NULL", pm1 ? "sa" : "fa");
  const bool f32 = out_dtype == HADQ_OUT_F32;
  if ((fa && !aligned(fa, 4)) || !aligned(scales, 4))
    return fail(HADQ_ERR_MISALIGNED, "fa and scales must be 4-byte aligned");
  if (!aligned(out, f32 ? 4 : 2)) return fail(HADQ_ERR_MISALIGNED, "out must be aligned to its element size");
  hadq::KronArgs k{};
  k.g.codes_in = static_cast<const uint8_t*>(codes);
  k.g.scales_in = scales;
  k.g.signs = signs;
  k.g.rot = f32 ? static_cast<float*>(out) : nullptr;
  k.g.out_bf16 = f32 ? nullptr : static_cast<uint16_t*>(out);
  k.g.rows = rows;
  k.g.dim = s.dim;
  k.g.block = b;
  k.g.group = s.G;
  k.g.rsqrt_b = (float)(1.0 / std::sqrt(double(b)));
  k.f = fa;
  k.s = sa;
  k.s_mul = (float)(1.0 / std::sqrt(double(a)));
  k.a = a;
  k.ap = (a + hadq::kKronR - 1) / hadq::kKronR * hadq::kKronR;
  return launch_kron(1, s, k, f32, reinterpret_cast<cudaStream_t>(stream));
}

hadq_status hadq_rotate_quantize_kron(const void* x, int64_t rows, int32_t a, const float* fa, int32_t b,
                                      const int8_t* signs, int32_t bits, int32_t group, void* codes, float* scales,
                                      float* rotated_out, hadq_stream_t stream) {
  return kron_forward(false, x, rows, a, fa, nullptr, b, signs, bits, group, codes, scales, rotated_out, stream);
}

hadq_status hadq_rotate_quantize_kron_pm1(const void* x, int64_t rows, int32_t a, const int8_t* sa, int32_t b,
                                          const int8_t* signs, int32_t bits, int32_t group, void* codes,
                                          float* scales, float* rotated_out, hadq_stream_t stream) {
  return kron_forward(true, x, rows, a, nullptr, sa, b, signs, bits, group, codes, scales, rotated_out, stream);
}

hadq_status hadq_dequant_rotate_inv_kron(const void* codes, const float* scales, int64_t rows, int32_t a,
                                         const float* fa, int32_t b, const int8_t* signs, int32_t bits,
                                         int32_t group, void* out, hadq_out_dtype out_dtype, hadq_stream_t stream) {
  return kron_inverse(false, codes, scales, rows, a, fa, nullptr, b, signs, bits, group, out, out_dtype, stream);
}

hadq_status hadq_dequant_rotate_inv_kron_pm1(const void* codes, const float* scales, int64_t rows, int32_t a,
                                             const int8_t* sa, int32_t b, const int8_t* signs, int32_t bits,
                                             int32_t group, void* out, hadq_out_dtype out_dtype,
                                             hadq_stream_t stream) {
  return kron_inverse(true, codes, scales, rows, a, nullptr, sa, b, signs, bits, group, out, out_dtype, stream);
}

const char* hadq_status_str(hadq_status st) {
  switch (st) {
    case HADQ_OK: return "ok";
    case HADQ_ERR_INVALID_ARG: return "invalid argument";
    case HADQ_ERR_UNSUPPORTED: return "unsupported combination";
    case HADQ_ERR_MISALIGNED: return "misaligned pointer";
    case HADQ_ERR_CUDA: return "CUDA error";
    case HADQ_ERR_DEVICE: return "a kernel gave up a bounded wait";
  }
  return "unknown status";
}

hadq_status hadq_device_status(hadq_stream_t stream) {
  g_last_error.clear();
  unsigned* word = hadq::tc_fault_word();
  if (!word) return fail(HADQ_ERR_CUDA, "the fault word has no device address");
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  unsigned v = 0;
  cudaError_t e = cudaStreamSynchronize(cs);
  if (e == cudaSuccess) e = cudaMemcpy(&v, word, sizeof v, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && v) e = cudaMemset(word, 0, sizeof v);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(HADQ_ERR_CUDA, "reading the fault word failed: %s", cudaGetErrorString(e));
  }
  if (v) return fail(HADQ_ERR_DEVICE, "a tcgen05 kernel waited past its limit; its outputs are void");
  return HADQ_OK;
}

hadq_status hadq_selftest_bounded_wait(void* scratch, hadq_stream_t stream) {
  g_last_error.clear();
  if (!scratch) return fail(HADQ_ERR_INVALID_ARG, "scratch must not be NULL");
  if (!aligned(scratch, 16)) return fail(HADQ_ERR_MISALIGNED, "scratch must be 16-byte aligned");
  hadq_status st = hadq_device_status(stream);  // start from a clear record
  if (st != HADQ_OK) return st;
  Shape s{};
  s.rows = 4;
  s.dim = 4096;
  s.B = 4096;
  s.G = 4096;
  s.bits = 4;
  s.has_signs = false;
  uint8_t* buf = static_cast<uint8_t*>(scratch);
  st = launch_h4096_tc(s, buf, nullptr, buf + 32768, reinterpret_cast<float*>(buf + 40960), 1.0f,
                       reinterpret_cast<cudaStream_t>(stream), 0);
  if (st != HADQ_OK) return st;
  return hadq_device_status(stream);
}

const char* hadq_last_error(void) { return g_last_error.c_str(); }

int64_t hadq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int32_t hadq_version(void) { return 1; }

}  // extern "C"
