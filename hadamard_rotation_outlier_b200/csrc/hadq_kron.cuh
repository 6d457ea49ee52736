// Kronecker rotation y = (F (x) H_b)(x * s) fused with the symmetric
// quantiser, and its inverse.
//
// The online down_proj rotation of QuaRot uses a Kronecker-product matrix,
// and widths without a Sylvester matrix take a stored Hadamard matrix
// ("QuaRot: rotation-based outlier suppression", msModelSlim, online
// rotation and FAQ).  The row of width a * b is viewed as X[a][b] (element
// i * b + j): y = vec(F X H_b^T) with F the caller's a x a factor (for a
// stored Hadamard matrix S_a: F = S_a / sqrt(a)) and H_b the Sylvester matrix.
//
// One CTA per row (grid-stride), the row in shared memory as float32:
//   1. butterflies along each b-wide sub-block (unnormalised H_b),
//   2. mixing across the a sub-blocks: out[r][j] = sum_i C[r][i] in[i][j],
//      with C = F (forward) or F^T (inverse) held transposed in shared memory;
//      a thread computes kKronR outputs of one column j from one read of each
//      input and 128-bit broadcast reads of the coefficients,
//   3. the quantiser of the generic path (forward) or the output (inverse).
// The 1/sqrt(b) of H_b is folded into the scale, as everywhere else.
#pragma once

#include <cuda_bf16.h>

#include "hadq_generic.cuh"
#include "hadq_mma.cuh"

namespace hadq {

constexpr int kKronR = 8;  // outputs per thread in the mixing step

struct KronArgs {
  GenericArgs g;      // x / codes_in, scales, signs, codes / out, rows, dim = a * b, block = b, group
  const float* f;     // [a][a] factor, row-major, device memory (null when s is given)
  const int8_t* s;    // [a][a] +-1 matrix S, row-major: the factor is S * s_mul (null when f is given)
  float s_mul;        // 1 / sqrt(a) for s
  int a;
  int ap;             // a rounded up to a multiple of kKronR (pitch of the transposed coefficients)
};

// Entry (r, i) of the factor.
__device__ __forceinline__ float kron_factor(const KronArgs& k, int r, int i) {
  return k.s ? float(k.s[r * k.a + i]) * k.s_mul : __ldg(k.f + r * k.a + i);
}

// Shared memory: in[dim] | out[dim] | coefficients [a][ap] | codes [dim] (int8);
// the register variant pads in and out by 4 floats per 32 (see kron_pad) and
// has no code area, which fits in the same size.
__host__ __device__ inline size_t kron_smem_bytes(int dim, int a) {
  const int ap = (a + kKronR - 1) / kKronR * kKronR;
  return size_t(2) * dim * 4 + size_t(a) * ap * 4 + ((size_t(dim) + 15) & ~size_t(15));
}

// Coefficients of the mixing step, transposed: ct[i * ap + r] = C[r][i] for
// C = F (transpose == false) or C = F^T; columns r >= a are zero.
__device__ __forceinline__ void kron_load_coeffs(const KronArgs& k, bool transpose, float* ct) {
  const int a = k.a, ap = k.ap;
  for (int e = threadIdx.x; e < a * ap; e += blockDim.x) {
    const int i = e / ap, r = e - i * ap;
    ct[e] = r < a ? (transpose ? kron_factor(k, i, r) : kron_factor(k, r, i)) : 0.0f;
  }
}

// Shared-memory index of row element e in the register variant: 4 floats of
// padding after every 32, so that 16-float runs owned by consecutive threads
// move with conflict-free 128-bit accesses.
__device__ __forceinline__ int kron_pad(int e) { return e + ((e >> 5) << 2); }

// out[r][j] = sum_i C[r][i] in[i][j] over the a x b row (b = 2^lb).
// PAD: in and out use kron_pad indices.
template <bool PAD>
__device__ __forceinline__ void kron_mix(const float* in, float* out, const float* ct, int a, int ap, int lb) {
  const int b = 1 << lb;
  const int tiles = ap / kKronR;
  for (int o = threadIdx.x; o < tiles * b; o += blockDim.x) {
    const int rt = o >> lb, j = o & (b - 1);
    float acc[kKronR];
#pragma unroll
    for (int r = 0; r < kKronR; ++r) acc[r] = 0.0f;
    const float* cp = ct + rt * kKronR;
#pragma unroll 4
    for (int i = 0; i < a; ++i) {
      const float z = in[PAD ? kron_pad(i * b + j) : i * b + j];
      const float4 c0 = *reinterpret_cast<const float4*>(cp + i * ap);
      const float4 c1 = *reinterpret_cast<const float4*>(cp + i * ap + 4);
      acc[0] = fmaf(c0.x, z, acc[0]);
      acc[1] = fmaf(c0.y, z, acc[1]);
      acc[2] = fmaf(c0.z, z, acc[2]);
      acc[3] = fmaf(c0.w, z, acc[3]);
      acc[4] = fmaf(c1.x, z, acc[4]);
      acc[5] = fmaf(c1.y, z, acc[5]);
      acc[6] = fmaf(c1.z, z, acc[6]);
      acc[7] = fmaf(c1.w, z, acc[7]);
    }
#pragma unroll
    for (int r = 0; r < kKronR; ++r)
      if (rt * kKronR + r < a) {
        const int e = (rt * kKronR + r) * b + j;
        out[PAD ? kron_pad(e) : e] = acc[r];
      }
  }
}

__host__ __device__ inline int kron_log2(int b) {
  int l = 0;
  while ((1 << l) < b) ++l;
  return l;
}

template <int BITS>
__global__ void __launch_bounds__(256) rq_kron_kernel(KronArgs k) {
  constexpr float QMAX = (float)((1 << (BITS - 1)) - 1);
  const GenericArgs& a = k.g;
  extern __shared__ __align__(16) float kbuf[];
  const int dim = a.dim, G = a.group, b = a.block;
  float* sin = kbuf;
  float* sout = kbuf + dim;
  float* ct = kbuf + 2 * dim;
  int8_t* scode = reinterpret_cast<int8_t*>(ct + k.a * k.ap);
  const int ngroups = dim / G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  kron_load_coeffs(k, false, ct);

  for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
    const int64_t base = row * dim;
    for (int i = threadIdx.x; i < dim; i += blockDim.x) {
      float f = __uint_as_float((uint32_t)a.x[base + i] << 16);
      if (a.signs && a.signs[i] < 0) f = -f;
      sin[i] = f;
    }
    __syncthreads();
    generic_stages(sin, dim, b);
    kron_mix<false>(sin, sout, ct, k.a, k.ap, kron_log2(b));
    __syncthreads();

    if (G <= 32) {
      for (int g = threadIdx.x; g < ngroups; g += blockDim.x) {
        float m = 0.0f;
        for (int i = 0; i < G; ++i) m = fmaxf(m, fabsf(sout[g * G + i]));
        a.scales[row * ngroups + g] = m * a.scale_mul;
        for (int i = 0; i < G; ++i) scode[g * G + i] = (int8_t)code_of(sout[g * G + i], m, QMAX);
      }
    } else {
      for (int g = warp; g < ngroups; g += nwarps) {
        float m = 0.0f;
        for (int i = lane; i < G; i += 32) m = fmaxf(m, fabsf(sout[g * G + i]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) a.scales[row * ngroups + g] = m * a.scale_mul;
        for (int i = lane; i < G; i += 32) scode[g * G + i] = (int8_t)code_of(sout[g * G + i], m, QMAX);
      }
    }
    if (a.rot)
      for (int i = threadIdx.x; i < dim; i += blockDim.x) a.rot[base + i] = sout[i] * a.rsqrt_b;
    __syncthreads();

    if constexpr (BITS == 8) {
      for (int i = threadIdx.x; i < dim; i += blockDim.x) a.codes[base + i] = (uint8_t)scode[i];
    } else {
      for (int p = threadIdx.x; p < dim / 2; p += blockDim.x)
        a.codes[base / 2 + p] = (uint8_t)((scode[2 * p] & 0xf) | ((scode[2 * p + 1] & 0xf) << 4));
    }
    __syncthreads();
  }
}

// Inverse: q * scale -> mixing with F^T -> butterflies -> signs -> output.
// Rows whose scales fall below 2^-100 run at 2^64 scale and are scaled back
// once at the end (the factor may mix every block, so the row is one unit).
template <int BITS>
__global__ void __launch_bounds__(256) dq_kron_kernel(KronArgs k, bool out_f32) {
  const GenericArgs& a = k.g;
  extern __shared__ __align__(16) float kbuf[];
  const int dim = a.dim, G = a.group, b = a.block;
  float* sin = kbuf;
  float* sout = kbuf + dim;
  float* ct = kbuf + 2 * dim;
  int* stiny = reinterpret_cast<int*>(ct + k.a * k.ap);
  const int ngroups = dim / G;
  kron_load_coeffs(k, true, ct);

  for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
    const int64_t base = row * dim;
    const float* srow = a.scales_in + row * ngroups;
    if (threadIdx.x == 0) *stiny = 0;
    __syncthreads();
    for (int g = threadIdx.x; g < ngroups; g += blockDim.x)
      if (srow[g] < kTinyScale && srow[g] != 0.0f) *stiny = 1;
    __syncthreads();
    const bool tiny = *stiny != 0;
    const float pre = (tiny ? kUp64 : 1.0f) * a.rsqrt_b;
    for (int i = threadIdx.x; i < dim; i += blockDim.x) {
      int qv;
      if constexpr (BITS == 8) {
        qv = (int8_t)a.codes_in[base + i];
      } else {
        const uint32_t byte = a.codes_in[(base + i) >> 1];
        qv = ((int32_t)((byte >> (4 * (i & 1))) << 28)) >> 28;
      }
      sin[i] = (float)qv * (srow[i / G] * pre);
    }
    __syncthreads();
    kron_mix<false>(sin, sout, ct, k.a, k.ap, kron_log2(b));
    __syncthreads();
    generic_stages(sout, dim, b);
    for (int i = threadIdx.x; i < dim; i += blockDim.x) {
      float f = sout[i];
      if (tiny) f *= kDown64;
      if (a.signs && a.signs[i] < 0) f = -f;
      if (out_f32) {
        a.rot[base + i] = f;
      } else {
        uint32_t bb = __float_as_uint(f);
        a.out_bf16[base + i] = (uint16_t)((bb + 0x7fffu + ((bb >> 16) & 1u)) >> 16);
      }
    }
    __syncthreads();
  }
}

// Register variant for b in 16..512 and groups of 16..512 columns (powers of
// two): one thread per 16 consecutive elements of the row (dim / 16 threads,
// at most 1024), so
//   - the b-butterflies run on bits 0-3 in registers and on the remaining
//     bits across the b / 16 lanes of the sub-block (lane shuffles, inside
//     one warp since b / 16 <= 32),
//   - the mixing goes through shared memory as above,
//   - each group's maximum is a shuffle over its G / 16 lanes and the codes
//     leave from registers.
template <int BITS>
__global__ void __launch_bounds__(1024) rq_kron16_kernel(KronArgs k) {
  constexpr float QMAX = (float)((1 << (BITS - 1)) - 1);
  const GenericArgs& a = k.g;
  extern __shared__ __align__(16) float kbuf[];
  const int dim = a.dim, b = a.block, G = a.group;
  const int pdim = kron_pad(dim);  // padded row length (a multiple of 4)
  float* sin = kbuf;
  float* sout = kbuf + pdim;
  float* ct = kbuf + 2 * pdim;
  const int t = threadIdx.x;
  const int e0 = 16 * t;
  const int lane = t & 31;
  const int lanes_b = b >> 4;  // lanes per sub-block
  const int lanes_g = G >> 4;  // lanes per scale group
  const int lb = kron_log2(b);
  const int lg = kron_log2(G);
  const int gpr = dim >> lg, my_g = e0 >> lg;  // scale groups per row, this thread's group
  kron_load_coeffs(k, false, ct);
  // sign masks of this thread's 16 columns (bf16 pairs)
  uint32_t smask[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) smask[i] = 0u;
  if (a.signs) {
    const uint4 sg = *reinterpret_cast<const uint4*>(a.signs + e0);
    const uint32_t w[4] = {sg.x, sg.y, sg.z, sg.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t word = w[i >> 1];
      const int sh = 16 * (i & 1);
      smask[i] = (((word >> (sh + 7)) & 1u) << 15) | (((word >> (sh + 15)) & 1u) << 31);
    }
  }

  for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
    const int64_t base = row * dim;
    float v[16];
    {
      const uint4* src = reinterpret_cast<const uint4*>(a.x + base + e0);
      const uint4 r0 = src[0], r1 = src[1];
      const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) bf16_pair_stage1(w[i] ^ smask[i], v[2 * i], v[2 * i + 1]);
    }
    reg_fwht_from<16, 1, 4>(v);
    for (int m = 1; m < lanes_b; m <<= 1) {  // bits 4.. of the sub-block index: lanes
      const float sg = (lane & m) ? -1.0f : 1.0f;
      lane_stage<16>(v, m, sg);
    }
#pragma unroll
    for (int i = 0; i < 16; i += 4)
      *reinterpret_cast<float4*>(sin + kron_pad(e0 + i)) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    __syncthreads();
    kron_mix<true>(sin, sout, ct, k.a, k.ap, lb);
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 16; i += 4) {
      const float4 q = *reinterpret_cast<const float4*>(sout + kron_pad(e0 + i));
      v[i] = q.x;
      v[i + 1] = q.y;
      v[i + 2] = q.z;
      v[i + 3] = q.w;
    }
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
    for (int o = 1; o < lanes_g; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((t & (lanes_g - 1)) == 0) a.scales[row * gpr + my_g] = m * a.scale_mul;
    if (a.rot) {
      float4* dst = reinterpret_cast<float4*>(a.rot + base + e0);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        dst[i] = make_float4(v[4 * i] * a.rsqrt_b, v[4 * i + 1] * a.rsqrt_b, v[4 * i + 2] * a.rsqrt_b,
                             v[4 * i + 3] * a.rsqrt_b);
    }
    uint32_t cc0[8], cc1[8];
    quantize8(v, m, QMAX, cc0);
    quantize8(v + 8, m, QMAX, cc1);
    if constexpr (BITS == 8) {
      *reinterpret_cast<uint4*>(a.codes + base + e0) =
          make_uint4(pack_i8x4(cc0[0], cc0[1], cc0[2], cc0[3]), pack_i8x4(cc0[4], cc0[5], cc0[6], cc0[7]),
                     pack_i8x4(cc1[0], cc1[1], cc1[2], cc1[3]), pack_i8x4(cc1[4], cc1[5], cc1[6], cc1[7]));
    } else {
      *reinterpret_cast<uint2*>(a.codes + (base + e0) / 2) = make_uint2(pack_i4x8(cc0), pack_i4x8(cc1));
    }
    __syncthreads();  // sin / sout are reused by the next row
  }
}

// ---------------------------------------------------------------------------
// Tensor-core variant of the forward transform for a <= 32.
//
// F (x) H_b = (I (x) H_b)(F (x) I): the mixing may run first, on the signed
// bf16 input itself, which bf16 holds exactly.  Per row, the mixing is then
// the product W[r][j] = sum_i F[r][i] X[i][j], a GEMM of M = b (columns j),
// N = a (rows r of F) and K = a, which runs as warp-level bf16 MMAs with
// float32 accumulation:
//   - F is split into three bf16 terms hi + mid + lo (exact to about 2^-24
//     of each entry; the products with the bf16 data are exact), applied
//     smallest first into one accumulator;
//   - X sits in shared memory as bf16 [i][j]; ldmatrix.trans hands each warp
//     the A fragments (16 columns j x 16 or 8 rows i), and the F terms stay in
//     registers as B fragments for the whole kernel;
//   - K and N are padded to multiples of 8 with zero rows of X and zero
//     entries of F.
// W goes to shared memory as float32, each thread reads back its 16
// consecutive outputs and finishes as the register variant does: bits 0-3
// of the b-butterflies in registers, the rest across lanes, then the group
// maxima and the codes.  KA = ceil(a / 8).
//
// Shared memory: X [8 KA][kron_tc_px(b) bytes] | W [8 KA][kron_tc_pw(b) floats]
// (W rows a .. 8 KA - 1 take the zero outputs of the N padding; never read).
// Row pitches: X rows are 2b + 16 bytes (an odd number of 16-byte units, so
// the eight rows of an ldmatrix tile fall in different banks); W rows hold
// b floats with 4 of padding after every 32 (the 128-bit reads of 16
// consecutive floats are conflict-free) and a pitch of 4 mod 32 words, so that
// the accumulator stores (8 columns x 4 row pairs per warp) are conflict-free
// too.  For b = 256 (the strided pass) the pitch is 16 mod 32 and column j of
// row r sits at (j ^ 8 ((r >> 1) & 3)) + 4 (j >> 5): the accumulator stores,
// the strided pass (two rows per warp) and the 128-bit reads are then all
// conflict-free.

__host__ __device__ inline int kron_tc_px(int b) { return 2 * b + 16; }

__host__ __device__ inline int kron_tc_pw(int b) {
  if (b == 256) return 304;
  const int base = b + (b >> 5) * 4;
  return base + ((36 - (base & 31)) & 31);
}

__host__ __device__ inline size_t kron_tc_smem_bytes(int a, int b) {
  const int ka = (a + 7) / 8;
  return size_t(8) * ka * kron_tc_px(b) + size_t(8) * ka * kron_tc_pw(b) * 4;
}

__device__ __forceinline__ int kron_tc_inner(int j) { return j + ((j >> 5) << 2); }

// The three bf16 terms of f (term 0 largest), as 16-bit patterns.
__device__ __forceinline__ void bf16_split3(float f, uint32_t (&t)[3]) {
  const __nv_bfloat16 h = __float2bfloat16_rn(f);
  const float r1 = f - __bfloat162float(h);  // exact
  const __nv_bfloat16 m = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(m);  // exact
  const __nv_bfloat16 l = __float2bfloat16_rn(r2);
  t[0] = __bfloat16_as_ushort(h);
  t[1] = __bfloat16_as_ushort(m);
  t[2] = __bfloat16_as_ushort(l);
}

// S256 (b = 256): bits 4-7 of the column index run as a strided pass over W
// (16 columns u + 16 k per thread, 4 register stages, written back) before the
// consecutive pass, instead of four lane-shuffle stages.
// Register caps: 64 (a 320-thread CTA three times per SM) for a <= 16, 96
// (twice) for 16 < a <= 24 and for the three-term split of a <= 24, 128 for
// a <= 32 with the split.  For the +-1 factor of a = 20, 96 registers and
// two CTAs ran 2.5 % faster than 64 registers and three.
template <int KA, int NS>
constexpr int kron_tc_maxreg() {
  return NS == 3 ? (KA <= 2 ? 64 : KA == 3 ? 96 : 128) : (KA <= 2 ? 64 : 96);
}

template <int BITS, int KA, int NS, bool S256>
__global__ void __maxnreg__((kron_tc_maxreg<KA, NS>())) rq_kron_tc_kernel(KronArgs k) {
  static_assert(NS == 1 || NS == 3, "one term (a +-1 factor) or three (a float32 factor)");
  constexpr float QMAX = (float)((1 << (BITS - 1)) - 1);
  const GenericArgs& a = k.g;
  extern __shared__ __align__(16) unsigned char tbuf[];
  // b = 256 (S256): the block and the shared-memory pitches are constants
  const int dim = a.dim, b = S256 ? 256 : a.block, G = a.group, fa = k.a;
  const int px = S256 ? kron_tc_px(256) : kron_tc_px(b), pw = S256 ? kron_tc_pw(256) : kron_tc_pw(b);
  const int64_t nrows = a.rows;
  const float scale_mul = a.scale_mul;
  unsigned char* xs = tbuf;
  float* ws = reinterpret_cast<float*>(tbuf + size_t(8) * KA * px);
  const int t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5, nwarps = blockDim.x >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int e0 = 16 * t;
  const int lb = S256 ? 8 : kron_log2(b);
  const int lanes_b = b >> 4, lanes_g = G >> 4;
  const int lg = kron_log2(G);
  const int gpr = dim >> lg, my_g = e0 >> lg;  // scale groups per row, this thread's group
  const int xi = e0 >> lb, xj = e0 & (b - 1);  // this thread's row and first column

  // zero X (rows a .. 8 KA - 1 stay zero: the K padding)
  for (int e = t; e < 8 * KA * px / 16; e += blockDim.x) reinterpret_cast<uint4*>(xs)[e] = make_uint4(0, 0, 0, 0);

  // B fragments: bf[s][nt][kk] = {C[r][i], C[r][i + 1]} (term s) with
  // r = 8 nt + g, i = 8 kk + 2 t4; zero outside a x a.  C = S itself for a
  // +-1 factor (one exact term; its 1 / sqrt(a) is in scale_mul and rsqrt_b),
  // else F in three terms.
  uint32_t bf[NS][KA][KA];
#pragma unroll
  for (int nt = 0; nt < KA; ++nt) {
#pragma unroll
    for (int kk = 0; kk < KA; ++kk) {
      const int r = 8 * nt + g, i = 8 * kk + 2 * t4;
      if constexpr (NS == 1) {
        const float f0 = (r < fa && i < fa) ? float(k.s[r * fa + i]) : 0.0f;
        const float f1 = (r < fa && i + 1 < fa) ? float(k.s[r * fa + i + 1]) : 0.0f;
        bf[0][nt][kk] = uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(f0))) |
                        (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(f1))) << 16);
      } else {
        const float f0 = (r < fa && i < fa) ? __ldg(k.f + r * fa + i) : 0.0f;
        const float f1 = (r < fa && i + 1 < fa) ? __ldg(k.f + r * fa + i + 1) : 0.0f;
        uint32_t s0[3], s1[3];
        bf16_split3(f0, s0);
        bf16_split3(f1, s1);
#pragma unroll
        for (int s = 0; s < 3; ++s) bf[s][nt][kk] = s0[s] | (s1[s] << 16);
      }
    }
  }

  // sign masks of this thread's 16 columns (bf16 pairs)
  uint32_t smask[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) smask[i] = 0u;
  if (a.signs) {
    const uint4 sg = *reinterpret_cast<const uint4*>(a.signs + e0);
    const uint32_t w[4] = {sg.x, sg.y, sg.z, sg.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t word = w[i >> 1];
      const int sh = 16 * (i & 1);
      smask[i] = (((word >> (sh + 7)) & 1u) << 15) | (((word >> (sh + 15)) & 1u) << 31);
    }
  }

  // this lane's ldmatrix row address (bytes, shared window) for k16 step 0 of
  // m-tile 0: x4 tiles (i 0-7, j 0-7), (i 0-7, j 8-15), (i 8-15, j 0-7),
  // (i 8-15, j 8-15) -> a0..a3; the x2 tail uses the first two
  const uint32_t xs_base = static_cast<uint32_t>(__cvta_generic_to_shared(xs));
  const int lm = lane >> 3, lr = lane & 7;
  const uint32_t a_addr = xs_base + uint32_t(((lm >> 1) * 8 + lr) * px + (lm & 1) * 16);
  const uint32_t a_addr_tail = xs_base + uint32_t(((KA - 1) * 8 + lr) * px + (lm & 1) * 16);
  const int half = (t >> 2) & 1;  // store order of the two 16-byte halves

  uint4 n0 = make_uint4(0, 0, 0, 0), n1 = n0;
  // this thread's input, codes and scale for the current row, stepped by the
  // grid's rows instead of recomputed from the row index
  const int64_t xstep = int64_t(gridDim.x) * dim;
  const uint16_t* xp = a.x + int64_t(blockIdx.x) * dim + e0;
  uint8_t* cp = a.codes + (int64_t(blockIdx.x) * dim + e0) * BITS / 8;
  float* sp = a.scales + int64_t(blockIdx.x) * gpr + my_g;
  const int64_t cstep = xstep * BITS / 8, sstep = int64_t(gridDim.x) * gpr;
  if (int64_t(blockIdx.x) < nrows) {
    const uint4* src = reinterpret_cast<const uint4*>(xp);
    n0 = src[0];
    n1 = src[1];
  }

  for (int64_t row = blockIdx.x; row < nrows; row += gridDim.x, xp += xstep, cp += cstep, sp += sstep) {
    const int64_t base = row * dim;
    {
      const uint4 s0 = make_uint4(n0.x ^ smask[0], n0.y ^ smask[1], n0.z ^ smask[2], n0.w ^ smask[3]);
      const uint4 s1 = make_uint4(n1.x ^ smask[4], n1.y ^ smask[5], n1.z ^ smask[6], n1.w ^ smask[7]);
      uint4* dst = reinterpret_cast<uint4*>(xs + xi * px + 2 * xj);
      dst[half] = half ? s1 : s0;
      dst[half ^ 1] = half ? s0 : s1;
    }
    if (row + gridDim.x < nrows) {
      const uint4* src = reinterpret_cast<const uint4*>(xp + xstep);
      n0 = src[0];
      n1 = src[1];
    }
    __syncthreads();

    // mixing: m-tile mt covers columns j = 16 mt .. 16 mt + 15
    for (int mt = warp; mt < (S256 ? 16 : (b >> 4)); mt += nwarps) {
      float d[KA][4];
#pragma unroll
      for (int nt = 0; nt < KA; ++nt) d[nt][0] = d[nt][1] = d[nt][2] = d[nt][3] = 0.0f;
#pragma unroll
      for (int kp = 0; kp < KA / 2; ++kp) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4_trans(a_addr + uint32_t(kp * 16 * px + mt * 32), a0, a1, a2, a3);
        // smallest term first; consecutive MMAs go to different accumulators
#pragma unroll
        for (int s = NS - 1; s >= 0; --s) {
#pragma unroll
          for (int nt = 0; nt < KA; ++nt)
            mma_bf16_k16(d[nt], a0, a1, a2, a3, bf[s][nt][2 * kp], bf[s][nt][2 * kp + 1]);
        }
      }
      if constexpr (KA & 1) {
        uint32_t a0, a1;
        ldsm_x2_trans(a_addr_tail + uint32_t(mt * 32), a0, a1);
#pragma unroll
        for (int s = NS - 1; s >= 0; --s) {
#pragma unroll
          for (int nt = 0; nt < KA; ++nt) mma_bf16_k8(d[nt], a0, a1, bf[s][nt][KA - 1]);
        }
      }
      // d[nt] = W[r][j], W[r + 1][j], W[r][j + 8], W[r + 1][j + 8] with
      // r = 8 nt + 2 t4, j = 16 mt + g
      const int j = 16 * mt + g;
      // rows 8 nt + 2 t4 (+1) have (r >> 1) & 3 = t4
      const int c0 = S256 ? (j ^ (8 * t4)) + 4 * (j >> 5) : kron_tc_inner(j);
      const int c1 = S256 ? ((j + 8) ^ (8 * t4)) + 4 * ((j + 8) >> 5) : kron_tc_inner(j + 8);
      float* w0 = ws + 2 * t4 * pw;
#pragma unroll
      for (int nt = 0; nt < KA; ++nt) {
        float* wr = w0 + 8 * nt * pw;  // row r = 8 nt + 2 t4 (rows >= a hold zeros, never read)
        wr[c0] = d[nt][0];
        wr[c1] = d[nt][2];
        wr[pw + c0] = d[nt][1];
        wr[pw + c1] = d[nt][3];
      }
    }
    __syncthreads();

    // butterflies along j of this thread's 16 outputs, then the quantiser
    float v[16];
    if constexpr (S256) {
      // columns u + 16 kk of row xi (u = t & 15), swizzled: even kk at pe,
      // odd kk at po, each + 36 (kk >> 1)
      const int f = (xi >> 1) & 3, u = t & 15;
      float* rowp = ws + xi * pw + (u ^ (8 * (f & 1)));
      float* pe = rowp + 16 * (f >> 1);
      float* po = rowp + 16 - 16 * (f >> 1);
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) v[kk] = ((kk & 1) ? po : pe)[36 * (kk >> 1)];
      reg_fwht<16, 4>(v);
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) ((kk & 1) ? po : pe)[36 * (kk >> 1)] = v[kk];
      // the 16 threads of row xi (t >> 4) are half of one warp and touch no
      // other row, so the warp's own barrier orders the pass and the reads
      __syncwarp();
      // the thread's 16 consecutive columns 16 u .. 16 u + 15: float4 i at
      // offset 4 (i ^ 2 (f & 1)) from the swizzled run start
      const float* base = ws + xi * pw + 36 * (u >> 1) + 16 * ((u & 1) ^ (f >> 1));
      const float* q0 = base + 8 * (f & 1);
      const float* q1 = base + 8 - 8 * (f & 1);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 q = *reinterpret_cast<const float4*>((i < 2 ? q0 : q1) + 4 * (i & 1));
        v[4 * i] = q.x;
        v[4 * i + 1] = q.y;
        v[4 * i + 2] = q.z;
        v[4 * i + 3] = q.w;
      }
    } else {
      const float* src = ws + xi * pw + kron_tc_inner(xj);
#pragma unroll
      for (int i = 0; i < 16; i += 4) {
        const float4 q = *reinterpret_cast<const float4*>(src + i);
        v[i] = q.x;
        v[i + 1] = q.y;
        v[i + 2] = q.z;
        v[i + 3] = q.w;
      }
    }
    reg_fwht<16, 4>(v);
    if constexpr (!S256) {
      for (int m = 1; m < lanes_b; m <<= 1) {  // bits 4.. of the column index: lanes
        const float sg = (lane & m) ? -1.0f : 1.0f;
        lane_stage<16>(v, m, sg);
      }
    }
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
    for (int o = 1; o < lanes_g; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((t & (lanes_g - 1)) == 0) *sp = m * scale_mul;
    if (a.rot) {
      float4* dst = reinterpret_cast<float4*>(a.rot + base + e0);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        dst[i] = make_float4(v[4 * i] * a.rsqrt_b, v[4 * i + 1] * a.rsqrt_b, v[4 * i + 2] * a.rsqrt_b,
                             v[4 * i + 3] * a.rsqrt_b);
    }
    // one multiplier for the 16 codes, paired magic-number FMAs
    const QInv q = make_qinv(m, QMAX);
    if (q.tiny) {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] *= 18446744073709551616.0f;
    }
    uint32_t cc0[8], cc1[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      magic_code2(v[2 * i], v[2 * i + 1], q.inv, cc0[2 * i], cc0[2 * i + 1]);
      magic_code2(v[8 + 2 * i], v[9 + 2 * i], q.inv, cc1[2 * i], cc1[2 * i + 1]);
    }
    if constexpr (BITS == 8) {
      *reinterpret_cast<uint4*>(cp) =
          make_uint4(pack_i8x4(cc0[0], cc0[1], cc0[2], cc0[3]), pack_i8x4(cc0[4], cc0[5], cc0[6], cc0[7]),
                     pack_i8x4(cc1[0], cc1[1], cc1[2], cc1[3]), pack_i8x4(cc1[4], cc1[5], cc1[6], cc1[7]));
    } else {
      *reinterpret_cast<uint2*>(cp) = make_uint2(pack_i4x8(cc0), pack_i4x8(cc1));
    }
  }
}

}  // namespace hadq
