/*
 * hadq.h -- C ABI of the fused Hadamard rotate + quantize library (libhadq.so)
 *
 * The library implements the online rotate-then-quantize step of QuaRot-style
 * rotation quantisation and its inverse, as CUDA kernels for sm_100a (B200).
 *
 *   forward:  y = (x * s) H_B   per B-wide block of each row       (rotation)
 *             scale_g = max_{i in g} |y_i| / qmax,  qmax = 2^(bits-1) - 1
 *             q_i = clamp(round_half_even(y_i / scale_g), -qmax, qmax)
 *   inverse:  x_hat = ((q * scale_g) H_B) * s
 *
 * Sources (page title, section):
 *   - H_B is the normalised Sylvester matrix H_1 = [1],
 *     H_2n = [[H, H], [H, -H]] / sqrt(2) ("Hartmann rotation, lightweight QAT,
 *     streaming attention", section 1, the Hadamard rotation of Q and K:
 *     Q_rot = Q H^T, and H H^T = I so Q_rot K_rot^T = Q K^T).
 *   - Block-diagonal H for widths that are not a power of two: rows are cut
 *     into B-wide blocks rotated independently ("Rotation quantisation: the
 *     outlier nemesis", section 2.1; block_size -1 means no blocking in the
 *     msModelSlim QuaRot YAML configuration).
 *   - Random +-1 signs before H (randomised Hadamard, "QuaRot hands-on",
 *     section 2.1).
 *   - Symmetric absmax scale, round, clip ("Rotation quantisation: the outlier
 *     nemesis", section 2.2 quant_error; "Hartmann rotation", section 1,
 *     scale = max|x| / 127); per-group scales (same page, section 6.2).
 *   - INT4 codes take half a byte and the KV cache is dequantised when read
 *     ("QuaRot hands-on", sections 2.2 and 2.3).
 *
 * Conventions for every entry point:
 *   - All tensors are row-major, contiguous, on the current CUDA device.  The
 *     caller owns every buffer; the library never allocates device memory.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream).
 *     Argument checks run on the host before any launch; on an error nothing
 *     is launched and no output is touched.
 *   - HADQ_ERR_CUDA reports a launch failure (cudaGetLastError after the
 *     launch); hadq_last_error() gives the text.  Faults during execution are
 *     reported by the next synchronising CUDA call, as for any kernel.
 *   - rows == 0 is a valid empty call: HADQ_OK, nothing launched, pointers
 *     may be NULL.
 *   - Inputs must be finite.  Non-finite inputs give unspecified codes (no
 *     fault).
 *   - Calls that touch the same output buffers must be ordered by the caller.
 */
#ifndef HADQ_H
#define HADQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The same type as cudaStream_t (a pointer to the runtime's stream object). */
struct CUstream_st;
typedef struct CUstream_st *hadq_stream_t;

typedef enum {
  HADQ_OK = 0,
  HADQ_ERR_INVALID_ARG = 1,  /* out-of-range size, NULL pointer, bad enum     */
  HADQ_ERR_UNSUPPORTED = 2,  /* valid maths, no kernel for it                 */
  HADQ_ERR_MISALIGNED = 3,   /* pointer not aligned to its element size       */
  HADQ_ERR_CUDA = 4,         /* the CUDA runtime reported an error            */
  HADQ_ERR_DEVICE = 5        /* a kernel gave up a bounded wait (see
                                hadq_device_status); its outputs are void   */
} hadq_status;

typedef enum { HADQ_OUT_BF16 = 0, HADQ_OUT_F32 = 1 } hadq_out_dtype;

/* Which kernel family a call dispatches to (see hadq_plan). */
typedef enum {
  HADQ_PATH_NONE = 0,      /* empty call, nothing launched                  */
  HADQ_PATH_BLOCKED = 1,   /* register butterflies, blocks of 8..256        */
  HADQ_PATH_FULL4096 = 2,  /* one 4096-point block per row, smem transposes */
  HADQ_PATH_GENERIC = 3,   /* shared-memory kernel, any valid combination   */
  HADQ_PATH_CHUNK = 4,     /* one 128-column chunk per thread, blocks <= 128,
                              slabs staged through shared memory            */
  HADQ_PATH_WIDE4096 = 5,  /* 4096-column blocks with one scale per block:
                              one block per warp, in-warp transpose         */
  HADQ_PATH_WIDE4096_MMA = 6, /* the same blocks (dim = 4096 when signs are
                              given) with the first 16-point stage as a bf16
                              tensor-core MMA against H_16                  */
  HADQ_PATH_CHUNK_MMA = 7, /* 128-point blocks, signs or none, the first
                              16-point stage as an MMA over 16 blocks at a
                              time and the other three in registers.
                              Forward (one scale per block): bf16 MMA on
                              the input, signs as XOR masks on its operand.
                              Inverse (scale groups of whole blocks): f16
                              MMA on the integer codes                      */
  HADQ_PATH_H4096_TC = 8   /* 4096-column blocks with one scale per block
                              (dim = 4096 when signs are given), forward, no
                              rotated_out: TMA-fed tcgen05 GEMM against
                              H_128 with TMEM accumulators, then five
                              register stages; one persistent CTA per SM    */
} hadq_path;

/* Kernel variant of a Kronecker-rotation call (see hadq_kron_plan). */
typedef enum {
  HADQ_KRON_SMEM = 0,   /* one CTA per row, the row in shared memory; any
                           valid shape, and every inverse                   */
  HADQ_KRON_REG16 = 1,  /* forward: 16 elements per thread, butterflies in
                           registers and lanes, mixing on the FP32 cores    */
  HADQ_KRON_MMA = 2     /* forward, a <= 32: mixing first, as bf16 tensor-
                           core MMAs against a three-term split of F, then
                           the register butterflies                         */
} hadq_kron_variant;

enum { HADQ_MAX_DIM = 32768 };

/*
 * hadq_rotate_quantize -- fused rotate + quantise of a [rows, dim] bf16 tensor.
 *
 *   x           device, bfloat16 [rows, dim], 2-byte aligned (16 for the fast
 *               paths; others fall back to the generic kernel).
 *   rows        >= 0.
 *   dim         1 .. HADQ_MAX_DIM; even when bits == 4.
 *   block       Hadamard block B: -1 = whole row (dim must be a power of two),
 *               else a power of two (1 allowed = no rotation) dividing dim.
 *   signs       device, int8 [dim], negative entry = -1, else +1; or NULL for
 *               no sign flip.  Applied to x before H.
 *   bits        4 or 8.
 *   group       scale group G in columns: -1 = one scale per row, else any
 *               divisor of dim.  Independent of block.
 *   codes       device output.  bits 8: int8 [rows, dim].  bits 4: uint8
 *               [rows, dim/2], element 2j in the low nibble of byte j, 4-bit
 *               two's complement, values in [-7, 7].
 *   scales      device output, float32 [rows, dim/G], 4-byte aligned.
 *               scale = max|y| / qmax of the group; 0 for an all-zero group
 *               (whose codes are then 0).
 *   rotated_out device output float32 [rows, dim] (4-byte aligned) receiving y
 *               itself, or NULL.  Meant for checking; costs 4 bytes/element.
 */
hadq_status hadq_rotate_quantize(const void *x, int64_t rows, int32_t dim, int32_t block,
                                 const int8_t *signs, int32_t bits, int32_t group,
                                 void *codes, float *scales, float *rotated_out,
                                 hadq_stream_t stream);

/*
 * hadq_dequant_rotate_inv -- x_hat = ((q * scale) H_B) * s for [rows, dim].
 *
 *   codes, scales  as produced by hadq_rotate_quantize with the same dim,
 *                  block, signs, bits and group (device pointers).  INT4 code
 *                  -8 is accepted and dequantised as -8 * scale.
 *   out            device output [rows, dim]: bfloat16 (round to nearest
 *                  even, 2-byte aligned) or float32 (4-byte aligned),
 *                  chosen by out_dtype.
 *   Other arguments and rules as for hadq_rotate_quantize.
 */
hadq_status hadq_dequant_rotate_inv(const void *codes, const float *scales, int64_t rows,
                                    int32_t dim, int32_t block, const int8_t *signs,
                                    int32_t bits, int32_t group, void *out,
                                    hadq_out_dtype out_dtype, hadq_stream_t stream);

/*
 * hadq_rotate_quantize_kron -- Kronecker rotation + quantisation for widths
 * a * b without a Sylvester matrix of their own: y = (F (x) H_b)(x * s), then
 * the symmetric quantiser of hadq_rotate_quantize.  QuaRot's online down_proj
 * rotation uses such a Kronecker-product matrix, and widths without a
 * Sylvester matrix take a stored Hadamard matrix ("QuaRot: rotation-based
 * outlier suppression", msModelSlim, online rotation and FAQ).
 *
 *   x     device bf16 [rows, a * b]; element i * b + j of a row is X[i][j].
 *   a     1..256; fa: device float32 [a][a], row-major, the factor exactly as
 *         it multiplies (for a stored +-1 Hadamard matrix S_a: S_a / sqrt(a);
 *         any orthogonal matrix gives a rotation).  y = vec(F X H_b^T).
 *   b     power of two >= 2; H_b is the normalised Sylvester matrix.
 *   signs, bits, group, codes, scales, rotated_out: as for
 *         hadq_rotate_quantize with dim = a * b (group divides a * b).
 *   Shared memory grows with a * b and a^2: combinations above 227 KB
 *   (about a * b > 24000 for small a) return HADQ_ERR_UNSUPPORTED.
 */
hadq_status hadq_rotate_quantize_kron(const void *x, int64_t rows, int32_t a, const float *fa,
                                      int32_t b, const int8_t *signs, int32_t bits, int32_t group,
                                      void *codes, float *scales, float *rotated_out,
                                      hadq_stream_t stream);

/*
 * hadq_dequant_rotate_inv_kron -- x_hat = ((F^T (x) H_b)(q * scale)) * s, the
 * inverse for an orthogonal F, with the codes and scales of
 * hadq_rotate_quantize_kron (same a, fa, b, signs, bits, group).  Output as
 * for hadq_dequant_rotate_inv.
 */
hadq_status hadq_dequant_rotate_inv_kron(const void *codes, const float *scales, int64_t rows,
                                         int32_t a, const float *fa, int32_t b,
                                         const int8_t *signs, int32_t bits, int32_t group,
                                         void *out, hadq_out_dtype out_dtype,
                                         hadq_stream_t stream);

/*
 * hadq_rotate_quantize_kron_pm1 / hadq_dequant_rotate_inv_kron_pm1 -- the
 * same transforms with the factor given as the stored +-1 Hadamard matrix
 * itself: F = S_a / sqrt(a) ("QuaRot: rotation-based outlier suppression",
 * msModelSlim, online rotation: widths without a Sylvester matrix use a
 * stored Hadamard matrix).
 *
 *   sa    device int8 [a][a], row-major, entries +1 / -1 (other values are
 *         used as given: the factor is whatever S_a / sqrt(a) they form).
 *   All other arguments, layouts, errors and outputs as for
 *   hadq_rotate_quantize_kron / hadq_dequant_rotate_inv_kron.
 * With a +-1 factor the tensor-core variant (see hadq_kron_plan) mixes with
 * S_a exactly, one bf16 term instead of three, and folds 1 / sqrt(a) into the
 * scale; the other variants multiply S_a by 1 / sqrt(a) (rounded to float32)
 * as they load it.
 */
hadq_status hadq_rotate_quantize_kron_pm1(const void *x, int64_t rows, int32_t a, const int8_t *sa,
                                          int32_t b, const int8_t *signs, int32_t bits,
                                          int32_t group, void *codes, float *scales,
                                          float *rotated_out, hadq_stream_t stream);
hadq_status hadq_dequant_rotate_inv_kron_pm1(const void *codes, const float *scales, int64_t rows,
                                             int32_t a, const int8_t *sa, int32_t b,
                                             const int8_t *signs, int32_t bits, int32_t group,
                                             void *out, hadq_out_dtype out_dtype,
                                             hadq_stream_t stream);

/*
 * hadq_kron_plan -- host-only: validate the sizes of a Kronecker call
 * (direction 0 = hadq_rotate_quantize_kron, 1 = its inverse) and report the
 * kernel variant it would launch.  `aligned16` says whether every pointer of
 * the call is 16-byte aligned.  The forward takes
 *   HADQ_KRON_MMA    for a <= 32, 16 <= b <= 512, a * b a multiple of 512 and
 *                    at most 8192, groups of 16..512 columns with
 *                    G / 16 dividing 32, all pointers 16-byte aligned;
 *   HADQ_KRON_REG16  for the same b, group and alignment otherwise, with
 *                    a * b <= 16384;
 *   HADQ_KRON_SMEM   for everything else.
 * Returns the status the call would return for these sizes (pointer checks
 * aside) and writes the variant to *variant.  Touches no GPU.
 */
hadq_status hadq_kron_plan(int32_t direction, int64_t rows, int32_t a, int32_t b, int32_t bits,
                           int32_t group, int32_t aligned16, int32_t *variant);

/*
 * hadq_rotate_quantize_asym -- rotate, then quantise with a zero point
 * ("Hartmann rotation, lightweight QAT, streaming attention", section 2, the
 * FakeQuantize forward: x_int = round(x / scale) + zero_point, clamped to
 * [0, 2^b - 1]).  Scale and zero point come from each group's range, which
 * always holds 0:
 *   lo = min(0, min y), hi = max(0, max y), scale = (hi - lo) / (2^b - 1),
 *   zero_point = clamp(round(-lo / scale), 0, 2^b - 1),
 *   q = clamp(round(y / scale) + zero_point, 0, 2^b - 1),
 * rounding half to even; an all-zero group gets scale 0, zero point 0, codes 0.
 *
 *   codes        device output, unsigned: bits 8 -> uint8 [rows, dim]; bits 4
 *                -> uint8 [rows, dim/2], element 2j in the low nibble, values
 *                0..15.
 *   scales       device output float32 [rows, dim/G].
 *   zero_points  device output uint8 [rows, dim/G].
 *   Other arguments as for hadq_rotate_quantize.  Kernel coverage: dim a
 *   multiple of 128, block 8..128, group 128 x (1, 2, 4, .., 32) columns (-1
 *   for rows of such a width), x, codes and signs 16-byte aligned; other valid
 *   combinations return HADQ_ERR_UNSUPPORTED.
 */
hadq_status hadq_rotate_quantize_asym(const void *x, int64_t rows, int32_t dim, int32_t block,
                                      const int8_t *signs, int32_t bits, int32_t group, void *codes,
                                      float *scales, uint8_t *zero_points, hadq_stream_t stream);

/*
 * hadq_dequant_rotate_inv_asym -- x_hat = (((q - zero_point) * scale) H_B) * s
 * for codes, scales and zero points written by hadq_rotate_quantize_asym (same
 * dim, block, signs, bits, group).  Output as for hadq_dequant_rotate_inv
 * (16-byte aligned); same kernel coverage as the forward call.
 */
hadq_status hadq_dequant_rotate_inv_asym(const void *codes, const float *scales,
                                         const uint8_t *zero_points, int64_t rows, int32_t dim,
                                         int32_t block, const int8_t *signs, int32_t bits,
                                         int32_t group, void *out, hadq_out_dtype out_dtype,
                                         hadq_stream_t stream);

/*
 * hadq_rotate_quantize_keep -- mixed-precision KV quantisation: a few tokens
 * stay in bf16, every other row is rotated and quantised as by
 * hadq_rotate_quantize ("HyQuant: mixed-precision quantisation for LLM
 * attention", method, key modules: vertical-line tokens and a local window
 * stay in full precision, the rest goes to low bit; the decode stage applies
 * the same split to the KV cache).
 *
 *   x          device bf16 [heads, tokens, dim]: row h * tokens + t.
 *   keep_slot  device int32 [tokens]: token t is kept when keep_slot[t] lies
 *              in [0, n_keep); any other value means "quantise".  Kept tokens
 *              should have distinct slots (two tokens on one slot leave
 *              either row there).  Which tokens to keep (sinks, vertical
 *              lines, a window) is the caller's choice.
 *   kept       device bf16 [heads, n_keep, dim] output, 16-byte aligned:
 *              kept[h][keep_slot[t]] = x[h][t], bit for bit.  May be NULL
 *              when n_keep == 0.
 *   codes,     as for hadq_rotate_quantize; the rows of kept tokens get codes 0
 *   scales     and scale 0.
 *   Other arguments as for hadq_rotate_quantize.  Kernel coverage: dim a
 *   multiple of 128 (at most 16384 when a group is wider than 128), block
 *   8..128, group = 128 x (1, 2, 4, .., 32) columns (-1 for a row of that
 *   width), fewer than 2^31 chunks of 128 columns, x, codes and signs
 *   16-byte aligned; other valid combinations return HADQ_ERR_UNSUPPORTED.
 */
hadq_status hadq_rotate_quantize_keep(const void *x, int64_t heads, int64_t tokens, int32_t dim,
                                      int32_t block, const int8_t *signs, int32_t bits,
                                      int32_t group, const int32_t *keep_slot, int32_t n_keep,
                                      void *codes, float *scales, void *kept,
                                      hadq_stream_t stream);

/*
 * hadq_dequant_rotate_inv_keep -- reads a mixed-precision cache back: rows of
 * kept tokens return their bf16 values from `kept` exactly (widened for
 * float32 output), every other row is dequantised and rotated back as by
 * hadq_dequant_rotate_inv.  Arguments as for hadq_rotate_quantize_keep and
 * hadq_dequant_rotate_inv (out 16-byte aligned, same kernel coverage).
 */
hadq_status hadq_dequant_rotate_inv_keep(const void *codes, const float *scales, const void *kept,
                                         const int32_t *keep_slot, int32_t n_keep, int64_t heads,
                                         int64_t tokens, int32_t dim, int32_t block,
                                         const int8_t *signs, int32_t bits, int32_t group,
                                         void *out, hadq_out_dtype out_dtype, hadq_stream_t stream);

/*
 * hadq_kv_decode_attention -- one decode step of attention over a KV cache
 * stored in the rotated basis as INT4 or INT8 codes.
 *
 * The cache rows are what hadq_rotate_quantize writes for dim 128, block 128
 * (or -1), group 128 (or -1), 64 or 32, bits 4 or 8 and the same signs:
 * K_rot = (K * s) H and V_rot = (V * s) H, quantised per row or per group.  Because H is orthogonal,
 * (q H)(K H)^T = q K^T ("Hartmann rotation, lightweight QAT, streaming
 * attention", section 1), so the scores come from the rotated query against
 * the dequantised rotated keys, and the output is rotated back once ("QuaRot
 * hands-on", sections 2.2 and 2.3: the 4-bit KV cache is dequantised when read,
 * the output transformed back):
 *
 *   q_rot  = (q * s) H
 *   p      = softmax_t( softmax_scale * q_rot . (kcode_t * kscale_t) )
 *   out    = ((sum_t p_t * vcode_t * vscale_t) H) * s
 *
 * (kscale_t, vscale_t: the scale of each element's group.)
 *
 *   q            device, bfloat16 [batch, n_q_heads, dim], 8-byte aligned.
 *   k_codes,     device [batch, n_kv_heads, token_stride, dim/2] bytes of packed
 *   v_codes      INT4 (element 2j in the low nibble of byte j), or [..., dim]
 *                int8 for bits 8; 16-byte aligned.  Only the first `tokens`
 *                rows of each head are read.
 *   k_scales,    device, float32 [batch, n_kv_heads, token_stride, 128/group]:
 *   v_scales     the per-group scales of the codes (one per row for group 128),
 *                4-byte aligned; for group 64 or 32, 16-byte aligned with
 *                token_stride * 128/group a multiple of 4 (HADQ_ERR_MISALIGNED
 *                otherwise).
 *   batch        >= 0 (0 = empty call).
 *   n_q_heads    >= 1, a multiple of n_kv_heads; query head h reads KV head
 *                h / (n_q_heads / n_kv_heads) (grouped-query attention).
 *   tokens       cached tokens attended over, 1 <= tokens <= token_stride,
 *                at most 2^30 (HADQ_ERR_UNSUPPORTED beyond).
 *   dim, block,  the cache's rotate+quantise parameters; the kernel supports
 *   bits, group  dim 128, block 128 or -1, bits 4 or 8, group 128 (or -1), 64 or 32
 *                and returns HADQ_ERR_UNSUPPORTED for any other valid
 *                combination.
 *   signs        device int8 [dim] (4-byte aligned) or NULL, as for the cache.
 *   softmax_scale  > 0 and finite (usually 1/sqrt(dim)).
 *   out          device output [batch, n_q_heads, dim]: bfloat16 (8-byte
 *                aligned) or float32 (16-byte aligned).
 *   workspace    device scratch of at least hadq_kv_decode_workspace_size()
 *                bytes, 256-byte aligned, owned by the caller.  It must be
 *                zero-filled before its first use; every call leaves it ready
 *                for the next one.  Calls sharing a workspace must be ordered
 *                (same stream, or synchronised).
 * Queries whose scaled rotated entries are all below 2^-100 in magnitude are
 * treated as zero (uniform weights).  No other rounding beyond float32.
 */
hadq_status hadq_kv_decode_attention(const void *q, const void *k_codes, const float *k_scales,
                                     const void *v_codes, const float *v_scales, int32_t batch,
                                     int32_t n_q_heads, int32_t n_kv_heads, int64_t tokens,
                                     int64_t token_stride, int32_t dim, int32_t block,
                                     const int8_t *signs, int32_t bits, int32_t group,
                                     float softmax_scale, void *out, hadq_out_dtype out_dtype,
                                     void *workspace, size_t workspace_bytes,
                                     hadq_stream_t stream);

/*
 * hadq_kv_decode_workspace_size -- host-only: bytes of workspace that
 * hadq_kv_decode_attention needs for these sizes on any device (an upper bound
 * that does not depend on the GPU).  Writes *bytes; validates like the call.
 */
hadq_status hadq_kv_decode_workspace_size(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                          int64_t tokens, size_t *bytes);

/*
 * hadq_kv_decode_attention_noalloc -- hadq_kv_decode_attention without a
 * caller workspace: the split partials and arrival counters live in a 16 MiB
 * scratch array that the library holds as a static device variable (256-byte
 * aligned, zero when the library loads, left at zero by every call).  Nothing
 * is allocated per call.
 *
 *   Arguments, layouts and results as for hadq_kv_decode_attention.
 *   Sizes whose partials exceed the scratch return HADQ_ERR_UNSUPPORTED
 *   (use hadq_kv_decode_attention with a workspace then).
 *   All calls in a process share the one scratch per device, so calls that
 *   could overlap on the GPU (different streams, no synchronisation) must not
 *   both use this entry point.
 */
hadq_status hadq_kv_decode_attention_noalloc(const void *q, const void *k_codes,
                                             const float *k_scales, const void *v_codes,
                                             const float *v_scales, int32_t batch,
                                             int32_t n_q_heads, int32_t n_kv_heads,
                                             int64_t tokens, int64_t token_stride, int32_t dim,
                                             int32_t block, const int8_t *signs, int32_t bits,
                                             int32_t group, float softmax_scale, void *out,
                                             hadq_out_dtype out_dtype, hadq_stream_t stream);

/*
 * hadq_plan -- host-only: validate the sizes of a call and report the kernel
 * family it would use.  direction 0 = rotate_quantize, 1 = dequant_rotate_inv.
 * `aligned16` says whether every pointer of the call is 16-byte aligned.
 * Returns the same status the call would return for these sizes (pointer
 * checks aside) and writes the path to *path.  Touches no GPU.  A forward
 * call planned as HADQ_PATH_H4096_TC that also asks for rotated_out runs
 * HADQ_PATH_WIDE4096_MMA instead.
 */
hadq_status hadq_plan(int32_t direction, int64_t rows, int32_t dim, int32_t block,
                      int32_t bits, int32_t group, int32_t has_signs, int32_t aligned16,
                      hadq_path *path);

/*
 * hadq_device_status -- synchronise `stream`, then report whether any bounded
 * wait inside the library's tcgen05 kernels (HADQ_PATH_H4096_TC) ran out on
 * the current device since the previous call, and clear the record.
 * HADQ_OK if none did; HADQ_ERR_DEVICE if one did (the outputs of the call
 * that gave up are void: every role of the kernel left its loop, waited for
 * its copies in flight and freed its tensor memory, so the context stays
 * usable); HADQ_ERR_CUDA if the synchronisation or the read failed.
 */
hadq_status hadq_device_status(hadq_stream_t stream);

/*
 * hadq_selftest_bounded_wait -- test of the bounded waits: launches the
 * HADQ_PATH_H4096_TC kernel on four blocks with the load of its only tile
 * withheld, so that every wait for it runs out (about one second), then
 * returns hadq_device_status(stream).  HADQ_ERR_DEVICE is the expected
 * result; afterwards the record is clear and the context usable.
 *   scratch  device buffer of at least 40976 bytes, 16-byte aligned, owned by
 *            the caller (the kernel is given it as input and outputs; with
 *            the load withheld it writes nothing).
 * Synchronises `stream`.
 */
hadq_status hadq_selftest_bounded_wait(void *scratch, hadq_stream_t stream);

/* Static description of a status code. */
const char *hadq_status_str(hadq_status status);

/* Detail of the most recent failure in the calling host thread ("" if none). */
const char *hadq_last_error(void);

/* Number of kernel launches issued by this process so far (all threads). */
int64_t hadq_launch_count(void);

/* ABI version, currently 1. */
int32_t hadq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HADQ_H */
