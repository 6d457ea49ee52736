// Kernel pointers of one kernel family, instantiated in this translation unit
// (the families compile in parallel; the C ABI in hadq_api.cu only calls these).
#include "hadq_kernels.h"
#include "hadq_blocked.cuh"

namespace hadq {
namespace {

template <int LOG_B, int BITS, int MAXT>
const void* rq_blocked_fn(bool signs) {
  return signs ? (const void*)rq_blocked_kernel<LOG_B, BITS, true, MAXT>
               : (const void*)rq_blocked_kernel<LOG_B, BITS, false, MAXT>;
}

template <int LOG_B, int BITS, int MAXT>
const void* dq_blocked_fn(bool signs, bool f32) {
  if (signs) return f32 ? (const void*)dq_blocked_kernel<LOG_B, BITS, true, true, MAXT>
                        : (const void*)dq_blocked_kernel<LOG_B, BITS, true, false, MAXT>;
  return f32 ? (const void*)dq_blocked_kernel<LOG_B, BITS, false, true, MAXT>
             : (const void*)dq_blocked_kernel<LOG_B, BITS, false, false, MAXT>;
}

template <int LOG_B, int BITS, int MAXT>
const void* pick_blocked_b(int direction, bool signs, bool f32) {
  return direction == 0 ? rq_blocked_fn<LOG_B, BITS, MAXT>(signs) : dq_blocked_fn<LOG_B, BITS, MAXT>(signs, f32);
}

template <int BITS, int MAXT>
const void* pick_blocked_t(int direction, int B, bool signs, bool f32) {
  switch (B) {
    case 32: return pick_blocked_b<5, BITS, MAXT>(direction, signs, f32);
    case 64: return pick_blocked_b<6, BITS, MAXT>(direction, signs, f32);
    case 128: return pick_blocked_b<7, BITS, MAXT>(direction, signs, f32);
    default: return pick_blocked_b<8, BITS, MAXT>(direction, signs, f32);
  }
}

const void* pick_blocked(int direction, int bits, int B, bool signs, bool f32, int threads) {
  if (threads <= 256)
    return bits == 8 ? pick_blocked_t<8, 256>(direction, B, signs, f32) : pick_blocked_t<4, 256>(direction, B, signs, f32);
  return bits == 8 ? pick_blocked_t<8, 512>(direction, B, signs, f32) : pick_blocked_t<4, 512>(direction, B, signs, f32);
}

}  // namespace

const void* blocked_kernel_ptr(int direction, int bits, int B, bool signs, bool f32, int threads) {
  return pick_blocked(direction, bits, B, signs, f32, threads);
}

}  // namespace hadq
