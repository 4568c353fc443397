// Host versions of the device helpers the lean attend kernel includes (test infrastructure).
#pragma once
#include <thread>

#include "emu_cuda.h"
#include "recsa_internal.h"
namespace recsa {
inline float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
inline float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }
inline uint32_t f32_to_bf16_bits(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7fffu + ((u >> 16) & 1u);
  return u >> 16;
}
inline uint32_t pack_bf16x2(float lo, float hi) { return f32_to_bf16_bits(lo) | (f32_to_bf16_bits(hi) << 16); }
inline uint32_t order_key(float f) {
  f += 0.0f;
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
#define cluster_barrier() \
  do { __syncwarp(); emu::g_cluster_bar.wait(__LINE__); } while (0)
#define cluster_arrive() \
  do { emu::t_cluster_gen = emu::g_cluster_bar.arrive(__LINE__); } while (0)
#define cluster_wait() \
  do { emu::g_cluster_bar.wait_gen(emu::t_cluster_gen, __LINE__); } while (0)
// a shared-memory "address": the offset from the CTA's shared memory
inline uint32_t smem_u32(const void *p) {
  return (uint32_t)(static_cast<const unsigned char *>(p) - emu::t_smem);
}
// the poll limit of a bounded wait; the "stuck" case lowers it (every wait then runs out)
inline uint32_t kMbarPolls = 1u << 16;
inline void mbar_init(uint64_t *bar, uint32_t count) {
  emu::MBar &b = emu::mbar_of(bar);
  std::lock_guard<std::mutex> lk(b.mu);
  b.count = b.pending = (int)count;
  b.tx = 0;
  b.completed = 0;
}
inline void mbar_fence_init() {}
inline void mbar_arrive(uint64_t *bar) {
  emu::MBar &b = emu::mbar_of(bar);
  std::lock_guard<std::mutex> lk(b.mu);
  --b.pending;
  emu::mbar_complete_if_done(b);
}
inline bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  if (emu::g_mbar_stuck) {  // a barrier that never completes: the wait must give up
    std::this_thread::yield();
    return false;
  }
  emu::MBar &b = emu::mbar_of(bar);
  bool done;
  {
    std::lock_guard<std::mutex> lk(b.mu);
    done = (uint32_t)(b.completed & 1) != parity;  // the phase of this parity has completed
  }
  if (!done) std::this_thread::yield();
  return done;
}
inline bool mbar_wait(uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < kMbarPolls; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}
}  // namespace recsa
