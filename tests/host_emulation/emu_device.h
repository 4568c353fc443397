// Host versions of the device helpers the lean attend kernel includes (test infrastructure).
#pragma once
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
}  // namespace recsa
