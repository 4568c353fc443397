// Host versions of the CUDA features the lean attend and append kernels use, for running their source on
// host threads (test infrastructure): one std::thread per CUDA thread; __syncthreads, the
// cluster barrier, __syncwarp, shuffles, ballots and warp reductions are real rendezvous
// of the threads that must take part, and a barrier that does not complete within 20 s
// reports where every thread waits.
#pragma once
#include <atomic>
#include <chrono>
#include <cmath>
#include <condition_variable>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#define __device__
#define __global__
#define __host__
#define __forceinline__ inline
#define __launch_bounds__(...)
#define __align__(n) alignas(n)
#define __shared__

struct alignas(8) uint2 { uint32_t x, y; };
struct alignas(16) uint4 { uint32_t x, y, z, w; };
struct alignas(8) float2 { float x, y; };
struct alignas(16) float4 { float x, y, z, w; };
inline uint2 make_uint2(uint32_t a, uint32_t b) { return {a, b}; }
inline uint4 make_uint4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) { return {a, b, c, d}; }
inline float2 make_float2(float a, float b) { return {a, b}; }
inline float4 make_float4(float a, float b, float c, float d) { return {a, b, c, d}; }

namespace emu {

struct Where {
  std::atomic<int> line{0};
  std::atomic<const char *> what{""};
};

// Barrier with a timeout; on timeout prints the waiting census and aborts.
struct TBarrier {
  std::mutex mu;
  std::condition_variable cv;
  int count = 0, arrived = 0;
  long gen = 0;
  std::string name;
  void init(int n, std::string nm) {
    count = n;
    arrived = 0;
    gen = 0;
    name = std::move(nm);
  }
  void wait(int line);
  long arrive(int line);             // split form: returns the generation to wait for
  void wait_gen(long my, int line);
};

extern thread_local int t_tid, t_block, t_crank, t_cs, t_grid;
extern int g_nt;  // threads per CTA
extern thread_local long t_cluster_gen;  // cluster-barrier generation this thread arrived at
extern thread_local unsigned char *t_smem;
extern std::vector<unsigned char *> g_cluster_smem;  // per cluster rank
extern size_t g_smem_bytes;
extern std::vector<TBarrier> g_cta_bar;       // per cluster rank
extern TBarrier g_cluster_bar;
extern std::vector<TBarrier> g_warp_bar;      // per (rank, warp)
extern std::vector<uint32_t> g_warp_slot;     // per (rank, warp, lane)
extern std::vector<Where> g_where;            // per (rank, tid)

void report_and_abort(const char *why);

inline void TBarrier::wait(int line) {
  g_where[t_crank * g_nt + t_tid].line = line;
  g_where[t_crank * g_nt + t_tid].what = name.c_str();
  std::unique_lock<std::mutex> lk(mu);
  const long my = gen;
  if (++arrived == count) {
    arrived = 0;
    ++gen;
    cv.notify_all();
    return;
  }
  if (!cv.wait_for(lk, std::chrono::seconds(20), [&] { return gen != my; })) {
    lk.unlock();
    char buf[256];
    snprintf(buf, sizeof buf, "barrier '%s' at line %d timed out (%d of %d arrived)", name.c_str(), line, arrived,
             count);
    report_and_abort(buf);
  }
}

inline long TBarrier::arrive(int line) {
  g_where[t_crank * g_nt + t_tid].line = line;
  g_where[t_crank * g_nt + t_tid].what = "cluster-arrive";
  std::lock_guard<std::mutex> lk(mu);
  const long my = gen;
  if (++arrived == count) {
    arrived = 0;
    ++gen;
    cv.notify_all();
  }
  return my;
}

inline void TBarrier::wait_gen(long my, int line) {
  g_where[t_crank * g_nt + t_tid].line = line;
  g_where[t_crank * g_nt + t_tid].what = name.c_str();
  std::unique_lock<std::mutex> lk(mu);
  if (!cv.wait_for(lk, std::chrono::seconds(20), [&] { return gen != my; })) {
    lk.unlock();
    char buf[256];
    snprintf(buf, sizeof buf, "barrier '%s' (split wait) at line %d timed out", name.c_str(), line);
    report_and_abort(buf);
  }
}

}  // namespace emu

struct ThreadIdx { unsigned x; };
#define threadIdx (ThreadIdx{(unsigned)emu::t_tid})
#define blockIdx (ThreadIdx{(unsigned)emu::t_block})
#define gridDim (ThreadIdx{(unsigned)emu::t_grid})

#define __syncthreads() emu::g_cta_bar[emu::t_crank].wait(__LINE__)
#define __syncwarp(...) emu::g_warp_bar[emu::t_crank * (emu::g_nt / 32) + emu::t_tid / 32].wait(__LINE__)

namespace emu {
template <typename T>
inline T warp_exchange(T v, int src, int line) {
  static_assert(sizeof(T) == 4, "32-bit values only");
  const int w = t_crank * (g_nt / 32) + t_tid / 32, lane = t_tid & 31;
  uint32_t u;
  std::memcpy(&u, &v, 4);
  g_warp_slot[w * 32 + lane] = u;
  g_warp_bar[w].wait(line);
  const uint32_t r = g_warp_slot[w * 32 + (src & 31)];
  g_warp_bar[w].wait(line);
  T out;
  std::memcpy(&out, &r, 4);
  return out;
}
}  // namespace emu
#define __shfl_sync(m, v, s) emu::warp_exchange((v), (s), __LINE__)
#define __shfl_xor_sync(m, v, x) emu::warp_exchange((v), (emu::t_tid & 31) ^ (x), __LINE__)
namespace emu {
inline unsigned ballot(bool p, int line) {
  const int w = t_crank * (g_nt / 32) + t_tid / 32, lane = t_tid & 31;
  g_warp_slot[w * 32 + lane] = p ? 1u : 0u;
  g_warp_bar[w].wait(line);
  unsigned b = 0;
  for (int i = 0; i < 32; ++i) b |= (g_warp_slot[w * 32 + i] ? 1u : 0u) << i;
  g_warp_bar[w].wait(line);
  return b;
}
}  // namespace emu
#define __ballot_sync(m, p) emu::ballot((p), __LINE__)
#define __all_sync(m, p) (emu::ballot((p), __LINE__) == 0xffffffffu)

inline int __popc(uint32_t x) { return __builtin_popcount(x); }
inline int __clz(uint32_t x) { return x ? __builtin_clz(x) : 32; }
inline uint32_t __umulhi(uint32_t a, uint32_t b) { return (uint32_t)(((uint64_t)a * b) >> 32); }
inline float __expf(float x) { return std::exp(x); }
inline float2 __fmul2_rn(float2 a, float2 b) { return {a.x * b.x, a.y * b.y}; }
inline float2 __ffma2_rn(float2 a, float2 b, float2 c) { return {std::fma(a.x, b.x, c.x), std::fma(a.y, b.y, c.y)}; }
inline float2 __fadd2_rn(float2 a, float2 b) { return {a.x + b.x, a.y + b.y}; }
inline float __fmaf_rn(float a, float b, float c) { return std::fma(a, b, c); }
template <typename T>
inline T __ldg(const T *p) { return *p; }
inline uint32_t atomicOr(uint32_t *p, uint32_t v) { return __atomic_fetch_or(p, v, __ATOMIC_SEQ_CST); }
inline float __uint_as_float(uint32_t u) { float f; std::memcpy(&f, &u, 4); return f; }
inline uint32_t __float_as_uint(float f) { uint32_t u; std::memcpy(&u, &f, 4); return u; }

namespace cg {
struct cluster_group {
  unsigned block_rank() const { return (unsigned)emu::t_crank; }
  template <typename T>
  T *map_shared_rank(T *p, unsigned rank) const {
    const unsigned char *b = emu::t_smem;
    const unsigned char *c = reinterpret_cast<const unsigned char *>(p);
    if (c < b || c >= b + emu::g_smem_bytes || rank >= (unsigned)emu::t_cs) {
      emu::report_and_abort("map_shared_rank of a pointer outside shared memory or to a bad rank");
    }
    return reinterpret_cast<T *>(emu::g_cluster_smem[rank] + (c - b));
  }
};
inline cluster_group this_cluster() { return {}; }
}  // namespace cg
inline int min(int a, int b) { return a < b ? a : b; }
inline int max(int a, int b) { return a > b ? a : b; }
inline long long min(long long a, long long b) { return a < b ? a : b; }
inline long long max(long long a, long long b) { return a > b ? a : b; }
inline long min(long a, long b) { return a < b ? a : b; }
inline long max(long a, long b) { return a > b ? a : b; }
namespace emu {
inline unsigned warp_reduce(unsigned v, bool is_max, int line) {
  const int w = t_crank * (g_nt / 32) + t_tid / 32, lane = t_tid & 31;
  g_warp_slot[w * 32 + lane] = v;
  g_warp_bar[w].wait(line);
  unsigned r = g_warp_slot[w * 32];
  for (int i = 1; i < 32; ++i) {
    const unsigned x = g_warp_slot[w * 32 + i];
    r = is_max ? (x > r ? x : r) : (x < r ? x : r);
  }
  g_warp_bar[w].wait(line);
  return r;
}
}  // namespace emu
#define __reduce_max_sync(m, v) emu::warp_reduce((v), true, __LINE__)
#define __reduce_min_sync(m, v) emu::warp_reduce((v), false, __LINE__)
namespace emu {
// __syncthreads_and: every thread's predicate, one barrier, the AND to all
extern std::vector<uint32_t> g_cta_pred;  // per (rank, tid)
inline int cta_and(bool p, int line) {
  g_cta_pred[t_crank * g_nt + t_tid] = p ? 1u : 0u;
  g_cta_bar[t_crank].wait(line);
  int all = 1;
  for (int i = 0; i < g_nt; ++i) all &= (int)g_cta_pred[t_crank * g_nt + i];
  g_cta_bar[t_crank].wait(line);
  return all;
}
// mbarrier with transaction counts: a phase completes when its arrivals and its expected
// bytes are all in
struct MBar {
  std::mutex mu;
  int count = 0, pending = 0;
  long tx = 0;
  long completed = 0;  // phases completed so far
};
MBar &mbar_of(const void *p);
inline bool g_mbar_stuck = false;  // every mbarrier wait fails (the timeout path)
inline void mbar_complete_if_done(MBar &b) {
  if (b.pending == 0 && b.tx == 0) {
    ++b.completed;
    b.pending = b.count;
  }
}
}  // namespace emu
#define __syncthreads_and(p) emu::cta_and((p), __LINE__)
inline unsigned max(unsigned a, unsigned b) { return a > b ? a : b; }
inline unsigned min(unsigned a, unsigned b) { return a < b ? a : b; }
