// Fused level-wise sparse attend (decode and causal prefill).
//
// Recursive Sparse Attention, abstract: each level above the tokens keeps at most k
// candidates, so a query reads O(log L) entries; the summaries of the candidates it
// does not keep share one softmax with the exact tokens; every entry is RoPE-rotated
// at its index among the candidates of its level.
//
// A tile is one (sequence, query, KV group): the G query heads of the group descend
// the group's tree together and select with the sum of their logits.  Per level a
// tile (1) rotates its heads at position n (the level's candidate count), (2) gathers
// the candidates' 256-byte bf16 key rows and RoPE-table rows, rotates each key at its
// candidate index and scores it, (3) keeps the top k by (group score desc, index asc),
// (4) folds the value rows of the candidates it does not keep into an fp32 online
// softmax and (5) expands the kept nodes (and, in causal prefill, the forced partial
// node) into the next level's candidate list, in node order.  The token level scores
// and folds every candidate.
//
// Two launch shapes share the row helpers below:
//   attend_cta_kernel  - one CTA, or a cluster of 2 or 4 CTAs, per tile.  Each level
//     costs one round trip to memory: key, value and table rows are issued together
//     (values speculatively), scores go to every CTA of the cluster through DSMEM, one
//     warp selects and expands while the others fold.  For few tiles (latency).
//   attend_warp_kernel - one warp per tile, persistent, no block-level barriers.  For
//     many tiles (prefill, batched decode): thousands of tiles are in flight.
// Rows are read with one half-warp per row: lane j (0..15) holds dims 4j..4j+3 and
// 64+4j..64+4j+3, which are exactly the RoPE pairs (i, i+64) it needs.
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "recsa_device.cuh"
#include "recsa_internal.h"

namespace cg = cooperative_groups;

namespace recsa {
namespace {

constexpr uint32_t kForced = 0x80000000u;  // candidate is a forced partial node
constexpr uint32_t kKept = 0x40000000u;    // candidate kept by top-k
constexpr uint32_t kNodeMask = 0x3fffffffu;
constexpr int kCtaThreads = 256;
constexpr int kCtaWarps = kCtaThreads / 32;
constexpr int kHalfWarps = 2 * kCtaWarps;           // 16 row slots per CTA
constexpr int kWarpKernelMaxWarps = 8;
constexpr int kTopkRegs = 8;                        // iterative top-k handles up to 256 candidates
// merge rows: m, l, 2 pad, acc[128] (the accumulator starts 16-byte aligned)
constexpr int kRedStride = kD + 4;
// CTA kernel scratch ints: [1] workspace bad, [2, 2 + 2W) per-warp ballot totals,
// [kNextCount + parity] next level's candidate count
constexpr int kNextCount = 2 + 2 * (kCtaThreads / 32);
constexpr int kMiscInts = kNextCount + 2;

struct AttendArgs {
  const uint16_t *k_tok, *v_tok, *k_node, *v_node;
  const uint16_t *q;
  void *out;
  const float2 *table;
  WsHeader *hdr;
  int32_t *sel_idx;
  int32_t *entries;
  const int64_t *seq_len;  // per-sequence lengths (NULL: every sequence has `length`)
  const int32_t *page_table;  // paged token caches: [B][cap >> page_shift] (NULL: contiguous)
  int32_t page_shift, num_pages;
  int64_t cap;
  int64_t length;  // decode: L; prefill: L before the chunk (the longest, with seq_len)
  int64_t row_off[kMaxLevels + 1];
  int64_t slots[kMaxLevels + 1];
  int32_t span[kMaxLevels + 1];   // b^l, saturated above any capacity
  int32_t nlen[kMaxLevels + 1];   // ceil(length / b^l): nodes of level l at the call's length
  int32_t levels;                 // levels above the tokens at capacity
  int32_t hkv, hq, b, top_k, nq, causal, out_fp32;
  int32_t sel_levels;
  int32_t table_rows_needed;
  int32_t max_cand;         // candidate buffer rows (multiple of 32)
  int32_t own_max;          // CTA kernel: logit rows per CTA
  int32_t tiles;
  int32_t warps_per_block;  // warp kernel
  float scale;
};

template <int G>
__host__ __device__ constexpr int log2g() {
  return G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : 3;
}

// ------------------------------------------------------------------ tile geometry

// Per-level geometry, copied to shared memory at kernel start (the level index is a
// runtime value; shared memory serves it without touching the parameter bank).
struct Geo {
  long long row_off[kMaxLevels + 1];
  long long slots[kMaxLevels + 1];
  int span[kMaxLevels + 1];
  int nlen[kMaxLevels + 1];
};
constexpr int kGeoBytes = (int)sizeof(Geo);

__device__ __forceinline__ void load_geo(const AttendArgs &a, Geo *g, int tid, int nthreads) {
  for (int l = tid; l <= kMaxLevels; l += nthreads) {
    g->row_off[l] = a.row_off[l];
    g->slots[l] = a.slots[l];
    g->span[l] = a.span[l];
    g->nlen[l] = a.nlen[l];
  }
}

struct TileInfo {
  int s, g, qi, T, p;
  int64_t bh;
};

__device__ __forceinline__ TileInfo tile_info(const AttendArgs &a, const Geo &geo, int tile) {
  TileInfo t;
  t.qi = tile % a.nq;
  const int sg = tile / a.nq;
  t.g = sg % a.hkv;
  t.s = sg / a.hkv;
  // a sequence's own length, held to [0, length] (the workspace check flags an entry outside)
  const int64_t len = a.seq_len ? min(max(a.seq_len[t.s], (int64_t)0), a.length) : a.length;
  t.p = (int)(a.causal ? len + t.qi : len);
  t.bh = (int64_t)t.s * a.hkv + t.g;
  // levels above the tokens: ceil(p / b^T) <= b  <=>  p <= b^(T+1), so T = #{l >= 1 : b^l < p}
  int T = 0;
  while (T < a.levels && geo.span[T + 1] < t.p) ++T;
  t.T = T;
  return t;
}

// Nodes of a level whose nodes span `span` tokens, over `p` tokens: ceil(p / span).
__device__ __forceinline__ int nodes_at(int p, int span) {
  return (int)(((uint32_t)p + (uint32_t)span - 1u) / (uint32_t)span);  // p < 2^31, span <= 2^30 + 1
}

// A per-sequence length outside [0, length] (tile_info clamped it) sets the index bit; one
// thread per tile, after the tile's work.
__device__ __forceinline__ void flag_bad_length(const AttendArgs &a, int s) {
  if (!a.seq_len) return;
  const int64_t raw = a.seq_len[s];
  if (raw < 0 || raw > a.length) atomicOr(&a.hdr->err, kErrIndex);
}

// Candidate count of the top level; *forced_pos = position of the forced partial node or -1.
__device__ __forceinline__ int top_candidates(const AttendArgs &a, const Geo &geo, const TileInfo &t,
                                              int *forced_pos) {
  *forced_pos = -1;
  if (t.T == 0) return t.p;
  if (!a.causal) return a.seq_len ? nodes_at(t.p, geo.span[t.T]) : geo.nlen[t.T];
  const int full = t.p / geo.span[t.T];
  if (t.p - full * geo.span[t.T]) {
    *forced_pos = full;
    return full + 1;
  }
  return full;
}

struct LevelRows {
  const uint16_t *k, *v;
  int64_t nrows;
  const int32_t *pages;  // level 0 of a paged cache: the sequence's page table (else NULL)
};

// Row of candidate `node` (node < nrows) relative to k / v: the node itself, or through the
// page table at level 0 of a paged cache (pages are Hkv * page_size rows apart); -1 for a
// page outside the pool.
template <bool kPaged>
__device__ __forceinline__ int64_t row_at(const AttendArgs &a, const LevelRows &lr, int64_t node) {
  if (!kPaged || !lr.pages) return node;
  const int pg = __ldg(lr.pages + (node >> a.page_shift));
  if ((unsigned)pg >= (unsigned)a.num_pages) return -1;
  return ((int64_t)pg * a.hkv << a.page_shift) + (node & ((int64_t(1) << a.page_shift) - 1));
}

template <bool kPaged>
__device__ __forceinline__ LevelRows level_rows(const AttendArgs &a, const Geo &geo, int lvl, int64_t bh) {
  LevelRows r;
  r.pages = nullptr;
  if (kPaged && lvl == 0) {  // head h's rows of page 0; pages are Hkv * page_size rows apart
    const int64_t h = bh % a.hkv;
    r.k = a.k_tok + (h << a.page_shift) * kD;
    r.v = a.v_tok + (h << a.page_shift) * kD;
    r.nrows = a.cap;
    r.pages = a.page_table + (bh / a.hkv) * (a.cap >> a.page_shift);
  } else if (lvl == 0) {
    r.k = a.k_tok + bh * a.cap * kD;
    r.v = a.v_tok + bh * a.cap * kD;
    r.nrows = a.cap;
  } else {
    const int64_t o = (geo.row_off[lvl] + bh * geo.slots[lvl]) * kD;
    r.k = a.k_node + o;
    r.v = a.v_node + o;
    r.nrows = geo.slots[lvl];
  }
  return r;
}

// Children of an expanded candidate `v` at level lvl (in node order); *last_forced tells
// whether the last visible child is itself a partial node (causal mode only).
__device__ __forceinline__ int child_count(const AttendArgs &a, const Geo &geo, uint32_t v, int lvl, int p,
                                           bool *last_forced) {
  const int node = (int)(v & kNodeMask);
  *last_forced = false;
  if (!a.causal) {
    const int nlen = a.seq_len ? nodes_at(p, geo.span[lvl - 1]) : geo.nlen[lvl - 1];
    return max(0, min(a.b, nlen - node * a.b));
  }
  if (!(v & kForced)) return a.b;
  const int sb = geo.span[lvl - 1];
  const int first = node * a.b;  // children starting before p are visible
  const int nch = max(0, min(a.b, (p - first * sb + sb - 1) / sb));
  if (nch > 0) *last_forced = (int64_t)(first + nch) * sb > p;
  return nch;
}

// ------------------------------------------------------------------ half-warp rows

struct Row8 {
  uint2 lo, hi;  // dims 4j..4j+3 and 64+4j..64+4j+3 (bf16)
};

__device__ __forceinline__ Row8 ldg_row8(const uint16_t *row, int j16) {
  Row8 r;
  r.lo = __ldg(reinterpret_cast<const uint2 *>(row + 4 * j16));
  r.hi = __ldg(reinterpret_cast<const uint2 *>(row + kHalf + 4 * j16));
  return r;
}

struct Trig4 {
  float4 a, b;  // frequencies (4j, 4j+1) and (4j+2, 4j+3): (cos, cos', sin, sin') each
};

__device__ __forceinline__ Trig4 ldg_trig4(const float2 *table, int pos, int j16) {
  const float4 *t = reinterpret_cast<const float4 *>(table + (int64_t)pos * kHalf + 4 * j16);
  Trig4 r;
  r.a = __ldg(t);
  r.b = __ldg(t + 1);
  return r;
}

// The same row and table reads as ldg_row8 / ldg_trig4, issued where they stand: the
// compiler keeps volatile asm in program order, so a level's rows go out before the
// previous level is folded instead of being sunk next to their first use.
__device__ __forceinline__ uint2 ld_nc_u2(const void *p) {
  uint2 r;
  asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}
__device__ __forceinline__ float4 ld_nc_f4(const void *p) {
  float4 r;
  asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w) : "l"(p));
  return r;
}
__device__ __forceinline__ Row8 ld_row8_now(const uint16_t *row, int j16) {
  Row8 r;
  r.lo = ld_nc_u2(row + 4 * j16);
  r.hi = ld_nc_u2(row + kHalf + 4 * j16);
  return r;
}
__device__ __forceinline__ Trig4 ld_trig4_now(const float2 *table, int pos, int j16) {
  const float4 *t = reinterpret_cast<const float4 *>(table + (int64_t)pos * kHalf + 4 * j16);
  Trig4 r;
  r.a = ld_nc_f4(t);
  r.b = ld_nc_f4(t + 1);
  return r;
}

__device__ __forceinline__ void unpack_row8(const Row8 &r, float (&lo)[4], float (&hi)[4]) {
  lo[0] = bf16_lo(r.lo.x);
  lo[1] = bf16_hi(r.lo.x);
  lo[2] = bf16_lo(r.lo.y);
  lo[3] = bf16_hi(r.lo.y);
  hi[0] = bf16_lo(r.hi.x);
  hi[1] = bf16_hi(r.hi.x);
  hi[2] = bf16_lo(r.hi.y);
  hi[3] = bf16_hi(r.hi.y);
}

// rotate-half RoPE of the 4 pairs (lo[t], hi[t]): lo' = lo c - hi s, hi' = hi c + lo s
__device__ __forceinline__ void rotate4(float (&lo)[4], float (&hi)[4], const Trig4 &tr) {
  const float c[4] = {tr.a.x, tr.a.y, tr.b.x, tr.b.y};
  const float s[4] = {tr.a.z, tr.a.w, tr.b.z, tr.b.w};
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const float l = lo[t], h = hi[t];
    lo[t] = l * c[t] - h * s[t];
    hi[t] = h * c[t] + l * s[t];
  }
}

template <int G>
__device__ __forceinline__ void rotated_query(const float *qraw, const Trig4 &tq, int j16, float (&qlo)[G][4],
                                              float (&qhi)[G][4]) {
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float4 l4 = *reinterpret_cast<const float4 *>(qraw + h * kD + 4 * j16);
    const float4 h4 = *reinterpret_cast<const float4 *>(qraw + h * kD + kHalf + 4 * j16);
    qlo[h][0] = l4.x;
    qlo[h][1] = l4.y;
    qlo[h][2] = l4.z;
    qlo[h][3] = l4.w;
    qhi[h][0] = h4.x;
    qhi[h][1] = h4.y;
    qhi[h][2] = h4.z;
    qhi[h][3] = h4.w;
    rotate4(qlo[h], qhi[h], tq);
  }
}

// Partial dot products of the rotated key row with the G rotated query heads
// (packed fp32 pairs: q2lo[h][u] = (qlo[h][2u], qlo[h][2u+1]), likewise q2hi).
template <int G>
__device__ __forceinline__ void dot_row8(const Row8 &k, const Trig4 &tr, const float2 (&q2lo)[G][2],
                                         const float2 (&q2hi)[G][2], float (&part)[G]) {
  // the key's RoPE pairs rotated two at a time (packed fp32): lo' = lo c - hi s,
  // hi' = hi c + lo s, with (c, c') and (s, s') straight from the table
  const float2 k01 = make_float2(bf16_lo(k.lo.x), bf16_hi(k.lo.x)), k23 = make_float2(bf16_lo(k.lo.y), bf16_hi(k.lo.y));
  const float2 g01 = make_float2(bf16_lo(k.hi.x), bf16_hi(k.hi.x)), g23 = make_float2(bf16_lo(k.hi.y), bf16_hi(k.hi.y));
  const float2 c01 = make_float2(tr.a.x, tr.a.y), s01 = make_float2(tr.a.z, tr.a.w);
  const float2 c23 = make_float2(tr.b.x, tr.b.y), s23 = make_float2(tr.b.z, tr.b.w);
  const float2 l01 = __ffma2_rn(k01, c01, __fmul2_rn(g01, make_float2(-s01.x, -s01.y)));
  const float2 l23 = __ffma2_rn(k23, c23, __fmul2_rn(g23, make_float2(-s23.x, -s23.y)));
  const float2 h01 = __ffma2_rn(g01, c01, __fmul2_rn(k01, s01));
  const float2 h23 = __ffma2_rn(g23, c23, __fmul2_rn(k23, s23));
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float2 x = __fmul2_rn(q2lo[h][0], l01);
    x = __ffma2_rn(q2lo[h][1], l23, x);
    x = __ffma2_rn(q2hi[h][0], h01, x);
    x = __ffma2_rn(q2hi[h][1], h23, x);
    part[h] = x.x + x.y;
  }
}

template <int G>
__device__ __forceinline__ void pack_query(const float (&qlo)[G][4], const float (&qhi)[G][4], float2 (&q2lo)[G][2],
                                           float2 (&q2hi)[G][2]) {
#pragma unroll
  for (int h = 0; h < G; ++h) {
    q2lo[h][0] = make_float2(qlo[h][0], qlo[h][1]);
    q2lo[h][1] = make_float2(qlo[h][2], qlo[h][3]);
    q2hi[h][0] = make_float2(qhi[h][0], qhi[h][1]);
    q2hi[h][1] = make_float2(qhi[h][2], qhi[h][3]);
  }
}

// Sum the G partials over the 16 lanes of a half-warp; afterwards lane j holds the
// full dot product of head (j >> (4 - log2 G)).
template <int G>
__device__ __forceinline__ float reduce16(const float (&v)[G], int j16) {
  constexpr unsigned F = 0xffffffffu;
  if constexpr (G == 1) {
    float x = v[0];
    x += __shfl_xor_sync(F, x, 8);
    x += __shfl_xor_sync(F, x, 4);
    x += __shfl_xor_sync(F, x, 2);
    x += __shfl_xor_sync(F, x, 1);
    return x;
  } else if constexpr (G == 2) {
    const bool b3 = j16 & 8;
    float x = (b3 ? v[1] : v[0]) + __shfl_xor_sync(F, b3 ? v[0] : v[1], 8);
    x += __shfl_xor_sync(F, x, 4);
    x += __shfl_xor_sync(F, x, 2);
    x += __shfl_xor_sync(F, x, 1);
    return x;
  } else if constexpr (G == 4) {
    const bool b3 = j16 & 8, b2 = j16 & 4;
    const float k0 = (b3 ? v[2] : v[0]) + __shfl_xor_sync(F, b3 ? v[0] : v[2], 8);
    const float k1 = (b3 ? v[3] : v[1]) + __shfl_xor_sync(F, b3 ? v[1] : v[3], 8);
    float x = (b2 ? k1 : k0) + __shfl_xor_sync(F, b2 ? k0 : k1, 4);
    x += __shfl_xor_sync(F, x, 2);
    x += __shfl_xor_sync(F, x, 1);
    return x;
  } else {
    static_assert(G == 8, "G must be 1, 2, 4 or 8");
    const bool b3 = j16 & 8, b2 = j16 & 4, b1 = j16 & 2;
    float k[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) k[i] = (b3 ? v[i + 4] : v[i]) + __shfl_xor_sync(F, b3 ? v[i] : v[i + 4], 8);
    const float m0 = (b2 ? k[2] : k[0]) + __shfl_xor_sync(F, b2 ? k[0] : k[2], 4);
    const float m1 = (b2 ? k[3] : k[1]) + __shfl_xor_sync(F, b2 ? k[1] : k[3], 4);
    float x = (b1 ? m1 : m0) + __shfl_xor_sync(F, b1 ? m0 : m1, 2);
    x += __shfl_xor_sync(F, x, 1);
    return x;
  }
}

// Sum over the heads after reduce16: the group score S of the row.
template <int G>
__device__ __forceinline__ float group_sum16(float x) {
  if constexpr (G >= 2) x += __shfl_xor_sync(0xffffffffu, x, 8);
  if constexpr (G >= 4) x += __shfl_xor_sync(0xffffffffu, x, 4);
  if constexpr (G >= 8) x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

template <int G>
__device__ __forceinline__ bool head_writer(int j16) {
  return (j16 & ((1 << (4 - log2g<G>())) - 1)) == 0;
}
template <int G>
__device__ __forceinline__ int head_of(int j16) {
  return j16 >> (4 - log2g<G>());
}

// ------------------------------------------------------------------ warp-level selection

// Mark (kKept) the top-k scorable candidates of cl[0..n) by (S desc, position asc); the
// candidate order is node order, so position breaks ties toward the lower node index.
__device__ void warp_topk(uint32_t *cl, const uint32_t *skey, int n, int k, int lane) {
  int m = 0;
  for (int c = lane; c < n; c += 32) m += (cl[c] & kForced) ? 0 : 1;
  m = warp_sum_int(m);
  if (k >= m) {
    for (int c = lane; c < n; c += 32)
      if (!(cl[c] & kForced)) cl[c] |= kKept;
  } else if (k > 0 && k <= 32 && n <= 32 * kTopkRegs) {
    uint32_t key[kTopkRegs];  // order keys of scorable candidates are >= 0x007fffff; 0 = not selectable
#pragma unroll
    for (int t = 0; t < kTopkRegs; ++t) {
      const int c = lane + 32 * t;
      key[t] = (c < n && !(cl[c] & kForced)) ? skey[c] : 0u;
    }
    for (int r = 0; r < k; ++r) {
      uint32_t best = 0u;
      int bi = 0x7fffffff;
#pragma unroll
      for (int t = 0; t < kTopkRegs; ++t)
        if (key[t] > best) {
          best = key[t];
          bi = lane + 32 * t;
        }
      const uint32_t mx = __reduce_max_sync(0xffffffffu, best);
      const int win = __reduce_min_sync(0xffffffffu, best == mx ? bi : 0x7fffffff);
#pragma unroll
      for (int t = 0; t < kTopkRegs; ++t)
        if (lane + 32 * t == win) key[t] = 0u;
      if (lane == (win & 31)) cl[win] |= kKept;
    }
  } else if (k > 0) {
    // rank: a candidate is kept when fewer than k scorable candidates beat it
    for (int c = lane; c < n; c += 32) {
      const uint32_t v = cl[c];
      if (v & kForced) continue;
      const uint32_t kc = skey[c];
      int better = 0;
      for (int e = 0; e < n; ++e) {
        if (cl[e] & kForced) continue;
        const uint32_t ke = skey[e];
        better += (ke > kc || (ke == kc && e < c)) ? 1 : 0;
      }
      if (better < k) cl[c] = v | kKept;
    }
  }
  __syncwarp();
}

// Kept node indices of this level, ascending, -1 padded (diagnostics).
__device__ void warp_write_selection(const AttendArgs &a, const uint32_t *cl, int n, int lvl, int tile, int lane) {
  if (a.sel_idx == nullptr || lvl > a.sel_levels) return;
  int32_t *dst = a.sel_idx + ((int64_t)tile * a.sel_levels + (lvl - 1)) * a.top_k;
  int cnt = 0;
  for (int base = 0; base < n; base += 32) {
    const int c = base + lane;
    const bool kept = c < n && (cl[c] & kKept);
    const unsigned bal = __ballot_sync(0xffffffffu, kept);
    if (kept) {
      const int r = cnt + __popc(bal & ((1u << lane) - 1u));
      if (r < a.top_k) dst[r] = (int32_t)(cl[c] & kNodeMask);
    }
    cnt += __popc(bal);
  }
  for (int t = cnt + lane; t < a.top_k; t += 32) dst[t] = -1;
}

// Next level's candidates: the children of the kept and forced candidates, in order.
__device__ int warp_expand(const AttendArgs &a, const Geo &geo, const uint32_t *cl, int n, int lvl, int p,
                           uint32_t *nx, int lane, uint32_t *err) {
  int total = 0;
  for (int base = 0; base < n; base += 32) {
    const int c = base + lane;
    const uint32_t v = c < n ? cl[c] : 0u;
    bool lf = false;
    const int nch = (c < n && (v & (kKept | kForced))) ? child_count(a, geo, v, lvl, p, &lf) : 0;
    int x = nch;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    const int off = total + x - nch;
    const int64_t first = (int64_t)(v & kNodeMask) * a.b;
    for (int t = 0; t < nch; ++t) {
      if (off + t >= a.max_cand) {
        atomicOr(err, kErrCount);
        break;
      }
      nx[off + t] = (uint32_t)(first + t) | ((lf && t == nch - 1) ? kForced : 0u);
    }
    total += __shfl_sync(0xffffffffu, x, 31);
  }
  __syncwarp();
  return min(total, a.max_cand);
}

__device__ __forceinline__ bool workspace_ok(const AttendArgs &a) {
  const volatile WsHeader *h = a.hdr;
  return h->magic == kWsMagic && h->table_rows >= a.table_rows_needed;
}

__device__ __forceinline__ void store_out4(const AttendArgs &a, int64_t at, float y0, float y1, float y2, float y3) {
  if (a.out_fp32) {
    *reinterpret_cast<float4 *>(reinterpret_cast<float *>(a.out) + at) = make_float4(y0, y1, y2, y3);
  } else {
    uint2 u;
    u.x = pack_bf16x2(y0, y1);
    u.y = pack_bf16x2(y2, y3);
    *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(a.out) + at) = u;
  }
}

// ================================================================== CTA / cluster kernel

struct CtaLayout {
  int misc, geo, q, cand, skey, rank, slog, ownk, fkey, fpos, kflag, red, clm, fin_cap, total;
};

// Finalists per level (two-stage selection): every CTA publishes the top k of each group
// of 32 of its own rows; used while top_k <= 32.
__host__ __device__ inline int finalist_cap(int CS, int own_max, int top_k) {
  return (top_k >= 1 && top_k <= 32) ? CS * ((own_max + 31) / 32) * top_k : 0;
}

__host__ __device__ inline int align128(int x) { return (x + 127) & ~127; }

__host__ __device__ inline CtaLayout cta_layout(int G, int CS, int max_cand, int own_max, int top_k) {
  CtaLayout L;
  int o = 0;
  auto take = [&o](int bytes) {
    const int r = o;
    o = align128(o + bytes);
    return r;
  };
  L.misc = take(kMiscInts * 4);
  L.geo = take(kGeoBytes);
  L.q = take(G * kD * 4);
  L.cand = take(2 * max_cand * 4);
  L.skey = take((CS > 1 ? 2 : 1) * max_cand * 4);
  L.rank = take(max_cand * 4);
  L.slog = take(2 * G * own_max * 4);  // by level parity: the next level scores while this one folds
  L.fin_cap = finalist_cap(CS, own_max, top_k);
  L.ownk = L.fin_cap ? take(own_max * 4) : 0;  // own keys: only the finalist path reads them
  L.fkey = take(2 * L.fin_cap * 4);  // by level parity: peers publish the next level's while this one reads
  L.fpos = take(2 * L.fin_cap * 4);
  L.kflag = take(L.fin_cap * 4 + 4);
  L.red = take(kCtaWarps * G * kRedStride * 4);
  L.clm = CS > 1 ? take(CS * G * kRedStride * 4) : 0;
  L.total = o;
  return L;
}

// Rows a half-warp gathers in one pass of the CTA kernel.
template <int RPH>
struct RowSet {
  Row8 k[RPH], v[RPH];
  Trig4 tr[RPH];
  int pos[RPH];
  bool ok[RPH];
};

__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// kTwoPerSm: the instance for more tiles than SMs (one CTA a tile): two CTAs share an SM
// (128 registers a thread), with fewer rows in flight and no gather of the next level ahead;
// a tile takes longer (1M, one wave: 66 against 52 us) but two run at once (512 tiles: 141
// against 179 us).
template <int G, int CS, bool kPaged = false, bool kTwoPerSm = false>
__global__ void __launch_bounds__(kCtaThreads, kTwoPerSm ? 2 : 1) attend_cta_kernel(const AttendArgs a) {
  static_assert(!kTwoPerSm || CS == 1, "two CTAs per SM only for a CTA per tile");
  constexpr int RPH = (CS == 4 || G == 8 || kTwoPerSm) ? 2 : 4;  // rows per half-warp per pass (register budget)
  constexpr int PASS = kHalfWarps * RPH;                           // rows per CTA per pass
  constexpr bool PIPE = RPH == 2 && !kTwoPerSm;  // gather the next level before folding this one
  extern __shared__ __align__(128) unsigned char smem[];
  const CtaLayout Ls = cta_layout(G, CS, a.max_cand, a.own_max, a.top_k);
  int *misc = reinterpret_cast<int *>(smem + Ls.misc);  // see kMiscInts
  Geo *geo_s = reinterpret_cast<Geo *>(smem + Ls.geo);
  load_geo(a, geo_s, threadIdx.x, kCtaThreads);
  __syncthreads();
  const Geo &geo = *geo_s;
  float *qraw = reinterpret_cast<float *>(smem + Ls.q);
  uint32_t *cand = reinterpret_cast<uint32_t *>(smem + Ls.cand);
  uint32_t *skey_all = reinterpret_cast<uint32_t *>(smem + Ls.skey);
  int *rank = reinterpret_cast<int *>(smem + Ls.rank);
  float *slog_all = reinterpret_cast<float *>(smem + Ls.slog);
  uint32_t *own_key = reinterpret_cast<uint32_t *>(smem + Ls.ownk);
  uint32_t *fkey_all = reinterpret_cast<uint32_t *>(smem + Ls.fkey);
  int *fpos_all = reinterpret_cast<int *>(smem + Ls.fpos);
  int *kflag = reinterpret_cast<int *>(smem + Ls.kflag);
  const int OWN = a.own_max, MC = a.max_cand, FCAP = Ls.fin_cap;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j16 = lane & 15, hw = warp * 2 + (lane >> 4);  // half-warp id 0..15
  int crank = 0;
  if constexpr (CS > 1) crank = (int)cg::this_cluster().block_rank();
  const int tile = blockIdx.x / CS;
  const TileInfo t = tile_info(a, geo, tile);
  uint32_t *err = &a.hdr->err;
  const int64_t out0 = (((int64_t)t.s * a.nq + t.qi) * a.hq + (int64_t)t.g * G) * kD;

  // workspace header: read now, checked before the output is written
  uint32_t hdr_magic = kWsMagic;
  int hdr_rows = a.table_rows_needed;
  if (tid == 0) {
    const volatile WsHeader *h = a.hdr;
    hdr_magic = h->magic;
    hdr_rows = h->table_rows;
  }
  // query rows of the group (q and out share the [B][Q][Hq][128] layout)
  uint2 qreg = make_uint2(0u, 0u);
  if (tid < G * kD / 4) qreg = __ldg(reinterpret_cast<const uint2 *>(a.q + out0) + tid);

  int fpos;
  int n = top_candidates(a, geo, t, &fpos);
  if (n > a.table_rows_needed - 1) {  // cannot happen for a valid launch; guards the table reads
    if (tid == 0) atomicOr(err, kErrCount);
    n = a.table_rows_needed - 1;
  }

  // Gather rows [pass0, pass0 + PASS) of this CTA's slice [.., hi_r) of level lvl.  cl == nullptr
  // means the top level, whose position i is node i.
  auto gather = [&](RowSet<RPH> &rs, int lvl, const uint32_t *cl, int pass0, int hi_r, bool values) {
    const LevelRows lr = level_rows<kPaged>(a, geo, lvl, t.bh);
#pragma unroll
    for (int r = 0; r < RPH; ++r) {
      const int i = pass0 + hw + kHalfWarps * r;
      rs.pos[r] = i;
      const uint32_t c = i < hi_r ? (cl ? cl[i] : ((uint32_t)i | (i == fpos ? kForced : 0u))) : kForced;
      const int64_t node = c & kNodeMask;
      const bool want = i < hi_r && !(c & kForced);
      const int64_t row = want && node < lr.nrows ? row_at<kPaged>(a, lr, node) : -1;
      rs.ok[r] = row >= 0;
      if (want && row < 0 && j16 == 0) atomicOr(err, kErrIndex);
      if (rs.ok[r]) {
        rs.k[r] = ldg_row8(lr.k + row * kD, j16);
        rs.tr[r] = ldg_trig4(a.table, i, j16);
        if (values) rs.v[r] = ldg_row8(lr.v + row * kD, j16);
      }
    }
  };

  float m_w[G], l_w[G];
  float2 acc[G][4];  // dims (4j, 4j+1), (4j+2, 4j+3), (64+4j, ..), (64+4j+2, ..)
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m_w[h] = -INFINITY;
    l_w[h] = 0.f;
#pragma unroll
    for (int d = 0; d < 4; ++d) acc[h][d] = make_float2(0.f, 0.f);
  }

  // Fold the entry rows of a row set (values in registers) into the warp's state.
  auto fold = [&](const RowSet<RPH> &rs, const bool (&ent)[RPH], const float *slog, int lo_r) {
    float mx[G];
#pragma unroll
    for (int h = 0; h < G; ++h) mx[h] = -INFINITY;
#pragma unroll
    for (int r = 0; r < RPH; ++r)
      if (ent[r]) {
#pragma unroll
        for (int h = 0; h < G; ++h) mx[h] = fmaxf(mx[h], slog[h * OWN + rs.pos[r] - lo_r]);
      }
    float mnew[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 16));
      mnew[h] = fmaxf(m_w[h], mx[h]);
      const float alpha = (mnew[h] == -INFINITY) ? 1.f : __expf(m_w[h] - mnew[h]);
      m_w[h] = mnew[h];
      l_w[h] *= alpha;
      const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
      for (int d = 0; d < 4; ++d) acc[h][d] = __fmul2_rn(acc[h][d], a2);
    }
    float ls[G];
#pragma unroll
    for (int h = 0; h < G; ++h) ls[h] = 0.f;
#pragma unroll
    for (int r = 0; r < RPH; ++r)
      if (ent[r]) {
        const Row8 &v = rs.v[r];
        const float2 v0 = make_float2(bf16_lo(v.lo.x), bf16_hi(v.lo.x)), v1 = make_float2(bf16_lo(v.lo.y), bf16_hi(v.lo.y));
        const float2 v2 = make_float2(bf16_lo(v.hi.x), bf16_hi(v.hi.x)), v3 = make_float2(bf16_lo(v.hi.y), bf16_hi(v.hi.y));
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float pr = __expf(slog[h * OWN + rs.pos[r] - lo_r] - mnew[h]);
          ls[h] += pr;
          const float2 p2 = make_float2(pr, pr);
          acc[h][0] = __ffma2_rn(p2, v0, acc[h][0]);
          acc[h][1] = __ffma2_rn(p2, v1, acc[h][1]);
          acc[h][2] = __ffma2_rn(p2, v2, acc[h][2]);
          acc[h][3] = __ffma2_rn(p2, v3, acc[h][3]);
        }
      }
#pragma unroll
    for (int h = 0; h < G; ++h) l_w[h] += ls[h] + __shfl_xor_sync(0xffffffffu, ls[h], 16);
  };

  // the top level's rows go out before anything waits on memory
  int per = (n + CS - 1) / CS;
  int lo_r = min(n, crank * per), hi_r = min(n, lo_r + per);
  RowSet<RPH> cur_rs, nxt_rs;
  bool preloaded = false;
  Trig4 tq_pre;
  if (hi_r - lo_r <= PASS) {
    gather(cur_rs, t.T, nullptr, lo_r, hi_r, true);
    tq_pre = ldg_trig4(a.table, n, j16);
    preloaded = true;
  }
  if (tid < G * kD / 4)
    *reinterpret_cast<float4 *>(qraw + 4 * tid) =
        make_float4(bf16_lo(qreg.x), bf16_hi(qreg.x), bf16_lo(qreg.y), bf16_hi(qreg.y));
  for (int i = tid; i < n; i += kCtaThreads) {
    cand[i] = (uint32_t)i | (i == fpos ? kForced : 0u);
    rank[i] = 0;
  }
  for (int i = tid; i < 2 * FCAP; i += kCtaThreads) fpos_all[i] = -1;
  if (tid == 0) misc[1] = (hdr_magic != kWsMagic || hdr_rows < a.table_rows_needed) ? 1 : 0;
  __syncthreads();
  if constexpr (CS > 1) cluster_barrier();  // every peer runs before the first DSMEM store

  int cur = 0, keys_read = 0, values_read = 0;
  for (int lvl = t.T; lvl >= 0; --lvl) {
    uint32_t *cl = cand + cur * MC;
    uint32_t *sk = skey_all + ((CS > 1) ? (lvl & 1) * MC : 0);
    float *slog = slog_all + (lvl & 1) * G * OWN;
    const bool single = hi_r - lo_r <= PASS;
    const LevelRows lr = level_rows<kPaged>(a, geo, lvl, t.bh);

    const int nforced = (a.causal && n > 0 && (cl[n - 1] & kForced)) ? 1 : 0;
    const int m = n - nforced;
    // two-stage selection: each CTA ranks its own rows within groups of 32 and publishes
    // the top k of each group as finalists; then every CTA ranks the finalists
    const int groups = (per + 31) / 32;  // groups per CTA (the same in every CTA)
    const int nfin = CS * groups * a.top_k;
    const bool fast = lvl > 0 && single && a.top_k >= 1 && a.top_k < m && nfin <= FCAP && nfin <= kCtaThreads;

    // 1. score this CTA's slice (rows preloaded, or gathered now)
    const Trig4 tq = preloaded ? tq_pre : ldg_trig4(a.table, n, j16);
    if (single && !preloaded) gather(cur_rs, lvl, cl, lo_r, hi_r, true);
    float2 q2lo[G][2], q2hi[G][2];
    {
      float qlo[G][4], qhi[G][4];
      rotated_query<G>(qraw, tq, j16, qlo, qhi);
      pack_query<G>(qlo, qhi, q2lo, q2hi);
    }
    auto score = [&](const RowSet<RPH> &rs) {
#pragma unroll
      for (int r = 0; r < RPH; ++r) {
        float part[G];
#pragma unroll
        for (int h = 0; h < G; ++h) part[h] = 0.f;
        if (rs.ok[r]) dot_row8<G>(rs.k[r], rs.tr[r], q2lo, q2hi, part);
        const float x = reduce16<G>(part, j16) * a.scale;
        const float S = group_sum16<G>(x);
        if (fast) {
          if (j16 == 0 && rs.pos[r] < hi_r) own_key[rs.pos[r] - lo_r] = rs.ok[r] ? order_key(S) : 0u;
          if (rs.ok[r] && head_writer<G>(j16)) slog[head_of<G>(j16) * OWN + rs.pos[r] - lo_r] = x;
        } else if (rs.ok[r]) {
          if (head_writer<G>(j16)) slog[head_of<G>(j16) * OWN + rs.pos[r] - lo_r] = x;
          if (lvl > 0 && j16 == 0) {
            const uint32_t key = order_key(S);
            if constexpr (CS > 1) {
              cg::cluster_group cluster = cg::this_cluster();
#pragma unroll
              for (int q = 0; q < CS; ++q) cluster.map_shared_rank(sk, q)[rs.pos[r]] = key;
            } else {
              sk[rs.pos[r]] = key;
            }
          }
        }
      }
    };
    if (single) {
      score(cur_rs);
    } else {
      for (int pass0 = lo_r; pass0 < hi_r; pass0 += PASS) {
        RowSet<RPH> rs;
        gather(rs, lvl, cl, pass0, hi_r, false);
        score(rs);
      }
    }
    preloaded = false;
    // the next count slot of this level's parity was last read two levels ago
    int *next_count = misc + kNextCount + (lvl & 1);
    if (tid == 0) *next_count = 0;
    keys_read += m;
    uint32_t *fkey = fkey_all + (lvl & 1) * FCAP;
    int *fpos = fpos_all + (lvl & 1) * FCAP;
    {  // the next level's finalist slots (read last two levels ago) start empty
      int *fnext = fpos_all + ((lvl - 1) & 1) * FCAP;
      for (int i = tid; i < FCAP; i += kCtaThreads) fnext[i] = -1;
    }
    if (fast) {
      __syncthreads();  // own keys
      const int own = hi_r - lo_r;
      const int tpi = min(32, 1 << (31 - __clz(kCtaThreads / max(own, 1))));  // lanes per item
      const int item = tid / tpi, q = tid - item * tpi;
      const uint32_t kc = item < own ? own_key[item] : 0u;
      const int g0 = item & ~31, gcnt = min(32, own - g0);
      int better = 0;
      if (item < own)
        for (int j = q; j < gcnt; j += tpi) {
          const uint32_t kj = own_key[g0 + j];
          better += (kj > kc || (kj == kc && g0 + j < item)) ? 1 : 0;
        }
      for (int o = 1; o < tpi; o <<= 1) better += __shfl_xor_sync(0xffffffffu, better, o);
      if (q == 0 && item < own && kc != 0u && better < a.top_k) {
        const int slot = (crank * groups + (item >> 5)) * a.top_k + better;
        if constexpr (CS > 1) {
          cg::cluster_group cluster = cg::this_cluster();
#pragma unroll
          for (int r = 0; r < CS; ++r) {
            cluster.map_shared_rank(fkey, r)[slot] = kc;
            cluster.map_shared_rank(fpos, r)[slot] = lo_r + item;
          }
        } else {
          fkey[slot] = kc;
          fpos[slot] = lo_r + item;
        }
      }
    }
    if constexpr (CS > 1) {
      cluster_barrier();  // also orders this CTA's shared memory (release/acquire)
    } else {
      __syncthreads();
    }

    int n_next = 0;
    if (fast) {
      // 2'. rank the finalists; the kept ones, in node order, expand into the next list
      const int tpi = min(32, 1 << (31 - __clz(kCtaThreads / nfin)));
      const int f = tid / tpi, q = tid - f * tpi;
      const int pf = f < nfin ? fpos[f] : -1;
      const uint32_t kf = f < nfin ? fkey[f] : 0u;
      int better = 0;
      if (pf >= 0)
        for (int j = q; j < nfin; j += tpi) {
          const int pj = fpos[j];
          const uint32_t kj = fkey[j];
          better += (pj >= 0 && (kj > kf || (kj == kf && pj < pf))) ? 1 : 0;
        }
      for (int o = 1; o < tpi; o <<= 1) better += __shfl_xor_sync(0xffffffffu, better, o);
      const bool kept = pf >= 0 && better < a.top_k;
      if (q == 0 && f < nfin) kflag[f] = kept ? 1 : 0;
      const int nkept = __syncthreads_count(q == 0 && kept);
      int32_t *sel = (a.sel_idx != nullptr && crank == 0 && lvl <= a.sel_levels)
                         ? a.sel_idx + ((int64_t)tile * a.sel_levels + (lvl - 1)) * a.top_k
                         : nullptr;
      if (sel)
        for (int u = nkept + tid; u < a.top_k; u += kCtaThreads) sel[u] = -1;
      uint32_t *nx = cand + (cur ^ 1) * MC;
      const LevelRows lb = level_rows<kPaged>(a, geo, lvl - 1, t.bh);
      auto expand_one = [&](uint32_t v, int e) {  // children of the e-th expanded node
        bool lf = false;
        const int nch = child_count(a, geo, v, lvl, t.p, &lf);
        const int off = e * a.b;
        const int first = (int)(v & kNodeMask) * a.b;
        for (int u = 0; u < nch && off + u < MC; ++u)
          nx[off + u] = (uint32_t)(first + u) | ((lf && u == nch - 1) ? kForced : 0u);
        if (off + nch > MC) atomicOr(err, kErrCount);
        atomicMax(next_count, min(off + nch, MC));
        if (nch > 0 && e % CS == crank && first + nch <= lb.nrows && !(kPaged && lb.pages)) {
          prefetch_l2(lb.k + (int64_t)first * kD, (uint32_t)nch * kRowBytes);
          prefetch_l2(lb.v + (int64_t)first * kD, (uint32_t)nch * kRowBytes);
        }
      };
      int e = 0;
      if (kept)
        for (int j = q; j < nfin; j += tpi) e += (kflag[j] && fpos[j] < pf) ? 1 : 0;
      for (int o = 1; o < tpi; o <<= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
      if (kept && q == 0) {
        const uint32_t v = cl[pf];
        cl[pf] = v | kKept;
        if (sel) sel[e] = (int32_t)(v & kNodeMask);
        expand_one(v, e);
      }
      if (nforced && tid == kCtaThreads - 1) expand_one(cl[n - 1], nkept);
      values_read += m - a.top_k;
      __syncthreads();
      n_next = min(*next_count, MC);
      if (n_next > a.table_rows_needed - 1) {
        if (tid == 0) atomicOr(err, kErrCount);
        n_next = a.table_rows_needed - 1;
      }
      for (int i = tid; i < n_next; i += kCtaThreads) rank[i] = 0;
    } else if (lvl > 0) {
      // 2. top-k by rank: a candidate is kept when fewer than k scorable candidates beat it
      const bool keep_all = a.top_k >= m;
      if (!keep_all && a.top_k > 0) {
        // items (candidate c, 64-wide segment of competitors); the forced candidate, if
        // any, is the last one and competes with nobody (c < m)
        const int nseg = (m + 63) / 64;
        for (int it = tid; it < m * nseg; it += kCtaThreads) {
          const int seg = it / m, c = it - seg * m;
          const uint32_t kc = sk[c];
          const int e0 = seg * 64, e1 = min(m, e0 + 64);
          const int mid = max(e0, min(c, e1));  // competitors below c win ties
          int better = 0;
          int e = e0;
          for (; e + 4 <= mid; e += 4) {
            const uint4 k4 = *reinterpret_cast<const uint4 *>(sk + e);
            better += (k4.x >= kc) + (k4.y >= kc) + (k4.z >= kc) + (k4.w >= kc);
          }
          for (; e < mid; ++e) better += sk[e] >= kc;
          if (e == c) ++e;
          for (; e < e1 && (e & 3); ++e) better += sk[e] > kc;
          for (; e + 4 <= e1; e += 4) {
            const uint4 k4 = *reinterpret_cast<const uint4 *>(sk + e);
            better += (k4.x > kc) + (k4.y > kc) + (k4.z > kc) + (k4.w > kc);
          }
          for (; e < e1; ++e) better += sk[e] > kc;
          if (better) atomicAdd(&rank[c], better);
        }
        __syncthreads();
      }
      values_read += m - min(a.top_k, m);
      // 3. kept flags and the next candidate list.  Expanded candidates (kept, or forced)
      //    are in node order and all but the last have exactly b children, so the e-th
      //    expanded candidate's children start at position e * b.
      uint32_t *nx = cand + (cur ^ 1) * MC;
      const LevelRows lb = level_rows<kPaged>(a, geo, lvl - 1, t.bh);
      int carry_e = 0, carry_k = 0;
      int32_t *sel = (a.sel_idx != nullptr && crank == 0 && lvl <= a.sel_levels)
                         ? a.sel_idx + ((int64_t)tile * a.sel_levels + (lvl - 1)) * a.top_k
                         : nullptr;
      for (int base = 0; base < n; base += kCtaThreads) {
        const int c = base + tid;
        const uint32_t v = c < n ? cl[c] : 0u;
        const bool forced = c < n && (v & kForced);
        const bool kept = c < n && !forced && a.top_k > 0 && (keep_all || rank[c] < a.top_k);
        const bool ex = kept || forced;
        const unsigned be = __ballot_sync(0xffffffffu, ex), bk = __ballot_sync(0xffffffffu, kept);
        if (lane == 0) {
          misc[2 + warp] = __popc(be);
          misc[2 + kCtaWarps + warp] = __popc(bk);
        }
        __syncthreads();
        int pe = carry_e + __popc(be & ((1u << lane) - 1u)), pk = carry_k + __popc(bk & ((1u << lane) - 1u));
        int te = 0, tk = 0;
#pragma unroll
        for (int w = 0; w < kCtaWarps; ++w) {
          const int xe = misc[2 + w], xk = misc[2 + kCtaWarps + w];
          if (w < warp) {
            pe += xe;
            pk += xk;
          }
          te += xe;
          tk += xk;
        }
        if (kept) {
          cl[c] = v | kKept;
          if (sel && pk < a.top_k) sel[pk] = (int32_t)(v & kNodeMask);
        }
        if (ex) {
          bool lf = false;
          const int nch = child_count(a, geo, v, lvl, t.p, &lf);
          const int off = pe * a.b;
          const int64_t first = (int64_t)(v & kNodeMask) * a.b;
          for (int u = 0; u < nch; ++u) {
            if (off + u >= MC) {
              atomicOr(err, kErrCount);
              break;
            }
            nx[off + u] = (uint32_t)(first + u) | ((lf && u == nch - 1) ? kForced : 0u);
          }
          atomicMax(next_count, off + nch);
          // warm L2 with the rows the next level gathers (one CTA of the cluster per node)
          if (nch > 0 && pe % CS == crank && first + nch <= lb.nrows) {
            prefetch_l2(lb.k + first * kD, (uint32_t)nch * kRowBytes);
            prefetch_l2(lb.v + first * kD, (uint32_t)nch * kRowBytes);
          }
        }
        __syncthreads();
        carry_e += te;
        carry_k += tk;
      }
      if (sel)
        for (int u = carry_k + tid; u < a.top_k; u += kCtaThreads) sel[u] = -1;
      n_next = min(*next_count, MC);
      if (n_next > a.table_rows_needed - 1) {
        if (tid == 0) atomicOr(err, kErrCount);
        n_next = a.table_rows_needed - 1;
      }
      for (int i = tid; i < n_next; i += kCtaThreads) rank[i] = 0;  // for the next level's count
    } else {
      values_read += n;
    }

    // 4. next level's rows go out before this level's fold (the pipelined shape)
    const int per2 = (n_next + CS - 1) / CS;
    const int lo2 = min(n_next, crank * per2), hi2 = min(n_next, lo2 + per2);
    if (PIPE && lvl > 0 && hi2 - lo2 <= PASS) {
      gather(nxt_rs, lvl - 1, cand + (cur ^ 1) * MC, lo2, hi2, true);
      tq_pre = ldg_trig4(a.table, n_next, j16);
      preloaded = true;
    }
    // 5. fold this level's entries
    if (single) {
      bool ent[RPH];
#pragma unroll
      for (int r = 0; r < RPH; ++r) ent[r] = cur_rs.ok[r] && (lvl == 0 || !(cl[cur_rs.pos[r]] & kKept));
      fold(cur_rs, ent, slog, lo_r);
    } else {
      for (int pass0 = lo_r; pass0 < hi_r; pass0 += PASS) {
        RowSet<RPH> rs;
        bool ent[RPH];
#pragma unroll
        for (int r = 0; r < RPH; ++r) {
          const int i = pass0 + hw + kHalfWarps * r;
          rs.pos[r] = i;
          const uint32_t c = i < hi_r ? cl[i] : (kForced | kKept);
          const int64_t node = c & kNodeMask;
          const int64_t row = i < hi_r && !(c & (kForced | kKept)) && node < lr.nrows ? row_at<kPaged>(a, lr, node) : -1;
          ent[r] = row >= 0;
          rs.ok[r] = ent[r];
          if (ent[r]) rs.v[r] = ldg_row8(lr.v + row * kD, j16);
        }
        fold(rs, ent, slog, lo_r);
      }
    }
    if (lvl == 0) break;
    if (preloaded) {
#pragma unroll
      for (int r = 0; r < RPH; ++r) {
        cur_rs.k[r] = nxt_rs.k[r];
        cur_rs.v[r] = nxt_rs.v[r];
        cur_rs.tr[r] = nxt_rs.tr[r];
        cur_rs.pos[r] = nxt_rs.pos[r];
        cur_rs.ok[r] = nxt_rs.ok[r];
      }
    }
    n = n_next;
    per = per2;
    lo_r = lo2;
    hi_r = hi2;
    cur ^= 1;
  }

  if (crank == 0 && tid == 0) flag_bad_length(a, t.s);
  if (a.entries != nullptr && crank == 0 && tid == 0) {
    a.entries[2 * (int64_t)tile] = keys_read;
    a.entries[2 * (int64_t)tile + 1] = values_read;
  }

  // merge: half-warps -> warp -> CTA -> cluster
  float *red = reinterpret_cast<float *>(smem + Ls.red);  // [warp][h][kRedStride]: m, l, pad, acc[128]
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float2 x[4];
#pragma unroll
    for (int d = 0; d < 4; ++d) {
      x[d].x = acc[h][d].x + __shfl_xor_sync(0xffffffffu, acc[h][d].x, 16);
      x[d].y = acc[h][d].y + __shfl_xor_sync(0xffffffffu, acc[h][d].y, 16);
    }
    float *r = red + (warp * G + h) * kRedStride;
    if (lane == 0) {
      r[0] = m_w[h];
      r[1] = l_w[h];
    }
    if (lane < 16) {
      *reinterpret_cast<float4 *>(r + 4 + 4 * j16) = make_float4(x[0].x, x[0].y, x[1].x, x[1].y);
      *reinterpret_cast<float4 *>(r + 4 + kHalf + 4 * j16) = make_float4(x[2].x, x[2].y, x[3].x, x[3].y);
    }
  }
  __syncthreads();
  const bool ws_bad = misc[1] != 0;
  float *clm = reinterpret_cast<float *>(smem + Ls.clm);  // [rank][h][kRedStride] on cluster rank 0
  for (int e = tid; e < G * kD / 4; e += kCtaThreads) {
    const int h = (4 * e) / kD, d0 = (4 * e) % kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kCtaWarps; ++w) M = fmaxf(M, red[(w * G + h) * kRedStride]);
    float l = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kCtaWarps; ++w) {
        const float *r = red + (w * G + h) * kRedStride;
        const float f = (r[0] == -INFINITY) ? 0.f : __expf(r[0] - M);
        l += f * r[1];
#pragma unroll
        for (int d = 0; d < 4; ++d) o[d] += f * r[4 + d0 + d];
      }
    }
    if constexpr (CS == 1) {
      const float inv = (l > 0.f && !ws_bad) ? 1.f / l : 0.f;
      store_out4(a, out0 + 4 * e, o[0] * inv, o[1] * inv, o[2] * inv, o[3] * inv);
    } else {
      cg::cluster_group cluster = cg::this_cluster();
      float *dst = cluster.map_shared_rank(clm, 0) + (crank * G + h) * kRedStride;
      if (d0 == 0) {
        dst[0] = M;
        dst[1] = l;
      }
#pragma unroll
      for (int d = 0; d < 4; ++d) dst[4 + d0 + d] = o[d];
    }
  }
  if constexpr (CS > 1) {
    cluster_barrier();
    if (crank == 0) {
      for (int e = tid; e < G * kD / 4; e += kCtaThreads) {
        const int h = (4 * e) / kD, d0 = (4 * e) % kD;
        float M = -INFINITY;
#pragma unroll
        for (int r = 0; r < CS; ++r) M = fmaxf(M, clm[(r * G + h) * kRedStride]);
        float l = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
        if (M != -INFINITY) {
#pragma unroll
          for (int r = 0; r < CS; ++r) {
            const float *x = clm + (r * G + h) * kRedStride;
            const float f = (x[0] == -INFINITY) ? 0.f : __expf(x[0] - M);
            l += f * x[1];
#pragma unroll
            for (int d = 0; d < 4; ++d) o[d] += f * x[4 + d0 + d];
          }
        }
        const float inv = (l > 0.f && !ws_bad) ? 1.f / l : 0.f;
        store_out4(a, out0 + 4 * e, o[0] * inv, o[1] * inv, o[2] * inv, o[3] * inv);
      }
    }
  }
  if (ws_bad && tid == 0 && crank == 0) atomicOr(err, kErrWs);
}

// ================================================================== lean cluster kernel
//
// One cluster of CS CTAs per tile, one memory round trip, one cluster barrier and one
// block barrier per level.  Every CTA holds the rows of its slice of the level in
// registers; it scores them and stores each group score into every CTA of the cluster;
// after the cluster barrier each CTA ranks all n scores itself, so every CTA knows the
// kept set without a second exchange.  The next level's rows are addressed
// straight from the kept mask (child i of the level belongs to the (i / b)-th expanded
// node), issued, and only then is this level's unkept part folded.

constexpr int kLeanMaxCand = 256;  // candidates per level the lean kernel ranks (one bit each)

struct LeanLayout {
  int geo, kbuf, mask, par, red, clm, total;
};

__host__ __device__ inline LeanLayout lean_layout(int G, int CS, int max_cand) {
  LeanLayout L;
  int o = 0;
  auto take = [&o](int bytes) {
    const int r = o;
    o = align128(o + bytes);
    return r;
  };
  L.geo = take(kGeoBytes);
  L.kbuf = take(2 * kLeanMaxCand * 4);  // group scores (order keys) by level parity
  L.mask = take(2 * 16 * 2);            // kept bits, 16 per half-word, by level parity
  L.par = take(2 * max_cand * 4);       // expanded node ids of the level above, by parity
  L.red = take(kCtaWarps * G * kRedStride * 4);
  L.clm = take(CS * G * kRedStride * 4);
  L.total = o;
  return L;
}

// #{j in [j0, j1) : k[j] > thr}
__device__ __forceinline__ int count_above(const uint32_t *k, int j0, int j1, uint32_t thr) {
  int cnt = 0, j = j0;
  for (; j < j1 && (j & 3); ++j) cnt += k[j] > thr;
  for (; j + 4 <= j1; j += 4) {
    const uint4 v = *reinterpret_cast<const uint4 *>(k + j);
    cnt += (v.x > thr) + (v.y > thr) + (v.z > thr) + (v.w > thr);
  }
  for (; j < j1; ++j) cnt += k[j] > thr;
  return cnt;
}

// Position of the e-th (0-based) set bit of the mask w[0..NW) (32 bits a word);
// e < popcount(w).
template <int NW>
__device__ __forceinline__ int nth_set(const uint32_t (&w)[8], int e) {
  int base = 0;
  uint32_t x = 0;
  bool found = false;
#pragma unroll
  for (int i = 0; i < NW; ++i) {
    const int c = __popc(w[i]);
    if (!found) {
      if (e < c) {
        x = w[i];
        base = i * 32;
        found = true;
      } else {
        e -= c;
      }
    }
  }
  int pos = 0;
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const int c = __popc(x & ((1u << s) - 1u));
    if (e >= c) {
      e -= c;
      x >>= s;
      pos += s;
    }
  }
  return base + pos;
}

__device__ __forceinline__ bool bit_of(const uint32_t (&w)[8], int pos) {
  uint32_t x = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) x = (i == (pos >> 5)) ? w[i] : x;
  return (x >> (pos & 31)) & 1u;
}

template <int G>
__device__ __forceinline__ void rotated_query_regs(const uint2 (&qlo)[G], const uint2 (&qhi)[G], const Trig4 &tq,
                                                   float2 (&q2lo)[G][2], float2 (&q2hi)[G][2]) {
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float lo[4], hi[4];
    Row8 r;
    r.lo = qlo[h];
    r.hi = qhi[h];
    unpack_row8(r, lo, hi);
    rotate4(lo, hi, tq);
    q2lo[h][0] = make_float2(lo[0], lo[1]);
    q2lo[h][1] = make_float2(lo[2], lo[3]);
    q2hi[h][0] = make_float2(hi[0], hi[1]);
    q2hi[h][1] = make_float2(hi[2], hi[3]);
  }
}

// Every slice of a level fits in RPH rows per half-warp: ceil(max_cand / CS) <= 16 RPH,
// and max_cand <= kLeanMaxCand (the launcher checks both).
template <int G, int CS, int RPH, bool kPaged = false>
__global__ void __launch_bounds__(kCtaThreads, 1) attend_lean_kernel(const AttendArgs a) {
  static_assert(CS == 2 || CS == 4, "the lean kernel runs in clusters of 2 or 4");
  constexpr unsigned F = 0xffffffffu;
  extern __shared__ __align__(128) unsigned char smem[];
  const LeanLayout Ls = lean_layout(G, CS, a.max_cand);
  Geo *geo_s = reinterpret_cast<Geo *>(smem + Ls.geo);
  uint32_t *kbuf = reinterpret_cast<uint32_t *>(smem + Ls.kbuf);
  uint16_t *mask16 = reinterpret_cast<uint16_t *>(smem + Ls.mask);
  int *par_all = reinterpret_cast<int *>(smem + Ls.par);
  float *red = reinterpret_cast<float *>(smem + Ls.red);  // [warp][h][kRedStride]: m, l, pad, acc[128]
  float *clm = reinterpret_cast<float *>(smem + Ls.clm);  // [rank][h][kRedStride], read on rank 0
  const int MC = a.max_cand;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j16 = lane & 15, hw = warp * 2 + (lane >> 4);
  const int crank = (int)cg::this_cluster().block_rank();
  const int tile = blockIdx.x / CS;
  uint32_t *err = &a.hdr->err;

  cg::cluster_group cluster = cg::this_cluster();
  load_geo(a, geo_s, tid, kCtaThreads);
  __syncthreads();
  const Geo &geo = *geo_s;
  const TileInfo t = tile_info(a, geo, tile);
  const int64_t out0 = (((int64_t)t.s * a.nq + t.qi) * a.hq + (int64_t)t.g * G) * kD;
  // lane j16 < CS stores the scores of its half-warp's rows into cluster CTA j16
  uint32_t *dst_kbuf = cluster.map_shared_rank(kbuf, (unsigned)(j16 % CS));
  // floor(x / b) = umulhi(x, bmagic) for 0 <= x < 2^32 / b
  const uint32_t bmagic = 0xffffffffu / (uint32_t)a.b + 1u;
  auto divb = [&](int x) { return (int)__umulhi((uint32_t)x, bmagic); };

  // the query heads of the group: dims 4j..4j+3 and 64+4j..64+4j+3 (bf16 pairs)
  uint2 qlo[G], qhi[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    qlo[h] = __ldg(reinterpret_cast<const uint2 *>(a.q + out0 + h * kD + 4 * j16));
    qhi[h] = __ldg(reinterpret_cast<const uint2 *>(a.q + out0 + h * kD + kHalf + 4 * j16));
  }

  int fpos;
  int n = top_candidates(a, geo, t, &fpos);
  const int n_cap = min(MC, a.table_rows_needed - 1);
  if (n > n_cap) {  // cannot happen for a valid launch; guards the buffers and the table
    if (tid == 0) atomicOr(err, kErrCount);
    n = n_cap;
  }
  if (fpos >= n) fpos = -1;

  Row8 ck[RPH], cv[RPH], nk[RPH], nv[RPH];
  Trig4 ctr[RPH], ntr[RPH];
  bool cok[RPH], nok[RPH];
  auto load_row = [&](const LevelRows &lr, int pos, int node, bool valid, Row8 &k, Row8 &v, Trig4 &tr, bool &ok) {
    const int64_t row = valid && node >= 0 && node < lr.nrows ? row_at<kPaged>(a, lr, node) : -1;
    ok = row >= 0;
    if (valid && !ok && j16 == 0) atomicOr(err, kErrIndex);
    if (ok) {
      k = ld_row8_now(lr.k + row * kD, j16);
      v = ld_row8_now(lr.v + row * kD, j16);
      tr = ld_trig4_now(a.table, pos, j16);
    }
  };
  // node of candidate `pos` of the current level: the top level lists its nodes in
  // order; below, candidate i is child i % b of the (i / b)-th expanded node above
  auto cand_node = [&](const int *par, bool top, int pos) -> int {
    if (top) return pos;
    const int e = divb(pos);
    return par[e] * a.b + (pos - e * a.b);
  };

  int per = (n + CS - 1) / CS;
  int lo = min(n, crank * per), hi = min(n, lo + per);
  {
    const LevelRows lr = level_rows<kPaged>(a, geo, t.T, t.bh);
#pragma unroll
    for (int r = 0; r < RPH; ++r) {
      const int pos = lo + hw + kHalfWarps * r;
      load_row(lr, pos, pos, pos < hi && pos != fpos, ck[r], cv[r], ctr[r], cok[r]);
    }
  }
  Trig4 tq = ldg_trig4(a.table, n, j16), ntq;
  cluster_barrier();  // every CTA of the cluster runs before the first store into a peer

  float m_w[G], l_w[G];
  float2 acc[G][4];  // dims (4j, 4j+1), (4j+2, 4j+3), (64+4j, ..), (64+4j+2, ..)
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m_w[h] = -INFINITY;
    l_w[h] = 0.f;
#pragma unroll
    for (int d = 0; d < 4; ++d) acc[h][d] = make_float2(0.f, 0.f);
  }
  int keys_read = 0, values_read = 0;

  // Fold the entry rows (values in registers, logits of every head in xs) into the
  // half-warp's online-softmax state.
  auto fold = [&](const Row8 (&vr)[RPH], const float (&xs)[RPH][G], const bool (&ent)[RPH]) {
    float mnew[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float mx = -INFINITY;
#pragma unroll
      for (int r = 0; r < RPH; ++r)
        if (ent[r]) mx = fmaxf(mx, xs[r][h]);
      mx = fmaxf(mx, __shfl_xor_sync(F, mx, 16));
      mnew[h] = fmaxf(m_w[h], mx);
      const float alpha = (mnew[h] == -INFINITY) ? 1.f : __expf(m_w[h] - mnew[h]);
      m_w[h] = mnew[h];
      l_w[h] *= alpha;
      const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
      for (int d = 0; d < 4; ++d) acc[h][d] = __fmul2_rn(acc[h][d], a2);
    }
    float ls[G];
#pragma unroll
    for (int h = 0; h < G; ++h) ls[h] = 0.f;
#pragma unroll
    for (int r = 0; r < RPH; ++r)
      if (ent[r]) {
        const Row8 &v = vr[r];
        const float2 v0 = make_float2(bf16_lo(v.lo.x), bf16_hi(v.lo.x)), v1 = make_float2(bf16_lo(v.lo.y), bf16_hi(v.lo.y));
        const float2 v2 = make_float2(bf16_lo(v.hi.x), bf16_hi(v.hi.x)), v3 = make_float2(bf16_lo(v.hi.y), bf16_hi(v.hi.y));
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float pr = __expf(xs[r][h] - mnew[h]);
          ls[h] += pr;
          const float2 p2 = make_float2(pr, pr);
          acc[h][0] = __ffma2_rn(p2, v0, acc[h][0]);
          acc[h][1] = __ffma2_rn(p2, v1, acc[h][1]);
          acc[h][2] = __ffma2_rn(p2, v2, acc[h][2]);
          acc[h][3] = __ffma2_rn(p2, v3, acc[h][3]);
        }
      }
#pragma unroll
    for (int h = 0; h < G; ++h) l_w[h] += ls[h] + __shfl_xor_sync(F, ls[h], 16);
  };

  for (int j = 0, lvl = t.T;; ++j, --lvl) {
    const int pb = j & 1;
    const bool top = lvl == t.T;
    const int *par_cur = par_all + pb * MC;  // written one level up (unused at the top)
    // 1. scores of this CTA's rows: logits of every head (xs) and the group score key
    float xs[RPH][G];
    uint32_t key[RPH];
    {
      float2 q2lo[G][2], q2hi[G][2];
      rotated_query_regs<G>(qlo, qhi, tq, q2lo, q2hi);
#pragma unroll
      for (int r = 0; r < RPH; ++r) {
        float part[G];
#pragma unroll
        for (int h = 0; h < G; ++h) part[h] = 0.f;
        if (cok[r]) dot_row8<G>(ck[r], ctr[r], q2lo, q2hi, part);
        const float x = reduce16<G>(part, j16) * a.scale;
        const float S = group_sum16<G>(x);  // shuffles: every lane, row or not
        key[r] = cok[r] ? order_key(S) : 0u;
#pragma unroll
        for (int h = 0; h < G; ++h) xs[r][h] = __shfl_sync(F, x, (lane & 16) | (h << (4 - log2g<G>())));
      }
    }
    const int m = n - (fpos >= 0 ? 1 : 0);
    keys_read += m;
    bool ent[RPH];
    if (lvl == 0) {
      values_read += n;
#pragma unroll
      for (int r = 0; r < RPH; ++r) ent[r] = cok[r];
      fold(cv, xs, ent);
      break;
    }

    // 2. the group scores go to every CTA of the cluster (lane j16 < CS of each
    //    half-warp into CTA j16); the barrier publishes them
    if (j16 < CS) {
#pragma unroll
      for (int r = 0; r < RPH; ++r) {
        const int pos = lo + hw + kHalfWarps * r;
        if (pos < hi) dst_kbuf[pb * kLeanMaxCand + pos] = key[r];
      }
    }
    // the ranking reads whole chunks of 8: positions n .. n rounded up to 8 score nothing
    if (tid < 8 && n + tid < ((n + 7) & ~7)) kbuf[pb * kLeanMaxCand + n + tid] = 0u;
    const LevelRows lb = level_rows<kPaged>(a, geo, lvl - 1, t.bh);
    cluster_barrier();

    // 3. rank: candidate c is kept when fewer than top_k scorable candidates beat it
    //    (higher score, or equal score at a lower position)
    uint32_t kw[8], ew[8];
    {
      const uint32_t *kb = kbuf + pb * kLeanMaxCand;
      int c, better;
      uint32_t kc;
      if (n <= 128) {
        // warp w ranks candidates 16w .. 16w+15 (lane j16), each half-warp taking half of
        // every chunk of 8 competitors: half p reads positions 8t+4p .. 8t+4p+3 of chunk t.
        // Chunks before 2w lie wholly below the warp's candidates (a tie there beats the
        // candidate: count >=), chunks after 2w+1 wholly above (count >); only the two
        // chunks of the warp's own candidates compare position by position.
        c = warp * 16 + j16;
        kc = c < n ? kb[c] : 0u;
        const uint32_t thr_lo = kc - 1u, thr_hi = kc;
        const int half4 = (lane >> 4) * 4, nch = (n + 7) >> 3, w0 = min(2 * warp, nch), w1 = min(2 * warp + 2, nch);
        better = 0;
#pragma unroll 4
        for (int t8 = 0; t8 < w0; ++t8) {
          const uint4 v = *reinterpret_cast<const uint4 *>(kb + 8 * t8 + half4);
          better += (v.x > thr_lo) + (v.y > thr_lo) + (v.z > thr_lo) + (v.w > thr_lo);
        }
        for (int t8 = w0; t8 < w1; ++t8) {
          const int j = 8 * t8 + half4;
          const uint4 v = *reinterpret_cast<const uint4 *>(kb + j);
          better += (v.x > (j < c ? thr_lo : thr_hi)) + (v.y > (j + 1 < c ? thr_lo : thr_hi)) +
                    (v.z > (j + 2 < c ? thr_lo : thr_hi)) + (v.w > (j + 3 < c ? thr_lo : thr_hi));
        }
#pragma unroll 4
        for (int t8 = w1; t8 < nch; ++t8) {
          const uint4 v = *reinterpret_cast<const uint4 *>(kb + 8 * t8 + half4);
          better += (v.x > thr_hi) + (v.y > thr_hi) + (v.z > thr_hi) + (v.w > thr_hi);
        }
        better += __shfl_xor_sync(F, better, 16);
      } else {
        c = tid;
        kc = c < n ? kb[c] : 0u;
        better = count_above(kb, 0, min(n, c), kc - 1u) + count_above(kb, min(n, c + 1), n, kc);
      }
      const unsigned bal = __ballot_sync(F, c < n && kc != 0u && better < a.top_k);
      if (lane == 0) {
        uint16_t *mk = mask16 + pb * 16;
        if (n <= 128) {
          mk[warp] = (uint16_t)(bal & 0xffffu);
        } else {
          mk[2 * warp] = (uint16_t)(bal & 0xffffu);
          mk[2 * warp + 1] = (uint16_t)(bal >> 16);
        }
      }
    }
    __syncthreads();
    {
      const uint4 w0 = *reinterpret_cast<const uint4 *>(mask16 + pb * 16);
      uint4 w1 = make_uint4(0u, 0u, 0u, 0u);
      if (n > 128) w1 = *reinterpret_cast<const uint4 *>(mask16 + pb * 16 + 8);
      kw[0] = w0.x, kw[1] = w0.y, kw[2] = w0.z, kw[3] = w0.w;
      kw[4] = w1.x, kw[5] = w1.y, kw[6] = w1.z, kw[7] = w1.w;
    }
    int nK = 0, nE = 0, last = -1;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      ew[i] = kw[i] | ((fpos >= 0 && (fpos >> 5) == i) ? (1u << (fpos & 31)) : 0u);
      nK += __popc(kw[i]);
      nE += __popc(ew[i]);
      if (ew[i]) last = i * 32 + 31 - __clz(ew[i]);
    }
    values_read += m - min(a.top_k, m);

    // 4. the next level: this CTA's slice, the slice's rows, the level's size and forced
    //    node.  Slices are cut from the expanded count alone: every CTA computes the same
    //    cut, and together the slices cover every position (CS * 16 RPH >= max_cand), so
    //    the row addresses need not wait for the last node's child count.
    auto nth = [&](const uint32_t (&w)[8], int e) { return n <= 128 ? nth_set<4>(w, e) : nth_set<8>(w, e); };
    const int per2 = min((nE * a.b + CS - 1) / CS, kHalfWarps * RPH);
    const int lo2 = crank * per2;
    int n_next = 0, fpos_next = -1;
    if (last >= 0) {
      bool lf = false;
      const int nch =
          child_count(a, geo, (uint32_t)cand_node(par_cur, top, last) | (last == fpos ? kForced : 0u), lvl, t.p, &lf);
      n_next = (nE - 1) * a.b + nch;
      if (lf) fpos_next = n_next - 1;
    }
    if (n_next > n_cap) {
      if (tid == 0) atomicOr(err, kErrCount);
      n_next = n_cap;
      if (fpos_next >= n_next) fpos_next = -1;
    }
    const int hi2 = min(n_next, lo2 + per2);
#pragma unroll
    for (int r = 0; r < RPH; ++r) {
      const int i = lo2 + hw + kHalfWarps * r;
      const bool valid = i < hi2 && i != fpos_next;
      int node = 0;
      if (valid) {
        const int e = divb(i);
        node = cand_node(par_cur, top, nth(ew, e)) * a.b + (i - e * a.b);
      }
      load_row(lb, i, node, valid, nk[r], nv[r], ntr[r], nok[r]);
    }
    ntq = ld_trig4_now(a.table, n_next, j16);
    if (tid < nE) par_all[(pb ^ 1) * MC + tid] = cand_node(par_cur, top, nth(ew, tid));
    if (a.sel_idx != nullptr && crank == 0 && lvl <= a.sel_levels) {
      int32_t *sel = a.sel_idx + ((int64_t)tile * a.sel_levels + (lvl - 1)) * a.top_k;
      for (int u = tid; u < a.top_k; u += kCtaThreads) sel[u] = u < nK ? cand_node(par_cur, top, nth(kw, u)) : -1;
    }

    // 5. fold this level's unkept candidates while the next level's rows are in flight
#pragma unroll
    for (int r = 0; r < RPH; ++r) ent[r] = cok[r] && !bit_of(kw, lo + hw + kHalfWarps * r);
    fold(cv, xs, ent);

#pragma unroll
    for (int r = 0; r < RPH; ++r) {
      ck[r] = nk[r];
      cv[r] = nv[r];
      ctr[r] = ntr[r];
      cok[r] = nok[r];
    }
    tq = ntq;
    n = n_next;
    fpos = fpos_next;
    lo = lo2;
    hi = hi2;
  }

  if (crank == 0 && tid == 0) flag_bad_length(a, t.s);
  if (a.entries != nullptr && crank == 0 && tid == 0) {
    a.entries[2 * (int64_t)tile] = keys_read;
    a.entries[2 * (int64_t)tile + 1] = values_read;
  }

  // merge: half-warps -> warp -> CTA (here) -> cluster (on rank 0)
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float2 x[4];
#pragma unroll
    for (int d = 0; d < 4; ++d) {
      x[d].x = acc[h][d].x + __shfl_xor_sync(F, acc[h][d].x, 16);
      x[d].y = acc[h][d].y + __shfl_xor_sync(F, acc[h][d].y, 16);
    }
    float *r = red + (warp * G + h) * kRedStride;
    if (lane == 0) {
      r[0] = m_w[h];
      r[1] = l_w[h];
    }
    if (lane < 16) {
      *reinterpret_cast<float4 *>(r + 4 + 4 * j16) = make_float4(x[0].x, x[0].y, x[1].x, x[1].y);
      *reinterpret_cast<float4 *>(r + 4 + kHalf + 4 * j16) = make_float4(x[2].x, x[2].y, x[3].x, x[3].y);
    }
  }
  __syncthreads();
  float *dst_clm = cluster.map_shared_rank(clm, 0u);
  for (int e = tid; e < G * kD / 4; e += kCtaThreads) {
    const int h = (4 * e) / kD, d0 = (4 * e) % kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kCtaWarps; ++w) M = fmaxf(M, red[(w * G + h) * kRedStride]);
    float l = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kCtaWarps; ++w) {
        const float *r = red + (w * G + h) * kRedStride;
        const float f = (r[0] == -INFINITY) ? 0.f : __expf(r[0] - M);
        l += f * r[1];
#pragma unroll
        for (int d = 0; d < 4; ++d) o[d] += f * r[4 + d0 + d];
      }
    }
    float *dst = dst_clm + (crank * G + h) * kRedStride;
    if (d0 == 0) {
      dst[0] = M;
      dst[1] = l;
    }
    *reinterpret_cast<float4 *>(dst + 4 + d0) = make_float4(o[0], o[1], o[2], o[3]);
  }
  cluster_barrier();  // every partial is in rank 0; no CTA stores into a peer after this
  if (crank == 0) {
    const bool ws_bad = !workspace_ok(a);
    for (int e = tid; e < G * kD / 4; e += kCtaThreads) {
      const int h = (4 * e) / kD, d0 = (4 * e) % kD;
      float M = -INFINITY;
#pragma unroll
      for (int r = 0; r < CS; ++r) M = fmaxf(M, clm[(r * G + h) * kRedStride]);
      float l = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
      if (M != -INFINITY) {
#pragma unroll
        for (int r = 0; r < CS; ++r) {
          const float *x = clm + (r * G + h) * kRedStride;
          const float f = (x[0] == -INFINITY) ? 0.f : __expf(x[0] - M);
          l += f * x[1];
#pragma unroll
          for (int d = 0; d < 4; ++d) o[d] += f * x[4 + d0 + d];
        }
      }
      const float inv = (l > 0.f && !ws_bad) ? 1.f / l : 0.f;
      store_out4(a, out0 + 4 * e, o[0] * inv, o[1] * inv, o[2] * inv, o[3] * inv);
    }
    if (ws_bad && tid == 0) atomicOr(err, kErrWs);
  }
}

// ================================================================== warp-per-tile kernel

__host__ __device__ inline int warp_slice_bytes(int G, int max_cand) {
  return (G * kD + (4 + G) * max_cand) * 4;  // q, 2 candidate lists, logits, keys, entry list
}

template <int G, bool kPaged = false>
__global__ void __launch_bounds__(kWarpKernelMaxWarps * 32, (G <= 4 ? 2 : 1)) attend_warp_kernel(const AttendArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int j16 = lane & 15, half = lane >> 4;
  const int MC = a.max_cand;
  float *qraw = reinterpret_cast<float *>(smem + (size_t)wib * warp_slice_bytes(G, MC));
  uint32_t *cand = reinterpret_cast<uint32_t *>(qraw + G * kD);
  float *slog = reinterpret_cast<float *>(cand + 2 * MC);
  uint32_t *skey = reinterpret_cast<uint32_t *>(slog + G * MC);
  int *list = reinterpret_cast<int *>(skey + MC);
  uint32_t *err = &a.hdr->err;
  const bool ws_ok = workspace_ok(a);
  if (!ws_ok && threadIdx.x == 0 && blockIdx.x == 0) atomicOr(err, kErrWs);
  const int nw = gridDim.x * a.warps_per_block;
  Geo *geo_s = reinterpret_cast<Geo *>(smem + (size_t)a.warps_per_block * warp_slice_bytes(G, MC));
  load_geo(a, geo_s, threadIdx.x, blockDim.x);
  __syncthreads();
  const Geo &geo = *geo_s;

  for (int tile = blockIdx.x * a.warps_per_block + wib; tile < a.tiles; tile += nw) {
    const TileInfo t = tile_info(a, geo, tile);
    const int64_t out0 = (((int64_t)t.s * a.nq + t.qi) * a.hq + (int64_t)t.g * G) * kD;
    if (!ws_ok) {
#pragma unroll
      for (int h = 0; h < G; ++h) store_out4(a, out0 + h * kD + 4 * lane, 0.f, 0.f, 0.f, 0.f);
      continue;
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const uint2 u = __ldg(reinterpret_cast<const uint2 *>(a.q + out0 + h * kD + 4 * lane));
      *reinterpret_cast<float4 *>(qraw + h * kD + 4 * lane) =
          make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
    }
    int fpos;
    int n = top_candidates(a, geo, t, &fpos);
    for (int i = lane; i < n; i += 32) cand[i] = (uint32_t)i | (i == fpos ? kForced : 0u);
    __syncwarp();

    float m_w[G], l_w[G];
    float2 acc[G][2];  // dims (4 lane, 4 lane + 1), (4 lane + 2, 4 lane + 3)
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m_w[h] = -INFINITY;
      l_w[h] = 0.f;
      acc[h][0] = acc[h][1] = make_float2(0.f, 0.f);
    }
    int cur = 0, keys_read = 0, values_read = 0;

    for (int lvl = t.T; lvl >= 0; --lvl) {
      uint32_t *cl = cand + cur * MC;
      if (n > a.table_rows_needed - 1) {
        if (lane == 0) atomicOr(err, kErrCount);
        n = a.table_rows_needed - 1;
      }
      const LevelRows lr = level_rows<kPaged>(a, geo, lvl, t.bh);
      float2 q2lo[G][2], q2hi[G][2];
      {
        float qlo[G][4], qhi[G][4];
        rotated_query<G>(qraw, ldg_trig4(a.table, n, j16), j16, qlo, qhi);
        pack_query<G>(qlo, qhi, q2lo, q2hi);
      }

      // keys pass: one row per half-warp per step, the next step's loads in flight
      Row8 kr_n;
      Trig4 tr_n;
      bool ok_n = false;
      auto fetch = [&](int i) {
        const uint32_t c = i < n ? cl[i] : kForced;
        const int64_t node = c & kNodeMask;
        const int64_t row = i < n && !(c & kForced) && node < lr.nrows ? row_at<kPaged>(a, lr, node) : -1;
        ok_n = row >= 0;
        if (i < n && !(c & kForced) && row < 0 && j16 == 0) atomicOr(err, kErrIndex);
        if (ok_n) {
          kr_n = ldg_row8(lr.k + row * kD, j16);
          tr_n = ldg_trig4(a.table, i, j16);
        }
      };
      fetch(half);
      for (int i0 = 0; i0 < n; i0 += 2) {
        const int i = i0 + half;
        const Row8 kr = kr_n;
        const Trig4 tr = tr_n;
        const bool ok = ok_n;
        fetch(i0 + 2 + half);
        float part[G];
#pragma unroll
        for (int h = 0; h < G; ++h) part[h] = 0.f;
        if (ok) dot_row8<G>(kr, tr, q2lo, q2hi, part);
        const float x = reduce16<G>(part, j16) * a.scale;
        const float S = group_sum16<G>(x);
        if (ok) {
          if (head_writer<G>(j16)) slog[i * G + head_of<G>(j16)] = x;
          if (j16 == 0) skey[i] = order_key(S);
        }
      }
      __syncwarp();

      // selection and the level's entries (unselected candidates; every token at level 0)
      int ne = 0;
      const int nforced = (a.causal && n > 0 && (cl[n - 1] & kForced)) ? 1 : 0;
      if (lvl > 0) {
        warp_topk(cl, skey, n, a.top_k, lane);
        warp_write_selection(a, cl, n, lvl, tile, lane);
        for (int base = 0; base < n; base += 32) {
          const int c = base + lane;
          const uint32_t v = c < n ? cl[c] : kForced;
          const bool e = c < n && !(v & (kKept | kForced)) && (int64_t)(v & kNodeMask) < lr.nrows;
          const unsigned bal = __ballot_sync(0xffffffffu, e);
          if (e) list[ne + __popc(bal & ((1u << lane) - 1u))] = c;
          ne += __popc(bal);
        }
      } else {
        for (int i = lane; i < n; i += 32) list[i] = i;
        ne = n;
      }
      keys_read += n - nforced;
      values_read += ne;
      __syncwarp();

      // online softmax: statistics of this level's entries, then the value rows
      float mx[G];
#pragma unroll
      for (int h = 0; h < G; ++h) mx[h] = -INFINITY;
      for (int e = lane; e < ne; e += 32) {
        const int pos = list[e];
#pragma unroll
        for (int h = 0; h < G; ++h) mx[h] = fmaxf(mx[h], slog[pos * G + h]);
      }
      float mnew[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        mx[h] = warp_max(mx[h]);
        mnew[h] = fmaxf(m_w[h], mx[h]);
        const float alpha = (mnew[h] == -INFINITY) ? 1.f : __expf(m_w[h] - mnew[h]);
        m_w[h] = mnew[h];
        l_w[h] *= alpha;
        const float2 a2 = make_float2(alpha, alpha);
        acc[h][0] = __fmul2_rn(acc[h][0], a2);
        acc[h][1] = __fmul2_rn(acc[h][1], a2);
      }
      float ls[G];
#pragma unroll
      for (int h = 0; h < G; ++h) ls[h] = 0.f;
      for (int e = lane; e < ne; e += 32) {
        const int pos = list[e];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float pr = __expf(slog[pos * G + h] - mnew[h]);
          slog[pos * G + h] = pr;
          ls[h] += pr;
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) l_w[h] += warp_sum(ls[h]);
      __syncwarp();
      for (int e0 = 0; e0 < ne; e0 += 8) {
        uint2 vv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (e0 + u < ne) {
            const int64_t row = row_at<kPaged>(a, lr, cl[list[e0 + u]] & kNodeMask);  // < 0: flagged by the key pass
            vv[u] = row >= 0 ? __ldg(reinterpret_cast<const uint2 *>(lr.v + row * kD + 4 * lane)) : make_uint2(0u, 0u);
          }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (e0 + u < ne) {
            const int pos = list[e0 + u];
            const float2 v01 = make_float2(bf16_lo(vv[u].x), bf16_hi(vv[u].x));
            const float2 v23 = make_float2(bf16_lo(vv[u].y), bf16_hi(vv[u].y));
            float pr[G];
            if constexpr (G % 4 == 0) {
#pragma unroll
              for (int h4 = 0; h4 < G; h4 += 4) {
                const float4 p4 = *reinterpret_cast<const float4 *>(slog + pos * G + h4);
                pr[h4] = p4.x;
                pr[h4 + 1] = p4.y;
                pr[h4 + 2] = p4.z;
                pr[h4 + 3] = p4.w;
              }
            } else {
#pragma unroll
              for (int h = 0; h < G; ++h) pr[h] = slog[pos * G + h];
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float2 p2 = make_float2(pr[h], pr[h]);
              acc[h][0] = __ffma2_rn(p2, v01, acc[h][0]);
              acc[h][1] = __ffma2_rn(p2, v23, acc[h][1]);
            }
          }
      }
      if (lvl == 0) break;
      n = warp_expand(a, geo, cl, n, lvl, t.p, cand + (cur ^ 1) * MC, lane, err);
      cur ^= 1;
      __syncwarp();
    }

#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float inv = l_w[h] > 0.f ? 1.f / l_w[h] : 0.f;
      store_out4(a, out0 + h * kD + 4 * lane, acc[h][0].x * inv, acc[h][0].y * inv, acc[h][1].x * inv,
                 acc[h][1].y * inv);
    }
    if (lane == 0) flag_bad_length(a, t.s);
    if (a.entries != nullptr && lane == 0) {
      a.entries[2 * (int64_t)tile] = keys_read;
      a.entries[2 * (int64_t)tile + 1] = values_read;
    }
    __syncwarp();
  }
}

// ================================================================== launch

int sm_count_cached() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <int G, int CS, bool kPaged>
int launch_cta(const AttendArgs &args, cudaStream_t stream, bool two_per_sm = false) {
  AttendArgs a = args;
  a.own_max = ((a.max_cand + CS - 1) / CS + 31) / 32 * 32;
  const CtaLayout L = cta_layout(G, CS, a.max_cand, a.own_max, a.top_k);
  if (L.total > 227 * 1024) {
    set_error("attend needs %d bytes of shared memory per CTA (limit 232448)", L.total);
    return -1;
  }
  auto kern = attend_cta_kernel<G, CS, kPaged>;
  // shape 4: the two-per-SM instance, where two CTAs' shared memory fits an SM (G <= 4:
  // with 8 query heads a tile, 128 registers a thread spill)
  if constexpr (CS == 1 && G <= 4)
    if (two_per_sm && 2 * (L.total + 1024) <= 228 * 1024) kern = attend_cta_kernel<G, 1, kPaged, true>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
  if (e != cudaSuccess) return (int)e;
  if constexpr (CS == 1) {
    kern<<<a.tiles, kCtaThreads, L.total, stream>>>(a);
    return (int)cudaGetLastError();
  } else {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.tiles * CS));
    cfg.blockDim = dim3(kCtaThreads);
    cfg.dynamicSmemBytes = (size_t)L.total;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) return (int)e;
    return (int)cudaGetLastError();
  }
}

template <int G, bool kPaged>
int launch_warp(const AttendArgs &args, cudaStream_t stream) {
  AttendArgs a = args;
  const int slice = warp_slice_bytes(G, a.max_cand);
  const int sms = sm_count_cached();
  int wpb = std::min(kWarpKernelMaxWarps, (227 * 1024 - kGeoBytes) / slice);
  // few tiles: spread them over the SMs rather than packing 8 per CTA
  wpb = std::max(1, std::min(wpb, (a.tiles + sms - 1) / sms));
  if (wpb < 1) {
    set_error("attend needs %d bytes of shared memory per warp", slice);
    return -1;
  }
  a.warps_per_block = wpb;
  const int smem = wpb * slice + kGeoBytes;
  auto kern = attend_warp_kernel<G, kPaged>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return (int)e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, wpb * 32, smem);
  if (e != cudaSuccess) return (int)e;
  per_sm = std::max(per_sm, 1);
  const int64_t need = (a.tiles + wpb - 1) / wpb;
  const int grid = (int)std::min<int64_t>(need, (int64_t)sms * per_sm);
  kern<<<grid, wpb * 32, smem, stream>>>(a);
  return (int)cudaGetLastError();
}

template <int G, int CS, int RPH, bool kPaged>
int launch_lean_shape(const AttendArgs &a, cudaStream_t stream) {
  const LeanLayout L = lean_layout(G, CS, a.max_cand);
  auto kern = attend_lean_kernel<G, CS, RPH, kPaged>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
  if (e != cudaSuccess) return (int)e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.tiles * CS));
  cfg.blockDim = dim3(kCtaThreads);
  cfg.dynamicSmemBytes = (size_t)L.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) return (int)e;
  return (int)cudaGetLastError();
}

// The lean cluster kernel where its slices fit in registers; kNoLeanShape otherwise.
constexpr int kNoLeanShape = -3;
template <int G, bool kPaged>
int launch_lean(const AttendArgs &a, int CS, cudaStream_t stream) {
  const int mc = a.max_cand;
  if (mc > kLeanMaxCand) return kNoLeanShape;
  if (CS == 4 && mc <= 4 * kHalfWarps * 2) return launch_lean_shape<G, 4, 2, kPaged>(a, stream);
  if constexpr (G <= 4) {
    if (CS == 4 && mc <= 4 * kHalfWarps * 3) return launch_lean_shape<G, 4, 3, kPaged>(a, stream);
    if (CS == 2 && mc <= 2 * kHalfWarps * 4) return launch_lean_shape<G, 2, 4, kPaged>(a, stream);
  }
  return kNoLeanShape;
}

// kPaged: the token caches are a paged pool (level-0 rows through the page table); the
// contiguous kernels carry no trace of it.
template <int G, bool kPaged>
int launch_gp(const AttendArgs &a, int kernel, int CS, cudaStream_t stream) {
  if (kernel == 2) return launch_warp<G, kPaged>(a, stream);
  if (kernel == 4) return launch_cta<G, 1, kPaged>(a, stream, true);
  if (kernel == 3) {
    const int rc = launch_lean<G, kPaged>(a, CS, stream);
    if (rc != kNoLeanShape) return rc;
  }
  switch (CS) {
    case 1: return launch_cta<G, 1, kPaged>(a, stream);
    case 2: return launch_cta<G, 2, kPaged>(a, stream);
    case 4: return launch_cta<G, 4, kPaged>(a, stream);
    default: return -2;
  }
}

template <int G>
int launch_g(const AttendArgs &a, int kernel, int CS, cudaStream_t stream) {
  return a.page_table ? launch_gp<G, true>(a, kernel, CS, stream) : launch_gp<G, false>(a, kernel, CS, stream);
}

}  // namespace

int launch_attend(const AttendLaunch &l, void *stream) {
  AttendArgs a = {};
  a.k_tok = reinterpret_cast<const uint16_t *>(l.tree.k_tok);
  a.v_tok = reinterpret_cast<const uint16_t *>(l.tree.v_tok);
  a.k_node = reinterpret_cast<const uint16_t *>(l.tree.k_node);
  a.v_node = reinterpret_cast<const uint16_t *>(l.tree.v_node);
  a.q = reinterpret_cast<const uint16_t *>(l.q);
  a.out = l.out;
  a.hdr = reinterpret_cast<WsHeader *>(l.ws);
  a.table = reinterpret_cast<const float2 *>(reinterpret_cast<const char *>(l.ws) + kWsHeader);
  a.sel_idx = l.debug ? l.debug->sel_idx : nullptr;
  a.sel_levels = l.debug ? l.debug->sel_levels : 0;
  a.entries = l.debug ? l.debug->entries : nullptr;
  a.cap = l.geom.capacity;
  a.length = l.length;
  a.seq_len = l.tree.seq_len;
  a.page_table = l.tree.page_table;
  a.page_shift = l.tree.page_table ? __builtin_ctz((unsigned)l.tree.page_size) : 0;
  a.num_pages = l.tree.page_table ? l.tree.num_pages : 0;
  for (int i = 0; i <= kMaxLevels; ++i) {
    a.row_off[i] = l.geom.row_off[i];
    a.slots[i] = l.geom.slots[i];
    const int64_t sp = std::min<int64_t>(l.geom.span[i], (int64_t)1 << 30 | 1);
    a.span[i] = (int32_t)sp;
    a.nlen[i] = (int32_t)((l.length + sp - 1) / sp);
  }
  a.levels = l.geom.levels_cap;
  a.hkv = l.geom.hkv;
  a.hq = l.geom.hkv * l.group;
  a.b = l.geom.b;
  a.top_k = l.top_k;
  a.nq = l.num_queries;
  a.causal = l.causal;
  a.out_fp32 = l.out_fp32;
  a.table_rows_needed = l.table_rows_needed;
  a.max_cand = l.max_cand;
  a.scale = l.scale;
  a.tiles = l.geom.batch * l.geom.hkv * l.num_queries;
  const int sms = sm_count_cached();
  int kernel = l.kernel;
  // A cluster (or CTA) per tile while every tile has its own SM, the lean cluster kernel
  // wherever its shape applies (launch_g falls back to the CTA kernel otherwise).  Up to
  // 4 waves of tiles a CTA per tile, two sharing an SM, still finishes first (1M, B = 4:
  // 256 tiles 75 us, 512 tiles 141 us, against 94 and 179 us one CTA per SM and ~245 us
  // for the warp-per-tile grid, which holds every tile at once only beyond that).
  if (kernel == 0) kernel = (a.tiles <= sms) ? 3 : (a.tiles <= 4 * sms) ? 4 : 2;
  int CS = l.cluster_size;
  if ((kernel == 1 || kernel == 3) && CS == 0) CS = (a.tiles * 4 <= sms) ? 4 : (a.tiles * 2 <= sms) ? 2 : 1;
  int rc;
  switch (l.group) {
    case 1: rc = launch_g<1>(a, kernel, CS, (cudaStream_t)stream); break;
    case 2: rc = launch_g<2>(a, kernel, CS, (cudaStream_t)stream); break;
    case 4: rc = launch_g<4>(a, kernel, CS, (cudaStream_t)stream); break;
    case 8: rc = launch_g<8>(a, kernel, CS, (cudaStream_t)stream); break;
    default: rc = -2;
  }
  if (rc == -2) set_error("unsupported group size %d or cluster size %d", l.group, CS);
  return rc;
}

}  // namespace recsa
