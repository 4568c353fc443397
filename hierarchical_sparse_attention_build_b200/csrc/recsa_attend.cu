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
constexpr int kPassRows = 2 * kHalfWarps;           // rows a CTA holds per pass (2 per half-warp)
constexpr int kWarpKernelMaxWarps = 8;
constexpr int kTopkRegs = 8;                        // iterative top-k handles up to 256 candidates
// merge rows: m, l, 2 pad, acc[128] (the accumulator starts 16-byte aligned)
constexpr int kRedStride = kD + 4;

struct AttendArgs {
  const uint16_t *k_tok, *v_tok, *k_node, *v_node;
  const uint16_t *q;
  void *out;
  const float2 *table;
  WsHeader *hdr;
  int32_t *sel_idx;
  int32_t *entries;
  int64_t cap;
  int64_t length;  // decode: L; prefill: L before the chunk
  int64_t row_off[kMaxLevels + 1];
  int64_t slots[kMaxLevels + 1];
  int64_t span[kMaxLevels + 1];
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

struct TileInfo {
  int s, g, qi, T;
  int64_t p, bh;
};

__device__ __forceinline__ TileInfo tile_info(const AttendArgs &a, int tile) {
  TileInfo t;
  t.qi = tile % a.nq;
  const int sg = tile / a.nq;
  t.g = sg % a.hkv;
  t.s = sg / a.hkv;
  t.p = a.causal ? a.length + t.qi : a.length;
  t.bh = (int64_t)t.s * a.hkv + t.g;
  int T = 0;
  int64_t n = t.p;
  while (n > a.b) {
    n = (n + a.b - 1) / a.b;
    ++T;
  }
  t.T = T;
  return t;
}

// Candidate count of the top level; *forced_pos = position of the forced partial node or -1.
__device__ __forceinline__ int top_candidates(const AttendArgs &a, const TileInfo &t, int *forced_pos) {
  *forced_pos = -1;
  if (t.T == 0) return (int)t.p;
  if (!a.causal) return (int)((a.length + a.span[t.T] - 1) / a.span[t.T]);
  const int full = (int)(t.p / a.span[t.T]);
  if (t.p % a.span[t.T]) {
    *forced_pos = full;
    return full + 1;
  }
  return full;
}

struct LevelRows {
  const uint16_t *k, *v;
  int64_t nrows;
};

__device__ __forceinline__ LevelRows level_rows(const AttendArgs &a, int lvl, int64_t bh) {
  LevelRows r;
  if (lvl == 0) {
    r.k = a.k_tok + bh * a.cap * kD;
    r.v = a.v_tok + bh * a.cap * kD;
    r.nrows = a.cap;
  } else {
    const int64_t o = (a.row_off[lvl] + bh * a.slots[lvl]) * kD;
    r.k = a.k_node + o;
    r.v = a.v_node + o;
    r.nrows = a.slots[lvl];
  }
  return r;
}

// Children of an expanded candidate `v` at level lvl (in node order); *last_forced tells
// whether the last visible child is itself a partial node (causal mode only).
__device__ __forceinline__ int child_count(const AttendArgs &a, uint32_t v, int lvl, int64_t p, bool *last_forced) {
  const int64_t node = v & kNodeMask;
  const int64_t sb = a.span[lvl - 1];
  *last_forced = false;
  if (!a.causal) {
    const int64_t n_below = (a.length + sb - 1) / sb;
    return (int)max((int64_t)0, min((int64_t)a.b, n_below - node * a.b));
  }
  if (!(v & kForced)) return a.b;
  const int64_t first = node * a.b;  // children starting before p are visible
  const int nch = (int)max((int64_t)0, min((int64_t)a.b, (p - first * sb + sb - 1) / sb));
  if (nch > 0) *last_forced = (first + nch) * sb > p;
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
  float4 a, b;  // (cos, sin) of the 4 frequencies 4j..4j+3
};

__device__ __forceinline__ Trig4 ldg_trig4(const float2 *table, int pos, int j16) {
  const float4 *t = reinterpret_cast<const float4 *>(table + (int64_t)pos * kHalf + 4 * j16);
  Trig4 r;
  r.a = __ldg(t);
  r.b = __ldg(t + 1);
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
  const float c[4] = {tr.a.x, tr.a.z, tr.b.x, tr.b.z};
  const float s[4] = {tr.a.y, tr.a.w, tr.b.y, tr.b.w};
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

// Partial dot products of the rotated key row with the G rotated query heads.
template <int G>
__device__ __forceinline__ void dot_row8(const Row8 &k, const Trig4 &tr, const float (&qlo)[G][4],
                                         const float (&qhi)[G][4], float (&part)[G]) {
  float lo[4], hi[4];
  unpack_row8(k, lo, hi);
  rotate4(lo, hi, tr);
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float x = 0.f;
#pragma unroll
    for (int t = 0; t < 4; ++t) x = fmaf(qlo[h][t], lo[t], fmaf(qhi[h][t], hi[t], x));
    part[h] = x;
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
__device__ int warp_expand(const AttendArgs &a, const uint32_t *cl, int n, int lvl, int64_t p, uint32_t *nx,
                           int lane, uint32_t *err) {
  int total = 0;
  for (int base = 0; base < n; base += 32) {
    const int c = base + lane;
    const uint32_t v = c < n ? cl[c] : 0u;
    bool lf = false;
    const int nch = (c < n && (v & (kKept | kForced))) ? child_count(a, v, lvl, p, &lf) : 0;
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
  int q, cand, skey, slog, red, clm, misc, total;
};

__host__ __device__ inline int align128(int x) { return (x + 127) & ~127; }

__host__ __device__ inline CtaLayout cta_layout(int G, int CS, int max_cand, int own_max) {
  CtaLayout L;
  int o = 0;
  auto take = [&o](int bytes) {
    const int r = o;
    o = align128(o + bytes);
    return r;
  };
  L.misc = take(64);
  L.q = take(G * kD * 4);
  L.cand = take(2 * max_cand * 4);
  L.skey = take((CS > 1 ? 2 : 1) * max_cand * 4);
  L.slog = take(G * own_max * 4);
  L.red = take(kCtaWarps * G * kRedStride * 4);
  L.clm = CS > 1 ? take(CS * G * kRedStride * 4) : 0;
  L.total = o;
  return L;
}

template <int G, int CS>
__global__ void __launch_bounds__(kCtaThreads, 1) attend_cta_kernel(const AttendArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const CtaLayout Ls = cta_layout(G, CS, a.max_cand, a.own_max);
  int *misc = reinterpret_cast<int *>(smem + Ls.misc);  // [0] next candidate count, [1] workspace bad
  float *qraw = reinterpret_cast<float *>(smem + Ls.q);
  uint32_t *cand = reinterpret_cast<uint32_t *>(smem + Ls.cand);
  uint32_t *skey_all = reinterpret_cast<uint32_t *>(smem + Ls.skey);
  float *slog = reinterpret_cast<float *>(smem + Ls.slog);
  const int OWN = a.own_max, MC = a.max_cand;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j16 = lane & 15, hw = warp * 2 + (lane >> 4);  // half-warp id 0..15
  int crank = 0;
  if constexpr (CS > 1) crank = (int)cg::this_cluster().block_rank();
  const int tile = blockIdx.x / CS;
  const TileInfo t = tile_info(a, tile);
  uint32_t *err = &a.hdr->err;
  const int64_t out0 = (((int64_t)t.s * a.nq + t.qi) * a.hq + (int64_t)t.g * G) * kD;

  if (tid == 0) misc[1] = workspace_ok(a) ? 0 : 1;
  {
    const uint16_t *qg = a.q + out0;  // q and out share the [B][Q][Hq][128] layout
    for (int e = tid; e < G * kD / 4; e += kCtaThreads) {
      const uint2 u = __ldg(reinterpret_cast<const uint2 *>(qg) + e);
      *reinterpret_cast<float4 *>(qraw + 4 * e) = make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
    }
  }
  int fpos;
  int n = top_candidates(a, t, &fpos);
  for (int i = tid; i < n; i += kCtaThreads) cand[i] = (uint32_t)i | (i == fpos ? kForced : 0u);
  __syncthreads();
  if (misc[1]) {  // identical in every CTA of the cluster: leave before any cluster barrier
    if (tid == 0 && crank == 0) atomicOr(err, kErrWs);
    if (crank == 0)
      for (int e = tid; e < G * kD / 4; e += kCtaThreads) store_out4(a, out0 + 4 * e, 0.f, 0.f, 0.f, 0.f);
    return;
  }
  if constexpr (CS > 1) cluster_barrier();  // every peer runs before the first DSMEM store

  float m_w[G], l_w[G], acc[G][8];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m_w[h] = -INFINITY;
    l_w[h] = 0.f;
#pragma unroll
    for (int d = 0; d < 8; ++d) acc[h][d] = 0.f;
  }
  int cur = 0, keys_read = 0, values_read = 0;

  // Fold up to two rows per half-warp (values in registers) into the warp's state.
  auto fold_rows = [&](const Row8 (&vr)[2], const int (&ii)[2], const bool (&ent)[2], int lo_r) {
    float mx[G];
#pragma unroll
    for (int h = 0; h < G; ++h) mx[h] = -INFINITY;
#pragma unroll
    for (int r = 0; r < 2; ++r)
      if (ent[r]) {
#pragma unroll
        for (int h = 0; h < G; ++h) mx[h] = fmaxf(mx[h], slog[h * OWN + ii[r] - lo_r]);
      }
    float mnew[G], alpha[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 16));
      mnew[h] = fmaxf(m_w[h], mx[h]);
      alpha[h] = (mnew[h] == -INFINITY) ? 1.f : expf(m_w[h] - mnew[h]);
      m_w[h] = mnew[h];
      l_w[h] *= alpha[h];
#pragma unroll
      for (int d = 0; d < 8; ++d) acc[h][d] *= alpha[h];
    }
    float ls[G];
#pragma unroll
    for (int h = 0; h < G; ++h) ls[h] = 0.f;
#pragma unroll
    for (int r = 0; r < 2; ++r)
      if (ent[r]) {
        float lo[4], hi[4];
        unpack_row8(vr[r], lo, hi);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float pr = expf(slog[h * OWN + ii[r] - lo_r] - mnew[h]);
          ls[h] += pr;
#pragma unroll
          for (int d = 0; d < 4; ++d) {
            acc[h][d] = fmaf(pr, lo[d], acc[h][d]);
            acc[h][4 + d] = fmaf(pr, hi[d], acc[h][4 + d]);
          }
        }
      }
#pragma unroll
    for (int h = 0; h < G; ++h) l_w[h] += ls[h] + __shfl_xor_sync(0xffffffffu, ls[h], 16);
  };

  for (int lvl = t.T; lvl >= 0; --lvl) {
    uint32_t *cl = cand + cur * MC;
    uint32_t *sk = skey_all + ((CS > 1) ? (lvl & 1) * MC : 0);
    if (n > a.table_rows_needed - 1) {  // cannot happen for a valid launch; guards the table read
      if (tid == 0) atomicOr(err, kErrCount);
      n = a.table_rows_needed - 1;
    }
    const int per = (n + CS - 1) / CS;
    const int lo_r = min(n, crank * per);
    const int hi_r = min(n, lo_r + per);
    const bool single = hi_r - lo_r <= kPassRows;
    const LevelRows lr = level_rows(a, lvl, t.bh);
    const Trig4 tq = ldg_trig4(a.table, n, j16);

    // 1. gather and score this CTA's slice; in one pass the values come along
    Row8 vr[2];
    int ii[2] = {lo_r, lo_r};
    bool ent[2] = {false, false};
    for (int pass0 = lo_r; pass0 < hi_r; pass0 += kPassRows) {
      Row8 kr[2];
      Trig4 tr[2];
      bool ok[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int i = pass0 + hw + kHalfWarps * r;
        ii[r] = i;
        const uint32_t c = i < hi_r ? cl[i] : kForced;
        const int64_t node = c & kNodeMask;
        ok[r] = i < hi_r && !(c & kForced) && node < lr.nrows;
        if (i < hi_r && !(c & kForced) && node >= lr.nrows && j16 == 0) atomicOr(err, kErrIndex);
        if (ok[r]) {
          kr[r] = ldg_row8(lr.k + node * kD, j16);
          tr[r] = ldg_trig4(a.table, i, j16);
          if (single) vr[r] = ldg_row8(lr.v + node * kD, j16);
        }
      }
      float qlo[G][4], qhi[G][4];
      rotated_query<G>(qraw, tq, j16, qlo, qhi);
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float part[G];
#pragma unroll
        for (int h = 0; h < G; ++h) part[h] = 0.f;
        if (ok[r]) dot_row8<G>(kr[r], tr[r], qlo, qhi, part);
        const float x = reduce16<G>(part, j16) * a.scale;
        const float S = group_sum16<G>(x);
        if (ok[r]) {
          if (head_writer<G>(j16)) slog[head_of<G>(j16) * OWN + ii[r] - lo_r] = x;
          if (lvl > 0 && j16 == 0) {
            const uint32_t key = order_key(S);
            if constexpr (CS > 1) {
              cg::cluster_group cluster = cg::this_cluster();
#pragma unroll
              for (int q = 0; q < CS; ++q) cluster.map_shared_rank(sk, q)[ii[r]] = key;
            } else {
              sk[ii[r]] = key;
            }
          }
        }
        ent[r] = ok[r];
      }
    }
    int nforced = (a.causal && n > 0 && (cl[n - 1] & kForced)) ? 1 : 0;
    const int m = n - nforced;
    keys_read += m;
    if constexpr (CS > 1) cluster_barrier();
    __syncthreads();

    // 2. selection (one warp), then fold own entries while that warp expands
    if (lvl > 0) {
      if (warp == 0) {
        warp_topk(cl, sk, n, a.top_k, lane);
        if (crank == 0) warp_write_selection(a, cl, n, lvl, tile, lane);
      }
      __syncthreads();
      values_read += m - min(a.top_k, m);
    } else {
      values_read += n;
    }
    if (lvl > 0 && warp == 0) misc[0] = warp_expand(a, cl, n, lvl, t.p, cand + (cur ^ 1) * MC, lane, err);
    if (single) {
      if (lvl > 0) {
#pragma unroll
        for (int r = 0; r < 2; ++r) ent[r] = ent[r] && !(cl[ii[r]] & kKept);
      }
      fold_rows(vr, ii, ent, lo_r);
    } else {
      for (int pass0 = lo_r; pass0 < hi_r; pass0 += kPassRows) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int i = pass0 + hw + kHalfWarps * r;
          ii[r] = i;
          const uint32_t c = i < hi_r ? cl[i] : (kForced | kKept);
          const int64_t node = c & kNodeMask;
          ent[r] = i < hi_r && !(c & (kForced | kKept)) && node < lr.nrows;
          if (ent[r]) vr[r] = ldg_row8(lr.v + node * kD, j16);
        }
        fold_rows(vr, ii, ent, lo_r);
      }
    }
    if (lvl == 0) break;
    __syncthreads();
    n = misc[0];
    cur ^= 1;
  }

  if (a.entries != nullptr && crank == 0 && tid == 0) {
    a.entries[2 * (int64_t)tile] = keys_read;
    a.entries[2 * (int64_t)tile + 1] = values_read;
  }

  // merge: half-warps -> warp -> CTA -> cluster
  float *red = reinterpret_cast<float *>(smem + Ls.red);  // [warp][h][kRedStride]: m, l, pad, acc[128]
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int d = 0; d < 8; ++d) acc[h][d] += __shfl_xor_sync(0xffffffffu, acc[h][d], 16);
    float *r = red + (warp * G + h) * kRedStride;
    if (lane == 0) {
      r[0] = m_w[h];
      r[1] = l_w[h];
    }
    if (lane < 16) {
      *reinterpret_cast<float4 *>(r + 4 + 4 * j16) = make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
      *reinterpret_cast<float4 *>(r + 4 + kHalf + 4 * j16) = make_float4(acc[h][4], acc[h][5], acc[h][6], acc[h][7]);
    }
  }
  __syncthreads();
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
        const float f = (r[0] == -INFINITY) ? 0.f : expf(r[0] - M);
        l += f * r[1];
#pragma unroll
        for (int d = 0; d < 4; ++d) o[d] += f * r[4 + d0 + d];
      }
    }
    if constexpr (CS == 1) {
      const float inv = l > 0.f ? 1.f / l : 0.f;
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
            const float f = (x[0] == -INFINITY) ? 0.f : expf(x[0] - M);
            l += f * x[1];
#pragma unroll
            for (int d = 0; d < 4; ++d) o[d] += f * x[4 + d0 + d];
          }
        }
        const float inv = l > 0.f ? 1.f / l : 0.f;
        store_out4(a, out0 + 4 * e, o[0] * inv, o[1] * inv, o[2] * inv, o[3] * inv);
      }
    }
  }
}

// ================================================================== warp-per-tile kernel

__host__ __device__ inline int warp_slice_bytes(int G, int max_cand) {
  return (G * kD + (4 + G) * max_cand) * 4;  // q, 2 candidate lists, logits, keys, entry list
}

template <int G>
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

  for (int tile = blockIdx.x * a.warps_per_block + wib; tile < a.tiles; tile += nw) {
    const TileInfo t = tile_info(a, tile);
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
    int n = top_candidates(a, t, &fpos);
    for (int i = lane; i < n; i += 32) cand[i] = (uint32_t)i | (i == fpos ? kForced : 0u);
    __syncwarp();

    float m_w[G], l_w[G], acc[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m_w[h] = -INFINITY;
      l_w[h] = 0.f;
#pragma unroll
      for (int d = 0; d < 4; ++d) acc[h][d] = 0.f;
    }
    int cur = 0, keys_read = 0, values_read = 0;

    for (int lvl = t.T; lvl >= 0; --lvl) {
      uint32_t *cl = cand + cur * MC;
      if (n > a.table_rows_needed - 1) {
        if (lane == 0) atomicOr(err, kErrCount);
        n = a.table_rows_needed - 1;
      }
      const LevelRows lr = level_rows(a, lvl, t.bh);
      float qlo[G][4], qhi[G][4];
      rotated_query<G>(qraw, ldg_trig4(a.table, n, j16), j16, qlo, qhi);

      // keys pass: one row per half-warp per step, the next step's loads in flight
      Row8 kr_n;
      Trig4 tr_n;
      bool ok_n = false;
      auto fetch = [&](int i) {
        const uint32_t c = i < n ? cl[i] : kForced;
        const int64_t node = c & kNodeMask;
        ok_n = i < n && !(c & kForced) && node < lr.nrows;
        if (i < n && !(c & kForced) && node >= lr.nrows && j16 == 0) atomicOr(err, kErrIndex);
        if (ok_n) {
          kr_n = ldg_row8(lr.k + node * kD, j16);
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
        if (ok) dot_row8<G>(kr, tr, qlo, qhi, part);
        const float x = reduce16<G>(part, j16) * a.scale;
        const float S = group_sum16<G>(x);
        if (ok) {
          if (head_writer<G>(j16)) slog[head_of<G>(j16) * MC + i] = x;
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
        for (int h = 0; h < G; ++h) mx[h] = fmaxf(mx[h], slog[h * MC + pos]);
      }
      float mnew[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        mx[h] = warp_max(mx[h]);
        mnew[h] = fmaxf(m_w[h], mx[h]);
        const float alpha = (mnew[h] == -INFINITY) ? 1.f : expf(m_w[h] - mnew[h]);
        m_w[h] = mnew[h];
        l_w[h] *= alpha;
#pragma unroll
        for (int d = 0; d < 4; ++d) acc[h][d] *= alpha;
      }
      float ls[G];
#pragma unroll
      for (int h = 0; h < G; ++h) ls[h] = 0.f;
      for (int e = lane; e < ne; e += 32) {
        const int pos = list[e];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float pr = expf(slog[h * MC + pos] - mnew[h]);
          slog[h * MC + pos] = pr;
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
            const int64_t node = cl[list[e0 + u]] & kNodeMask;
            vv[u] = __ldg(reinterpret_cast<const uint2 *>(lr.v + node * kD + 4 * lane));
          }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (e0 + u < ne) {
            const int pos = list[e0 + u];
            const float v0 = bf16_lo(vv[u].x), v1 = bf16_hi(vv[u].x), v2 = bf16_lo(vv[u].y), v3 = bf16_hi(vv[u].y);
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float pr = slog[h * MC + pos];
              acc[h][0] = fmaf(pr, v0, acc[h][0]);
              acc[h][1] = fmaf(pr, v1, acc[h][1]);
              acc[h][2] = fmaf(pr, v2, acc[h][2]);
              acc[h][3] = fmaf(pr, v3, acc[h][3]);
            }
          }
      }
      if (lvl == 0) break;
      n = warp_expand(a, cl, n, lvl, t.p, cand + (cur ^ 1) * MC, lane, err);
      cur ^= 1;
      __syncwarp();
    }

#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float inv = l_w[h] > 0.f ? 1.f / l_w[h] : 0.f;
      store_out4(a, out0 + h * kD + 4 * lane, acc[h][0] * inv, acc[h][1] * inv, acc[h][2] * inv, acc[h][3] * inv);
    }
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

template <int G, int CS>
int launch_cta(const AttendArgs &args, cudaStream_t stream) {
  AttendArgs a = args;
  a.own_max = ((a.max_cand + CS - 1) / CS + 31) / 32 * 32;
  const CtaLayout L = cta_layout(G, CS, a.max_cand, a.own_max);
  if (L.total > 227 * 1024) {
    set_error("attend needs %d bytes of shared memory per CTA (limit 232448)", L.total);
    return -1;
  }
  auto kern = attend_cta_kernel<G, CS>;
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

template <int G>
int launch_warp(const AttendArgs &args, cudaStream_t stream) {
  AttendArgs a = args;
  const int slice = warp_slice_bytes(G, a.max_cand);
  const int sms = sm_count_cached();
  int wpb = std::min(kWarpKernelMaxWarps, (227 * 1024) / slice);
  // few tiles: spread them over the SMs rather than packing 8 per CTA
  wpb = std::max(1, std::min(wpb, (a.tiles + sms - 1) / sms));
  if (wpb < 1) {
    set_error("attend needs %d bytes of shared memory per warp", slice);
    return -1;
  }
  a.warps_per_block = wpb;
  const int smem = wpb * slice;
  auto kern = attend_warp_kernel<G>;
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

template <int G>
int launch_g(const AttendArgs &a, int kernel, int CS, cudaStream_t stream) {
  if (kernel == 2) return launch_warp<G>(a, stream);
  switch (CS) {
    case 1: return launch_cta<G, 1>(a, stream);
    case 2: return launch_cta<G, 2>(a, stream);
    case 4: return launch_cta<G, 4>(a, stream);
    default: return -2;
  }
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
  for (int i = 0; i <= kMaxLevels; ++i) {
    a.row_off[i] = l.geom.row_off[i];
    a.slots[i] = l.geom.slots[i];
    a.span[i] = l.geom.span[i];
  }
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
  if (kernel == 0) kernel = (a.tiles <= 2 * sms) ? 1 : 2;  // CTA per tile while it fits two waves
  int CS = l.cluster_size;
  if (kernel == 1 && CS == 0) CS = (a.tiles * 4 <= sms) ? 4 : (a.tiles * 2 <= sms) ? 2 : 1;
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
