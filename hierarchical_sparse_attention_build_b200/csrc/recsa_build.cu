// Tree build (one level per launch), append with path update (all levels in one launch),
// chunk append and RoPE table kernels.
//
// Recursive Sparse Attention, abstract: every node summarises its subtree with one
// key, made by a per-layer pooler shared by all levels, and one mean-pooled value.
// Here a parent key is W @ (mean of the children's stored pre-RoPE keys) and a parent
// value is the token-count-weighted mean of the children's values (the subtree mean);
// both are rounded to bf16 when stored and the next level reads the stored rows.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "recsa_device.cuh"
#include "recsa_internal.h"

namespace recsa {
namespace {

constexpr int kBuildThreads = 256;
constexpr int kBuildWarps = kBuildThreads / 32;
// Nodes per warp: 8 for a whole level; 1 for small launches (a prefill or decode step
// extends one node per level and head), so their nodes run side by side, not in turn.
constexpr int kNodesPerWarp = 8;
constexpr int kFewNodes = 1;
__host__ __device__ constexpr size_t build_smem(int npw) {
  return (size_t)(kD * kD + kBuildWarps * npw * kD) * sizeof(float);
}

struct BuildArgs {
  const uint16_t *src_k;  // level l-1 rows (token cache or node arena)
  const uint16_t *src_v;
  int64_t src_row_off;    // arena row offset of level l-1 (0 for tokens)
  int64_t src_slots;      // rows per (sequence, head) block at level l-1
  uint16_t *dst_k;
  uint16_t *dst_v;
  int64_t dst_row_off;
  int64_t dst_slots;
  int64_t n_prev;         // valid rows of level l-1 at this length
  int64_t span_prev;      // tokens under a level l-1 node (b^(l-1))
  int64_t length;
  int64_t j0, nj;         // nodes [j0, j0 + nj) of level l, for every (sequence, head)
  int32_t b;
  int32_t bh;             // batch * Hkv
  int32_t hkv;
  int64_t span;           // tokens under a level l node (b^l)
  const int64_t *seq_len; // per-sequence lengths (NULL: every sequence has `length`)
  const int32_t *pages;   // level 1 over a paged token cache: the page table (else NULL)
  int64_t pages_per_seq;
  int32_t page_shift, num_pages;
  const float *pooler;    // [128][128] row-major W
};

// Rows of one (sequence, head) of the level below, relative to its base: contiguous...
struct PlainRows {
  static constexpr bool kPaged = false;
  __device__ __forceinline__ int64_t operator()(int64_t c) const { return c; }
};
// ...or token rows of a paged cache, base = head h's rows of page 0 (pages are
// Hkv * page_size rows apart); -1 for a page outside the pool (the row is skipped).
struct PagedRows {
  static constexpr bool kPaged = true;
  const int32_t *pages;  // this sequence's page table
  int64_t stride;        // Hkv << shift
  int shift, num_pages;
  __device__ __forceinline__ int64_t operator()(int64_t c) const {
    const int pg = __ldg(pages + (c >> shift));
    if ((unsigned)pg >= (unsigned)num_pages) return -1;
    return (int64_t)pg * stride + (c & ((int64_t(1) << shift) - 1));
  }
};

// Wt[k][o] = W[o][k] into shared memory.  A thread moves 16-byte pieces of W; the 32 lanes of
// a warp take 32 consecutive rows o at the same column, so each shared-memory store fills 32
// banks, and a thread's pieces are all loaded before any is stored.
template <int NT>
__device__ __forceinline__ void load_wt(const float *__restrict__ W, float *Wt, int tid) {
  constexpr int kPieces = kD * kD / 4 / NT;
  static_assert(kD * kD / 4 % NT == 0, "threads must divide the pooler's 16-byte pieces");
  float4 w[kPieces];
#pragma unroll
  for (int i = 0; i < kPieces; ++i) {
    const int e = tid + i * NT;  // piece e: row o = e % 128, columns 4 * (e / 128) .. +3
    w[i] = __ldg(reinterpret_cast<const float4 *>(W) + (e & (kD - 1)) * (kD / 4) + (e >> 7));
  }
#pragma unroll
  for (int i = 0; i < kPieces; ++i) {
    const int e = tid + i * NT;
    const int o = e & (kD - 1), k = (e >> 7) * 4;
    Wt[(k + 0) * kD + o] = w[i].x;
    Wt[(k + 1) * kD + o] = w[i].y;
    Wt[(k + 2) * kD + o] = w[i].z;
    Wt[(k + 3) * kD + o] = w[i].w;
  }
}

// One child row piece (the lane's 4 dims): through the read-only path for a level written by
// an earlier launch, an ordinary load for one this kernel may have written.
template <bool kReadOnly>
__device__ __forceinline__ uint2 ld_child(const uint16_t *p) {
  if constexpr (kReadOnly)
    return __ldg(reinterpret_cast<const uint2 *>(p));
  else
    return *reinterpret_cast<const uint2 *>(p);
}

// The lane's 4 dims of node means over children [c0, c1) of level l-1 (kb, vb point at the
// lane's dims of the (sequence, head) block's first row).  Key: plain mean of the children's
// stored keys.  Value: token-count-weighted mean; every child but the level's last covers
// span_prev tokens, so the children are summed with weight 1 and the last child, if it covers
// fewer tokens, then gets its share f = tokens / span_prev.
template <bool kReadOnly, class Rows>
__device__ __forceinline__ void node_means(const uint16_t *kb, const uint16_t *vb, int64_t c0, int64_t c1,
                                           int64_t n_prev, int64_t length, int64_t span_prev, float ks[4],
                                           float vs[4], const Rows &rows) {
  float2 ks2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};  // dims (0,1), (2,3) of the lane's 4
  float2 vs2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll 16  // a whole node's children (b = 16) in flight at once
  for (int64_t c = c0; c < c1; ++c) {
    const int64_t r = rows(c);
    if (Rows::kPaged && r < 0) continue;
    const uint2 ku = ld_child<kReadOnly>(kb + r * kD);
    const uint2 vu = ld_child<kReadOnly>(vb + r * kD);
    ks2[0] = __fadd2_rn(ks2[0], make_float2(bf16_lo(ku.x), bf16_hi(ku.x)));
    ks2[1] = __fadd2_rn(ks2[1], make_float2(bf16_lo(ku.y), bf16_hi(ku.y)));
    vs2[0] = __fadd2_rn(vs2[0], make_float2(bf16_lo(vu.x), bf16_hi(vu.x)));
    vs2[1] = __fadd2_rn(vs2[1], make_float2(bf16_lo(vu.y), bf16_hi(vu.y)));
  }
  ks[0] = ks2[0].x, ks[1] = ks2[0].y, ks[2] = ks2[1].x, ks[3] = ks2[1].y;
  vs[0] = vs2[0].x, vs[1] = vs2[0].y, vs[2] = vs2[1].x, vs[3] = vs2[1].y;
  const float nch = (float)(c1 - c0);
  float wsum = nch;
  if (c1 == n_prev && c1 > c0) {
    const int64_t last_tokens = length - (c1 - 1) * span_prev;
    if (last_tokens < span_prev) {
      const float f1 = (float)last_tokens / (float)span_prev - 1.f;
      const int64_t r = rows(c1 - 1);
      const uint2 vu = (Rows::kPaged && r < 0) ? make_uint2(0u, 0u) : ld_child<kReadOnly>(vb + r * kD);
      vs[0] = __fmaf_rn(f1, bf16_lo(vu.x), vs[0]);
      vs[1] = __fmaf_rn(f1, bf16_hi(vu.x), vs[1]);
      vs[2] = __fmaf_rn(f1, bf16_lo(vu.y), vs[2]);
      vs[3] = __fmaf_rn(f1, bf16_hi(vu.y), vs[3]);
      wsum += f1;
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    ks[i] = ks[i] / nch;
    vs[i] = vs[i] / wsum;
  }
}

// key = W @ mean for NPW nodes whose key means are rows [NPW][128] in shared memory; lane
// owns outputs 4*lane .. 4*lane+3, as the pairs (4l, 4l+1) and (4l+2, 4l+3) of packed fp32
// FMAs (each output's terms in k order).
template <int NPW>
__device__ __forceinline__ void apply_w(const float *Wt, const float *mean_rows, int lane, float acc[NPW][4]) {
  float2 acc2[NPW][2];
#pragma unroll
  for (int n = 0; n < NPW; ++n) acc2[n][0] = acc2[n][1] = make_float2(0.f, 0.f);
  const float4 *Wt4 = reinterpret_cast<const float4 *>(Wt);
  const float4 *M4 = reinterpret_cast<const float4 *>(mean_rows);
#pragma unroll 2
  for (int k = 0; k < kD; k += 4) {
    float2 w[4][2];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float4 wt = Wt4[(k + t) * 32 + lane];
      w[t][0] = make_float2(wt.x, wt.y);
      w[t][1] = make_float2(wt.z, wt.w);
    }
#pragma unroll
    for (int n = 0; n < NPW; ++n) {
      const float4 m = M4[n * 32 + (k >> 2)];
      const float mt[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 mm = make_float2(mt[t], mt[t]);
        acc2[n][0] = __ffma2_rn(mm, w[t][0], acc2[n][0]);
        acc2[n][1] = __ffma2_rn(mm, w[t][1], acc2[n][1]);
      }
    }
  }
#pragma unroll
  for (int n = 0; n < NPW; ++n) {
    acc[n][0] = acc2[n][0].x;
    acc[n][1] = acc2[n][0].y;
    acc[n][2] = acc2[n][1].x;
    acc[n][3] = acc2[n][1].y;
  }
}

__device__ __forceinline__ void store_row4(uint16_t *p, const float x[4]) {
  uint2 o;
  o.x = pack_bf16x2(x[0], x[1]);
  o.y = pack_bf16x2(x[2], x[3]);
  *reinterpret_cast<uint2 *>(p) = o;
}

// One CTA handles blocks of 8 * NPW nodes: each warp streams the children of NPW nodes
// (lane = 4 consecutive dims, one 256-byte row per warp load), forms the child means in
// fp32, writes the value rows, then applies W to its own key means (W^T resident in shared
// memory).  Warps share only W^T, so they never wait for one another after it is loaded.
template <int NPW, bool kPaged>
__global__ void __launch_bounds__(kBuildThreads, 2) build_level_kernel(const BuildArgs a) {
  constexpr int kNodesPerBlock = kBuildWarps * NPW;
  extern __shared__ __align__(16) float smem_f[];
  float *Wt = smem_f;               // Wt[k][o] = W[o][k]
  float *Mean = smem_f + kD * kD;   // [8 * NPW][128] key means
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  load_wt<kBuildThreads>(a.pooler, Wt, tid);
  __syncthreads();

  const int64_t total = (int64_t)a.bh * a.nj;
  for (int64_t base = (int64_t)blockIdx.x * kNodesPerBlock; base < total;
       base += (int64_t)gridDim.x * kNodesPerBlock) {
    bool live[NPW];
    for (int t = 0; t < NPW; ++t) {
      const int nl = warp * NPW + t;
      const int64_t id = base + nl;
      float ks[4] = {0.f, 0.f, 0.f, 0.f}, vs[4] = {0.f, 0.f, 0.f, 0.f};
      live[t] = id < total;
      if (live[t]) {
        const int64_t bhi = id / a.nj;
        const int64_t j = a.j0 + id % a.nj;
        int64_t length = a.length, n_prev = a.n_prev;
        if (a.seq_len) {  // this sequence's own length: its level has ceil(len / b^l) nodes
          length = min(max(a.seq_len[bhi / a.hkv], (int64_t)0), a.length);
          n_prev = (length + a.span_prev - 1) / a.span_prev;
          live[t] = j < (length + a.span - 1) / a.span;
        }
        if (live[t]) {
          const int64_t c0 = j * a.b;
          const int64_t c1 = min(c0 + (int64_t)a.b, n_prev);
          if (kPaged) {  // level 1 over a paged token cache
            const int64_t h = bhi % a.hkv;
            const PagedRows rows{a.pages + (bhi / a.hkv) * a.pages_per_seq, (int64_t)a.hkv << a.page_shift,
                                 a.page_shift, a.num_pages};
            const uint16_t *kb = a.src_k + (h << a.page_shift) * kD + lane * 4;
            const uint16_t *vb = a.src_v + (h << a.page_shift) * kD + lane * 4;
            node_means<true>(kb, vb, c0, c1, n_prev, length, a.span_prev, ks, vs, rows);
          } else {
            const uint16_t *kb = a.src_k + (a.src_row_off + bhi * a.src_slots) * kD + lane * 4;
            const uint16_t *vb = a.src_v + (a.src_row_off + bhi * a.src_slots) * kD + lane * 4;
            node_means<true>(kb, vb, c0, c1, n_prev, length, a.span_prev, ks, vs, PlainRows{});
          }
          store_row4(a.dst_v + (a.dst_row_off + bhi * a.dst_slots + j) * kD + lane * 4, vs);
        }
      }
      *reinterpret_cast<float4 *>(Mean + nl * kD + lane * 4) = make_float4(ks[0], ks[1], ks[2], ks[3]);
    }
    __syncwarp();  // a warp applies W to its own nodes only: warps run out of step, so some
                   // stream children while others compute
    float acc[NPW][4];
    apply_w<NPW>(Wt, Mean + warp * NPW * kD, lane, acc);
#pragma unroll
    for (int n = 0; n < NPW; ++n) {
      const int64_t id = base + warp * NPW + n;
      if (live[n]) {
        const int64_t bhi = id / a.nj;
        const int64_t j = a.j0 + id % a.nj;
        store_row4(a.dst_k + (a.dst_row_off + bhi * a.dst_slots + j) * kD + lane * 4, acc[n]);
      }
    }
    __syncwarp();  // this warp's Mean rows are rewritten next
  }
}

// Append and path update in one launch: one CTA per (sequence, KV head).  The CTA copies
// its chunk of new tokens into the token cache, then walks up the levels and rebuilds, at
// each level l, the nodes [j0[l], j1[l]) whose spans meet the new tokens (the nodes above
// them are those nodes' ancestors).  A thread owns one dimension of the key (threads
// 0..127) or of the value (128..255): it sums that dimension over the node's children and
// forms its mean.  The key output o = W[o] . mean is one fp32 FMA chain over k = 0..127: the
// key thread of dimension o runs k < 64 and the value thread of the same o continues with
// k >= 64, each with its half of W row o in registers.  Per element these are the level
// build's operations in the level build's order, so the extended tree equals a full build
// bit for bit.  Rows written at level l are read at level l+1 by other threads of the same
// CTA after a __syncthreads; no two CTAs touch the same rows.
struct ExtendArgs {
  const uint4 *k_new, *v_new;   // [B][C][Hkv][128] bf16, as 16-byte pieces
  uint16_t *k_tok, *v_tok;      // [B][Hkv][capacity][128]
  uint16_t *k_node, *v_node;    // node arena
  const float *pooler;
  const int64_t *seq_len;       // per-sequence lengths before the append (NULL: all `at`)
  const int32_t *pages;         // paged token cache: the page table (NULL: contiguous)
  int32_t page_shift, num_pages;
  uint32_t *err;                // optional error word: a sequence without room is flagged
  int64_t capacity;
  int64_t at;                   // first new slot (the length before the append; the longest one)
  int32_t chunk, hkv, b, levels;  // levels = T(at + chunk)
  int64_t row_off[kMaxLevels + 1];
  int64_t slots[kMaxLevels + 1];
  int64_t span[kMaxLevels + 1];
};
constexpr int kExtendThreads = 2 * kD;  // one thread per key dimension and per value dimension
constexpr int kHalfK = kD / 2;          // W columns held by each thread of a dimension
// W^T staged as Wt[k][o ^ (k / 4 % 32)]: the coalesced row loads (a warp reads one W row)
// and the per-thread row reads both hit 32 distinct banks.
// W^T staging, the key mean, the first half of the key, and per level the rebuilt node range
// [j0, j1) and the node count of the level below
constexpr size_t kExtendSmem = (size_t)(kD * kD + 2 * kD) * sizeof(float) + 3 * (kMaxLevels + 1) * sizeof(int64_t);

// x / y and ceil(x / y) for x >= 0, y >= 1, in 32 bits whenever the operands fit (a 64-bit
// division is a long instruction sequence; lengths and spans of real trees fit 32 bits).
__device__ __forceinline__ int64_t div_nn(int64_t x, int64_t y) {
  if (y > x) return 0;
  if (x <= 0xffffffffLL) return (int64_t)((uint32_t)x / (uint32_t)y);
  return x / y;
}
__device__ __forceinline__ int64_t ceil_div_nn(int64_t x, int64_t y) { return x > 0 ? div_nn(x - 1, y) + 1 : 0; }

__device__ __forceinline__ void prefetch_l2(const void *p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

template <bool kPaged>
__global__ void __launch_bounds__(kExtendThreads, 1) extend_kernel(const ExtendArgs a) {
  extern __shared__ __align__(16) float smem_f[];
  float *Wt = smem_f;               // swizzled W^T (staging only)
  float *mean = smem_f + kD * kD;   // the node's key mean
  float *part = mean + kD;          // key outputs after k < 64
  int64_t *lv_j0 = reinterpret_cast<int64_t *>(part + kD);  // per level: nodes [j0, j1) rebuilt,
  int64_t *lv_j1 = lv_j0 + (kMaxLevels + 1);                 // the level below's node count
  int64_t *lv_np = lv_j1 + (kMaxLevels + 1);
  const int tid = threadIdx.x;
  const int64_t bhi = blockIdx.x;   // (sequence, head)
  const int d = tid & (kD - 1);
  const bool is_v = tid >= kD;
  // this sequence's length before (at) and after (length) the append, and its levels
  int64_t at = a.at;
  if (a.seq_len) {  // a sequence outside [0, at] (no room for the chunk) is left as it is
    at = a.seq_len[bhi / a.hkv];
    if (at < 0 || at > a.at) {
      if (a.err && tid == 0) atomicOr(a.err, kErrIndex);
      return;  // the whole CTA: every thread reads the same length
    }
  }
  const int64_t length = at + a.chunk;
  int t_old = 0, t_new = 0;  // T(n) = #{l >= 1 : b^l < n}
  while (t_new < a.levels && a.span[t_new + 1] < length) ++t_new;
  while (t_old < t_new && a.span[t_old + 1] < at) ++t_old;
  // level l rebuilds nodes [j0, j1): those whose spans meet the new tokens (a level that
  // becomes new is built whole); the first warp works the levels out side by side, once,
  // rather than every thread on the walk's dependent path
  if (tid < 32)
    for (int l = tid + 1; l <= t_new; l += 32) {
      lv_j0[l] = l <= t_old ? div_nn(at, a.span[l]) : 0;
      lv_j1[l] = ceil_div_nn(length, a.span[l]);
      lv_np[l] = ceil_div_nn(length, a.span[l - 1]);
    }
  // token t of this (sequence, head): row tok_base + tok_row(t), -1 for a page outside the pool
  const int64_t h = bhi % a.hkv;
  const int64_t tok_base = kPaged ? (h << a.page_shift) * kD : bhi * a.capacity * kD;
  const PagedRows paged{kPaged ? a.pages + (bhi / a.hkv) * (a.capacity >> a.page_shift) : nullptr,
                        (int64_t)a.hkv << a.page_shift, a.page_shift, a.num_pages};
  auto tok_row = [&](int64_t t) -> int64_t { return kPaged ? paged(t) : t; };

  // W in flight (a warp reads one 512-byte row) while the tokens are appended and the first
  // children load
  constexpr int kPieces = kD * kD / 4 / kExtendThreads;
  float4 w[kPieces];
#pragma unroll
  for (int i = 0; i < kPieces; ++i) w[i] = __ldg(reinterpret_cast<const float4 *>(a.pooler) + tid + i * kExtendThreads);
  {
    const int64_t s = bhi / a.hkv;
    for (int64_t e = tid; e < (int64_t)a.chunk * 16; e += kExtendThreads) {  // 16 pieces a row
      const int64_t src = ((s * a.chunk + (e >> 4)) * a.hkv + h) * 16 + (e & 15);
      const int64_t row = tok_row(at + (e >> 4));
      if (row < 0) continue;
      const int64_t dst = (tok_base + row * kD) / 8 + (e & 15);  // in 16-byte pieces
      reinterpret_cast<uint4 *>(a.k_tok)[dst] = __ldg(a.k_new + src);
      reinterpret_cast<uint4 *>(a.v_tok)[dst] = __ldg(a.v_new + src);
    }
  }
  __syncthreads();  // the level ranges are in place, and the appended rows are read below by other threads
  // every child row the walk reads above level 1, into L2 ahead of the dependent levels
  // (K and V, two 128-byte lines each)
  for (int l = 2; l <= t_new; ++l) {
    const int64_t c0 = lv_j0[l] * a.b, c1 = min(lv_j1[l] * a.b, lv_np[l]);
    const int64_t base = (a.row_off[l - 1] + bhi * a.slots[l - 1]) * kD;
    for (int64_t e = tid; e < (c1 - c0) * 4; e += kExtendThreads)
      prefetch_l2(((e & 2) ? a.v_node : a.k_node) + base + (c0 + (e >> 2)) * kD + (e & 1) * (kD / 2));
  }

  float wr[kHalfK];  // W[d][64 * is_v + i]
  bool w_ready = false;
  const int kbase = is_v ? kHalfK : 0;
  for (int l = 1; l <= t_new; ++l) {
    const int64_t span_prev = a.span[l - 1];
    const int64_t n_prev = lv_np[l], j0 = lv_j0[l], j1 = lv_j1[l];
    const uint16_t *src = l == 1 ? (is_v ? a.v_tok : a.k_tok) + tok_base
                                 : (is_v ? a.v_node : a.k_node) + (a.row_off[l - 1] + bhi * a.slots[l - 1]) * kD;
    uint16_t *dk = a.k_node + (a.row_off[l] + bhi * a.slots[l]) * kD;
    uint16_t *dv = a.v_node + (a.row_off[l] + bhi * a.slots[l]) * kD;
    for (int64_t j = j0; j < j1; ++j) {
      const int64_t c0 = j * a.b, c1 = min(c0 + (int64_t)a.b, n_prev);
      // the level below's row of child c (tokens through the page table when paged)
      auto child = [&](int64_t c) -> int64_t { return l == 1 ? tok_row(c) : c; };
      float sum = 0.f;
#pragma unroll 16
      for (int64_t c = c0; c < c1; ++c) {
        const int64_t r = child(c);
        if (r >= 0) sum += bf16_lo(src[r * kD + d]);
      }
      const float nch = (float)(c1 - c0);
      if (is_v) {  // token-weighted: the level's last child gets its share tokens / span_prev
        float wsum = nch;
        if (c1 == n_prev && c1 > c0) {
          const int64_t last_tokens = length - (c1 - 1) * span_prev;
          if (last_tokens < span_prev) {
            const float f1 = (float)last_tokens / (float)span_prev - 1.f;
            const int64_t r = child(c1 - 1);
            sum = __fmaf_rn(f1, r >= 0 ? bf16_lo(src[r * kD + d]) : 0.f, sum);
            wsum += f1;
          }
        }
        dv[j * kD + d] = (uint16_t)f32_to_bf16_bits(sum / wsum);
      } else {
        mean[d] = sum / nch;
      }
      if (!w_ready) {  // first node: W^T through shared memory into each thread's registers
#pragma unroll
        for (int i = 0; i < kPieces; ++i) {
          const int e = tid + i * kExtendThreads;
          const int o = e >> 5, q = e & 31;  // W[o][4q .. 4q+3]
          Wt[(4 * q + 0) * kD + (o ^ q)] = w[i].x;
          Wt[(4 * q + 1) * kD + (o ^ q)] = w[i].y;
          Wt[(4 * q + 2) * kD + (o ^ q)] = w[i].z;
          Wt[(4 * q + 3) * kD + (o ^ q)] = w[i].w;
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < kHalfK; ++i) {
          const int k = kbase + i;
          wr[i] = Wt[k * kD + (d ^ ((k >> 2) & 31))];
        }
        w_ready = true;
      }
      __syncthreads();  // the key mean in place
      const float4 *m4 = reinterpret_cast<const float4 *>(mean + kbase);
      float acc = 0.f;
      if (!is_v) {
#pragma unroll
        for (int i = 0; i < kHalfK / 4; ++i) {
          const float4 m = m4[i];
          acc = __fmaf_rn(m.x, wr[4 * i + 0], acc);
          acc = __fmaf_rn(m.y, wr[4 * i + 1], acc);
          acc = __fmaf_rn(m.z, wr[4 * i + 2], acc);
          acc = __fmaf_rn(m.w, wr[4 * i + 3], acc);
        }
        part[d] = acc;
      }
      __syncthreads();  // the first half of every key output in place
      if (is_v) {
        acc = part[d];
#pragma unroll
        for (int i = 0; i < kHalfK / 4; ++i) {
          const float4 m = m4[i];
          acc = __fmaf_rn(m.x, wr[4 * i + 0], acc);
          acc = __fmaf_rn(m.y, wr[4 * i + 1], acc);
          acc = __fmaf_rn(m.z, wr[4 * i + 2], acc);
          acc = __fmaf_rn(m.w, wr[4 * i + 3], acc);
        }
        dk[j * kD + d] = (uint16_t)f32_to_bf16_bits(acc);
      }
      __syncthreads();  // mean and part are rewritten next, and the next level reads these rows
    }
  }
}

// k_new / v_new [B][C][Hkv][128] -> token caches [B][Hkv][capacity][128] at slot `at + i`.
// With a page table the slot is row (at + i) % page_size of head h in page
// pages[b][(at + i) / page_size]; a page outside the pool is skipped.
__global__ void append_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new, uint16_t *k_tok,
                              uint16_t *v_tok, int64_t capacity, int64_t at, int chunk, int hkv, int64_t rows,
                              const int32_t *pages, int page_shift, int num_pages) {
  const int64_t n16 = rows * 16;  // 16-byte pieces
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n16; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = e >> 4;
    const int part = (int)(e & 15);
    const int h = (int)(row % hkv);
    const int64_t bi_i = row / hkv;
    const int64_t i = bi_i % chunk;
    const int64_t bi = bi_i / chunk;
    int64_t dst;
    if (pages) {
      const int64_t t = at + i;
      const int pg = __ldg(pages + bi * (capacity >> page_shift) + (t >> page_shift));
      if ((unsigned)pg >= (unsigned)num_pages) continue;
      dst = ((((int64_t)pg * hkv + h) << page_shift) + (t & ((int64_t(1) << page_shift) - 1))) * kD + part * 8;
    } else {
      dst = ((bi * hkv + h) * capacity + at + i) * kD + part * 8;
    }
    reinterpret_cast<uint4 *>(k_tok + dst)[0] = k_new[e];
    reinterpret_cast<uint4 *>(v_tok + dst)[0] = v_new[e];
  }
}

// RoPE table, computed in fp64 and stored fp32: for position pos and frequency pair u
// (frequencies 2u, 2u+1, angle pos * base^(-2i/128)) the four floats
// table[pos][u] = (cos_2u, cos_2u+1, sin_2u, sin_2u+1), so a pair of frequencies loads
// as packed (cos, cos') and (sin, sin') operands.
__global__ void rope_table_kernel(float *table, int rows, double base, WsHeader *hdr) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx < rows * kHalf) {
    const int pos = idx / kHalf, i = idx % kHalf;
    const double inv_freq = pow(base, -2.0 * (double)i / (double)kD);
    double s, c;
    sincos((double)pos * inv_freq, &s, &c);
    float *pair = table + (size_t)pos * (2 * kHalf) + (i >> 1) * 4 + (i & 1);
    pair[0] = (float)c;
    pair[2] = (float)s;
  }
  if (idx == 0) {
    hdr->err = 0u;
    hdr->table_rows = rows;
    hdr->rope_base = (float)base;
    __threadfence();
    hdr->magic = kWsMagic;
  }
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

// Dynamic shared memory above 48 KB is opted into once per device and host thread.
int configure_smem() {
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return (int)e;
  if (configured_device == dev) return 0;
  e = cudaFuncSetAttribute(build_level_kernel<kNodesPerWarp, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)build_smem(kNodesPerWarp));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(build_level_kernel<kFewNodes, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)build_smem(kFewNodes));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(build_level_kernel<kNodesPerWarp, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)build_smem(kNodesPerWarp));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(build_level_kernel<kFewNodes, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)build_smem(kFewNodes));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(extend_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kExtendSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(extend_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kExtendSmem);
  if (e != cudaSuccess) return (int)e;
  configured_device = dev;
  return 0;
}

}  // namespace

int launch_rope_table(void *ws, int rows, double base, void *stream) {
  auto *hdr = reinterpret_cast<WsHeader *>(ws);
  auto *table = reinterpret_cast<float *>(reinterpret_cast<char *>(ws) + kWsHeader);
  const int n = rows * kHalf;
  const int threads = 256;
  const int blocks = (n + threads - 1) / threads;
  rope_table_kernel<<<blocks, threads, 0, (cudaStream_t)stream>>>(table, rows, base, hdr);
  return (int)cudaGetLastError();
}

int launch_build_level(const TreeGeom &g, const recsa_tree &t, int level, int64_t length, int64_t j0, int64_t j1,
                       void *stream) {
  if (j1 <= j0) return 0;
  BuildArgs a;
  const bool from_tokens = level == 1;
  a.src_k = reinterpret_cast<const uint16_t *>(from_tokens ? t.k_tok : t.k_node);
  a.src_v = reinterpret_cast<const uint16_t *>(from_tokens ? t.v_tok : t.v_node);
  a.src_row_off = from_tokens ? 0 : g.row_off[level - 1];
  a.src_slots = g.slots[level - 1];
  a.dst_k = reinterpret_cast<uint16_t *>(t.k_node);
  a.dst_v = reinterpret_cast<uint16_t *>(t.v_node);
  a.dst_row_off = g.row_off[level];
  a.dst_slots = g.slots[level];
  a.span_prev = g.span[level - 1];
  a.n_prev = ceil_div(length, a.span_prev);
  a.length = length;
  a.j0 = j0;
  a.nj = j1 - j0;
  a.b = g.b;
  a.bh = g.batch * g.hkv;
  a.hkv = g.hkv;
  a.span = g.span[level];
  a.seq_len = t.seq_len;
  a.pages = from_tokens ? t.page_table : nullptr;
  a.page_shift = t.page_table ? __builtin_ctz((unsigned)t.page_size) : 0;
  a.pages_per_seq = t.page_table ? g.capacity >> a.page_shift : 0;
  a.num_pages = t.page_table ? t.num_pages : 0;
  a.pooler = t.pooler;
  const int rc = configure_smem();
  if (rc != 0) return rc;
  const int64_t nodes = (int64_t)a.bh * a.nj;
  const int64_t full_grid = (int64_t)sm_count() * 2;
  // one pass of warps with a node each when it fits, else 8 nodes a warp over a grid of 2 CTAs
  // per SM; the paged instances read level 1 through the page table
  const bool few = nodes <= full_grid * kBuildWarps * kFewNodes;
  const int npw = few ? kFewNodes : kNodesPerWarp;
  const int64_t grid = few ? ceil_div(nodes, kBuildWarps * kFewNodes)
                           : std::min<int64_t>(ceil_div(nodes, kBuildWarps * kNodesPerWarp), full_grid);
  auto kern = few ? (a.pages ? build_level_kernel<kFewNodes, true> : build_level_kernel<kFewNodes, false>)
                  : (a.pages ? build_level_kernel<kNodesPerWarp, true> : build_level_kernel<kNodesPerWarp, false>);
  kern<<<(unsigned)grid, kBuildThreads, build_smem(npw), (cudaStream_t)stream>>>(a);
  return (int)cudaGetLastError();
}

int launch_extend(const TreeGeom &g, const recsa_tree &t, const void *k_new, const void *v_new, int64_t at,
                  int chunk, int levels, void *stream, uint32_t *err) {
  ExtendArgs a;
  a.err = err;
  a.k_new = reinterpret_cast<const uint4 *>(k_new);
  a.v_new = reinterpret_cast<const uint4 *>(v_new);
  a.k_tok = reinterpret_cast<uint16_t *>(t.k_tok);
  a.v_tok = reinterpret_cast<uint16_t *>(t.v_tok);
  a.k_node = reinterpret_cast<uint16_t *>(t.k_node);
  a.v_node = reinterpret_cast<uint16_t *>(t.v_node);
  a.pooler = t.pooler;
  a.seq_len = t.seq_len;
  a.pages = t.page_table;
  a.page_shift = t.page_table ? __builtin_ctz((unsigned)t.page_size) : 0;
  a.num_pages = t.page_table ? t.num_pages : 0;
  a.capacity = g.capacity;
  a.at = at;
  a.chunk = chunk;
  a.hkv = g.hkv;
  a.b = g.b;
  a.levels = levels;
  for (int l = 0; l <= kMaxLevels; ++l) {
    a.row_off[l] = g.row_off[l];
    a.slots[l] = g.slots[l];
    a.span[l] = g.span[l];
  }
  const int rc = configure_smem();
  if (rc != 0) return rc;
  const int64_t grid = (int64_t)g.batch * g.hkv;
  auto kern = a.pages ? extend_kernel<true> : extend_kernel<false>;
  kern<<<(unsigned)grid, kExtendThreads, kExtendSmem, (cudaStream_t)stream>>>(a);
  return (int)cudaGetLastError();
}

// seq_len[s] += count, held to `limit` (a sequence the append skipped stays where it was).
__global__ void advance_lengths_kernel(int64_t *seq_len, int batch, int64_t count, int64_t limit) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < batch && seq_len[i] >= 0 && seq_len[i] + count <= limit) seq_len[i] += count;
}

int launch_advance_lengths(int64_t *seq_len, int batch, int64_t count, int64_t limit, void *stream) {
  const int threads = 128;
  advance_lengths_kernel<<<(batch + threads - 1) / threads, threads, 0, (cudaStream_t)stream>>>(seq_len, batch, count,
                                                                                               limit);
  return (int)cudaGetLastError();
}

int launch_append(const TreeGeom &g, const recsa_tree &t, const void *k_new, const void *v_new, int64_t at,
                  int chunk, void *stream) {
  const int64_t rows = (int64_t)g.batch * chunk * g.hkv;
  const int64_t n16 = rows * 16;
  const int threads = 256;
  const int64_t grid = std::min<int64_t>(ceil_div(n16, threads), (int64_t)sm_count() * 8);
  append_kernel<<<(unsigned)grid, threads, 0, (cudaStream_t)stream>>>(
      reinterpret_cast<const uint4 *>(k_new), reinterpret_cast<const uint4 *>(v_new),
      reinterpret_cast<uint16_t *>(t.k_tok), reinterpret_cast<uint16_t *>(t.v_tok), g.capacity, at, chunk, g.hkv,
      rows, t.page_table, t.page_table ? __builtin_ctz((unsigned)t.page_size) : 0, t.page_table ? t.num_pages : 0);
  return (int)cudaGetLastError();
}

}  // namespace recsa
