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
#include "recsa_umma.cuh"

namespace recsa {

// Set by a build or append kernel whose wait on the tensor cores gave up (reported by
// recsa_check_device_errors); the kernel leaves the affected keys unwritten and returns.
__device__ uint32_t g_build_err;

namespace {


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

// A run of rows into L2 (16-byte aligned start, a multiple of 16 bytes).
__device__ __forceinline__ void prefetch_rows_l2(const void *p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
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

__device__ __forceinline__ void store_row4(uint16_t *p, const float x[4]) {
  uint2 o;
  o.x = pack_bf16x2(x[0], x[1]);
  o.y = pack_bf16x2(x[2], x[3]);
  *reinterpret_cast<uint2 *>(p) = o;
}

// The level build with the pooler product on the tensor cores.  One CTA per SM, persistent
// over tiles of 128 nodes (the level's nodes of every (sequence, head), in order).  Warp w
// streams nodes 8w .. 8w+7 of a tile: the children's sums give the value row (stored at
// once) and the key mean, whose three bf16 parts go to row 8w + n of the A operand.  Then
// one thread issues the pooler product into one of two TMEM accumulators (W, the B operand,
// stays in shared memory), and the warps stream the next tile while the tensor cores work.
// The finished accumulator is read back during the next tile (warp w: lanes 32 (w % 4) ..,
// columns 32 (w / 4) ..), rounded to bf16 and stored.  A is single-buffered: a tile's first
// A row is written once the previous tile's product has completed.  Sixteen warps keep 16
// nodes' children (128 KB) in flight per SM.
constexpr int kMmaThreads = 512;
constexpr int kMmaWarps = kMmaThreads / 32;
constexpr int kMmaNodesPerWarp = umma::kM / kMmaWarps;  // 16
constexpr size_t kMmaSmem = 2 * (size_t)umma::kOperandBytes + 128;  // A, B, barriers, TMEM address

template <bool kPaged>
__global__ void __launch_bounds__(kMmaThreads, 1) build_level_mma_kernel(const BuildArgs a) {
  extern __shared__ __align__(128) unsigned char smem_u8[];
  unsigned char *A = smem_u8, *Bop = smem_u8 + umma::kOperandBytes;
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem_u8 + 2 * umma::kOperandBytes);  // product done, by accumulator
  uint32_t *tmem_s = reinterpret_cast<uint32_t *>(bar + 2);
  uint32_t *flag_s = tmem_s + 1;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (warp == 0) {
    umma::tmem_alloc(tmem_s, 2 * umma::kTmemCols);
    umma::tmem_relinquish();
  }
  if (tid == 32) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    mbar_fence_init();
    *flag_s = 0u;
  }
  umma::load_pooler_operand<kMmaThreads>(a.pooler, Bop, tid);
  umma::fence_async_smem();
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();
  const uint32_t tmem = *tmem_s;

  const int64_t total = (int64_t)a.bh * a.nj;
  const int64_t tiles = (total + umma::kM - 1) / umma::kM;
  // node `id` of the launch: (sequence, head), node index, and whether it exists at its
  // sequence's length
  auto locate = [&](int64_t id, int64_t &bhi, int64_t &j, int64_t &length, int64_t &n_prev) -> bool {
    if (id >= total) return false;
    bhi = id / a.nj;
    j = a.j0 + id % a.nj;
    length = a.length;
    n_prev = a.n_prev;
    if (a.seq_len) {  // this sequence's own length: its level has ceil(len / b^l) nodes
      length = min(max(a.seq_len[bhi / a.hkv], (int64_t)0), a.length);
      n_prev = (length + a.span_prev - 1) / a.span_prev;
      return j < (length + a.span - 1) / a.span;
    }
    return true;
  };
  // the accumulator of tile `tile` (buffer buf) -> key rows
  auto epilogue = [&](int64_t tile, int buf) {
    const int rq = warp & 3, cq = warp >> 2;  // lanes 32 rq .., columns 32 cq ..
    const int row = 32 * rq + lane;
    uint32_t v[32];
    umma::tmem_ld32(tmem + (uint32_t)buf * umma::kTmemCols + ((uint32_t)(32 * rq) << 16) + 32u * cq, v);
    umma::tmem_wait_ld();
    int64_t bhi, j, length, n_prev;
    if (locate(tile * umma::kM + row, bhi, j, length, n_prev)) {
      uint4 *dst = reinterpret_cast<uint4 *>(a.dst_k + (a.dst_row_off + bhi * a.dst_slots + j) * kD + 32 * cq);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        dst[q] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                            pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                            pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                            pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
    }
  };

  uint32_t ph[2] = {0u, 0u};
  bool pending[2] = {false, false};  // a product issued on the accumulator and not yet waited for
  bool ok = true;
  int64_t prev = -1;
  int it = 0;
  for (int64_t tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++it) {
    const int buf = it & 1;
    for (int n = 0; n < kMmaNodesPerWarp; ++n) {
      const int row = warp * kMmaNodesPerWarp + n;
      int64_t bhi, j, length, n_prev;
      float ks[4] = {0.f, 0.f, 0.f, 0.f}, vs[4] = {0.f, 0.f, 0.f, 0.f};
      // the warp's next node's children (two contiguous runs, K and V) into L2 while this
      // node's stream: the loads of the next node then wait on L2, not DRAM (a paged token
      // cache scatters them, so it is not prefetched)
      if (!kPaged && lane == 0) {
        int64_t bh2, j2, len2, np2;
        const int64_t nid = n + 1 < kMmaNodesPerWarp ? tile * umma::kM + row + 1
                                                     : (tile + gridDim.x) * umma::kM + warp * kMmaNodesPerWarp;
        if (locate(nid, bh2, j2, len2, np2)) {
          const int64_t c0 = j2 * a.b, cnt = min(c0 + (int64_t)a.b, np2) - c0;
          if (cnt > 0) {
            const int64_t r0 = (a.src_row_off + bh2 * a.src_slots + c0) * kD;
            prefetch_rows_l2(a.src_k + r0, (uint32_t)(cnt * kD * 2));
            prefetch_rows_l2(a.src_v + r0, (uint32_t)(cnt * kD * 2));
          }
        }
      }
      if (locate(tile * umma::kM + row, bhi, j, length, n_prev)) {
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
      if (n == 0 && prev >= 0) {
        // the previous tile's product has read A: its accumulator is read back below
        const int pb = buf ^ 1;
        const bool done = __all_sync(0xffffffffu, mbar_wait(&bar[pb], ph[pb]));  // one answer a warp
        if (!done) {
          ok = false;
          break;
        }
        ph[pb] ^= 1u;
        pending[pb] = false;
        umma::fence_after_sync();
      }
      umma::store_row4_parts(A, row, lane * 4, ks);
    }
    if (!ok && lane == 0) atomicOr(flag_s, 1u);
    __syncthreads();
    if (*flag_s) {
      ok = false;
      break;
    }
    if (prev >= 0) epilogue(prev, buf ^ 1);
    // every row of A written: visible to the tensor cores, then one thread issues the product
    umma::fence_async_smem();
    umma::fence_before_sync();
    __syncthreads();
    if (tid == 0) {
      umma::fence_after_sync();
      umma::issue_pooler(tmem + (uint32_t)buf * umma::kTmemCols, smem_u32(A), smem_u32(Bop));
      umma::commit(&bar[buf]);
    }
    pending[buf] = true;
    prev = tile;
  }
  if (ok && prev >= 0) {
    const int pb = (it - 1) & 1;
    if (__all_sync(0xffffffffu, mbar_wait(&bar[pb], ph[pb]))) {
      ph[pb] ^= 1u;
      pending[pb] = false;
      umma::fence_after_sync();
      epilogue(prev, pb);
    } else {
      ok = false;
    }
  }
  if (!ok && lane == 0) atomicOr(flag_s, 1u);
  __syncthreads();
  if (*flag_s && tid == 0) {
    // a product did not complete within the wait limit: report it, and give the tensor
    // cores a last bounded wait on every product still out before the accumulators are freed
    atomicOr(&g_build_err, kErrTimeout);
    for (int b2 = 0; b2 < 2; ++b2)
      if (pending[b2]) mbar_wait(&bar[b2], ph[b2]);
  }
  umma::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    umma::fence_after_sync();
    umma::tmem_dealloc(tmem, 2 * umma::kTmemCols);
  }
}

// Append and path update in one launch: one CTA per (sequence, KV head).  The CTA copies
// its chunk of new tokens into the token cache, then walks up the levels and rebuilds, at
// each level l, the nodes [j0[l], j1[l]) whose spans meet the new tokens (the nodes above
// them are those nodes' ancestors).  A thread owns one dimension of the key (threads
// 0..127) or of the value (128..255): it sums that dimension over the node's children and
// forms its mean, in the level build's operation order.  The level's key means (up to 128
// nodes at a time) go to an operand and a thread of a warp of its own issues the level
// build's split-bf16 pooler product with the operands' roles exchanged (W as A, the means as
// B, N = the node count rounded up to 16), so the extended tree equals a full build bit for
// bit.  Rows
// written at level l are read at level l+1 by other threads of the same CTA after a
// __syncthreads; no two CTAs touch the same rows.
//
// The walk's critical path is one product a level (48 MMA instructions, ~2.5K cycles).  What
// else is on it is kept short on the path of a single token (one node a level): the node's
// children other than the last are unchanged rows, summed ahead (the next level's while this
// level's product runs), and its last child is the node rebuilt one level below, which the
// thread owning the dimension already holds (key thread d reads accumulator lane d, value
// thread d formed the value); the sum then continues with it in the children's order.
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
// One thread per key dimension and per value dimension, and one more warp that allocates the
// accumulator and issues the pooler product: a thread issuing the product's 48 MMA
// instructions is held for about as long as the product runs (~2.5K cycles, measured), so the
// dimension threads work out the next level's head start meanwhile.
constexpr int kExtendDimThreads = 2 * kD;
constexpr int kExtendThreads = kExtendDimThreads + 32;
constexpr int kExtendIssuer = kExtendDimThreads;  // the issuing thread (lane 0 of the last warp)
// W's and the means' operands of the pooler product, the product's barrier and the TMEM
// address, and per level the rebuilt node range [j0, j1) and the node count of the level below
constexpr size_t kExtendSmem = 2 * (size_t)umma::kOperandBytes + 128 + 3 * (kMaxLevels + 1) * sizeof(int64_t);

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
  extern __shared__ __align__(128) unsigned char smem_u8[];
  unsigned char *Wop = smem_u8, *Mop = smem_u8 + umma::kOperandBytes;  // W's parts, the key means' parts
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem_u8 + 2 * umma::kOperandBytes);
  uint32_t *tmem_s = reinterpret_cast<uint32_t *>(bar + 1);
  int64_t *lv_j0 = reinterpret_cast<int64_t *>(smem_u8 + 2 * umma::kOperandBytes + 128);  // per level: nodes
  int64_t *lv_j1 = lv_j0 + (kMaxLevels + 1);  // [j0, j1) rebuilt, the level below's node count
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
  const int warp = tid >> 5;
  const bool dims = tid < kExtendDimThreads;  // a dimension thread (else the issuing warp)
  if (warp == 0)
    for (int l = tid + 1; l <= t_new; l += 32) {
      lv_j0[l] = l <= t_old ? div_nn(at, a.span[l]) : 0;
      lv_j1[l] = ceil_div_nn(length, a.span[l]);
      lv_np[l] = ceil_div_nn(length, a.span[l - 1]);
    }
  if (tid == 32) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  // token t of this (sequence, head): row tok_base + tok_row(t), -1 for a page outside the pool
  const int64_t h = bhi % a.hkv;
  const int64_t tok_base = kPaged ? (h << a.page_shift) * kD : bhi * a.capacity * kD;
  const PagedRows paged{kPaged ? a.pages + (bhi / a.hkv) * (a.capacity >> a.page_shift) : nullptr,
                        (int64_t)a.hkv << a.page_shift, a.page_shift, a.num_pages};
  auto tok_row = [&](int64_t t) -> int64_t { return kPaged ? paged(t) : t; };
  // level l's rows of this (sequence, head), the thread's half (K or V); level 0 = the tokens
  auto level_rows = [&](int l) -> uint16_t * {
    return l == 0 ? (is_v ? a.v_tok : a.k_tok) + tok_base
                  : (is_v ? a.v_node : a.k_node) + (a.row_off[l] + bhi * a.slots[l]) * kD;
  };
  // The single-token path: a level rebuilds one node whose last child is the one rebuilt
  // below (at level 1: the one new token).  `carry` is that child's dimension d as stored
  // (bf16), valid while `have_carry`.
  float carry = 0.f;
  bool have_carry = false;
  if (dims && a.chunk == 1 && t_new >= 1 && tok_row(at) >= 0) {
    const int64_t s = bhi / a.hkv;
    const uint16_t *src = reinterpret_cast<const uint16_t *>(is_v ? a.v_new : a.k_new);
    carry = bf16_lo(__ldg(src + ((s * a.hkv + h) * kD + d)));
    have_carry = true;
  }
  __syncthreads();  // the level ranges are in place
  // the sum of children [c0, c1) of a node of level l (rows of level l-1, in order), this
  // thread's dim: 16 rows' loads in flight at a time, then their adds in child order (a loop
  // with a run-time trip count would leave a partial node's rows to a rolled remainder loop,
  // one L2 round trip each)
  auto child_sum = [&](int l, int64_t c0, int64_t c1) -> float {
    const uint16_t *src = level_rows(l - 1);
    float sum = 0.f;
    for (int64_t cb = c0; cb < c1; cb += 16) {
      float x[16];
      bool in[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int64_t r = cb + i < c1 ? (l == 1 ? tok_row(cb + i) : cb + i) : -1;
        in[i] = r >= 0;
        x[i] = in[i] ? bf16_lo(src[r * kD + d]) : 0.f;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (in[i]) sum += x[i];
    }
    return sum;
  };
  // The single-token path's head start at level l, worked out while the level below is
  // still in progress: the sum over the node's children before the last, the child count,
  // and for a value the share of a last child that covers fewer tokens than its span (the
  // same terms, in the same order, as for a node summed whole below).
  struct Head {
    float pre, nch, f1, wsum;
    bool part;          // the last child gets the share f1 + 1
    uint16_t *v_dst;    // this thread's element of the node's value row
  };
  auto head_start = [&](int l) -> Head {
    Head hs{0.f, 1.f, 0.f, 1.f, false, nullptr};
    if (!dims || l > t_new || lv_j1[l] - lv_j0[l] != 1) return hs;
    const int64_t j = lv_j0[l], n_prev = lv_np[l];
    const int64_t c0 = j * a.b, c1 = min(c0 + (int64_t)a.b, n_prev);
    hs.pre = child_sum(l, c0, c1 - 1);
    hs.nch = (float)(c1 - c0);
    hs.wsum = hs.nch;
    const int64_t last_tokens = length - (c1 - 1) * a.span[l - 1];
    if (last_tokens < a.span[l - 1]) {
      hs.part = true;
      hs.f1 = (float)last_tokens / (float)a.span[l - 1] - 1.f;
      hs.wsum += hs.f1;
    }
    hs.v_dst = a.v_node + (a.row_off[l] + bhi * a.slots[l] + j) * kD + d;
    return hs;
  };
  if (!dims) {
    // the issuing warp, while the others stage W: every child row the walk reads into L2
    // ahead of the dependent levels (K and V, two 128-byte lines each; level 1 only on the
    // single-token path, a node's token rows), then the accumulator
    const int lane = tid & 31;
    for (int l = 1; l <= t_new; ++l) {
      const int64_t c0 = lv_j0[l] * a.b, c1 = min(lv_j1[l] * a.b, lv_np[l]);
      if (l == 1 && (kPaged || !(a.chunk == 1 && lv_j1[1] - lv_j0[1] == 1))) continue;
      const uint16_t *kb = l == 1 ? a.k_tok + tok_base : a.k_node + (a.row_off[l - 1] + bhi * a.slots[l - 1]) * kD;
      const uint16_t *vb = l == 1 ? a.v_tok + tok_base : a.v_node + (a.row_off[l - 1] + bhi * a.slots[l - 1]) * kD;
      for (int64_t e = lane; e < (c1 - c0) * 4; e += 32)
        prefetch_l2(((e & 2) ? vb : kb) + (c0 + (e >> 2)) * kD + (e & 1) * (kD / 2));
    }
    umma::tmem_alloc(tmem_s, umma::kTmemCols);
    umma::tmem_relinquish();
  } else {
    umma::load_pooler_operand<kExtendDimThreads, 16>(a.pooler, Wop, tid);  // W's three parts
    const int64_t s = bhi / a.hkv;
    for (int64_t e = tid; e < (int64_t)a.chunk * 16; e += kExtendDimThreads) {  // 16 pieces a row
      const int64_t src = ((s * a.chunk + (e >> 4)) * a.hkv + h) * 16 + (e & 15);
      const int64_t row = tok_row(at + (e >> 4));
      if (row < 0) continue;
      const int64_t dst = (tok_base + row * kD) / 8 + (e & 15);  // in 16-byte pieces
      reinterpret_cast<uint4 *>(a.k_tok)[dst] = __ldg(a.k_new + src);
      reinterpret_cast<uint4 *>(a.v_tok)[dst] = __ldg(a.v_new + src);
    }
  }
  umma::fence_async_smem();
  umma::fence_before_sync();
  __syncthreads();  // W and the TMEM address are in place, and the appended rows are read
                    // below by other threads
  umma::fence_after_sync();
  const uint32_t tmem = *tmem_s;
  uint32_t ph = 0u;
  bool ok = true;
  Head hs = head_start(1);  // level 1's (the token rows before the new one)

  for (int l = 1; l <= t_new && ok; ++l) {
    const int64_t span_prev = a.span[l - 1];
    const int64_t n_prev = lv_np[l], j0 = lv_j0[l], j1 = lv_j1[l];
    const uint16_t *src = level_rows(l - 1);
    uint16_t *dk = a.k_node + (a.row_off[l] + bhi * a.slots[l]) * kD;
    uint16_t *dv = a.v_node + (a.row_off[l] + bhi * a.slots[l]) * kD;
    // one node whose last child the thread holds: the head start plus that child
    const bool single = have_carry && j1 - j0 == 1;
    for (int64_t g0 = j0; g0 < j1 && ok; g0 += umma::kM) {  // up to 128 nodes a product
      const int64_t g1 = min(j1, g0 + (int64_t)umma::kM);
      const int cnt = (int)(g1 - g0);
      // the key mean's three bf16 parts into row m of the means' operand
      auto put_key_mean = [&](int m, float mean) {
        uint32_t p0, p1, p2;
        umma::split3(mean, p0, p1, p2);
        const int off = umma::operand_offset(m, d);
        *reinterpret_cast<uint16_t *>(Mop + off) = (uint16_t)p0;
        *reinterpret_cast<uint16_t *>(Mop + umma::kPartBytes + off) = (uint16_t)p1;
        *reinterpret_cast<uint16_t *>(Mop + 2 * umma::kPartBytes + off) = (uint16_t)p2;
      };
      if (!dims) {
      } else if (single) {
        float sum = hs.pre + carry;
        if (is_v) {
          if (hs.part) sum = __fmaf_rn(hs.f1, carry, sum);
          const uint32_t vbits = f32_to_bf16_bits(sum / hs.wsum);
          *hs.v_dst = (uint16_t)vbits;
          carry = bf16_lo(vbits);  // the value as stored: the next level's last child
        } else {
          put_key_mean(0, sum / hs.nch);
        }
      } else {
        for (int64_t j = g0; j < g1; ++j) {
          const int64_t c0 = j * a.b, c1 = min(c0 + (int64_t)a.b, n_prev);
          float sum = child_sum(l, c0, c1);
          const float nch = (float)(c1 - c0);
          if (is_v) {  // token-weighted: the level's last child gets its share tokens / span_prev
            float wsum = nch;
            if (c1 == n_prev && c1 > c0) {
              const int64_t last_tokens = length - (c1 - 1) * span_prev;
              if (last_tokens < span_prev) {
                const float f1 = (float)last_tokens / (float)span_prev - 1.f;
                const int64_t r = l == 1 ? tok_row(c1 - 1) : c1 - 1;
                sum = __fmaf_rn(f1, r >= 0 ? bf16_lo(src[r * kD + d]) : 0.f, sum);
                wsum += f1;
              }
            }
            const uint32_t vbits = f32_to_bf16_bits(sum / wsum);
            dv[j * kD + d] = (uint16_t)vbits;
            carry = bf16_lo(vbits);
          } else {
            put_key_mean((int)(j - g0), sum / nch);
          }
        }
      }
      umma::fence_async_smem();
      umma::fence_before_sync();
      __syncthreads();  // the key means in place
      if (tid == kExtendIssuer) {
        umma::fence_after_sync();
        umma::issue_pooler_t(tmem, smem_u32(Wop), smem_u32(Mop), (cnt + 15) & ~15);
        umma::commit(bar);
      }
      // the next level's head start while the tensor cores work (with one node rebuilt here,
      // its children before the last are rows this launch does not change)
      if (j1 - j0 == 1) hs = head_start(l + 1);
      const bool done = __all_sync(0xffffffffu, mbar_wait(bar, ph));  // one answer a warp
      ph ^= 1u;
      umma::fence_after_sync();
      if (done && warp < 4) {
        // keys of nodes g0 .. g1-1: key thread d reads accumulator lane d (warp w, lanes
        // 32w ..), one column a node; a warp stores 64 contiguous bytes of each row
        uint32_t v[32];
        if (cnt == 1) {  // one node: column 0, kept as the next level's last child
          umma::tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16), v);
          umma::tmem_wait_ld();
          const uint32_t kbits = f32_to_bf16_bits(__uint_as_float(v[0]));
          dk[g0 * kD + d] = (uint16_t)kbits;
          carry = bf16_lo(kbits);
        } else {
          for (int cb = 0; cb < cnt; cb += 32) {
            umma::tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)cb, v);
            umma::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (cb + i < cnt) dk[(g0 + cb + i) * kD + d] = (uint16_t)f32_to_bf16_bits(__uint_as_float(v[i]));
          }
        }
      }
      // the accumulator is read and these rows are written before the next product is
      // issued and the next level reads them (the product has read the means' operand)
      umma::fence_before_sync();
      if (!__syncthreads_and(done)) {
        // the product did not complete within the wait limit: report it; the walk stops
        if (tid == kExtendIssuer) {
          if (a.err) atomicOr(a.err, kErrTimeout);
          atomicOr(&g_build_err, kErrTimeout);
          mbar_wait(bar, ph ^ 1u);  // a last bounded wait before the accumulator is freed
        }
        ok = false;
      }
    }
    have_carry = j1 - j0 == 1;  // the node rebuilt here is the next level's last child
  }
  umma::fence_before_sync();
  __syncthreads();
  if (warp == kExtendIssuer / 32) {
    umma::fence_after_sync();
    umma::tmem_dealloc(tmem, umma::kTmemCols);
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
  e = cudaFuncSetAttribute(build_level_mma_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kMmaSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(build_level_mma_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kMmaSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(extend_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kExtendSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(extend_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kExtendSmem);
  if (e != cudaSuccess) return (int)e;
  configured_device = dev;
  return 0;
}

}  // namespace

int read_build_errors(uint32_t *bits) {
  uint32_t v = 0u, zero = 0u;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_build_err, sizeof(v));
  if (e == cudaSuccess && v != 0u) e = cudaMemcpyToSymbol(g_build_err, &zero, sizeof(zero));
  *bits = v;
  return (int)e;
}

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
  // tiles of 128 nodes over a persistent grid of one CTA per SM; the paged instance reads
  // level 1 through the page table
  const int64_t tiles = ceil_div((int64_t)a.bh * a.nj, (int64_t)umma::kM);
  const int64_t grid = std::min<int64_t>(tiles, (int64_t)sm_count());
  auto kern = a.pages ? build_level_mma_kernel<true> : build_level_mma_kernel<false>;
  kern<<<(unsigned)grid, kMmaThreads, kMmaSmem, (cudaStream_t)stream>>>(a);
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
