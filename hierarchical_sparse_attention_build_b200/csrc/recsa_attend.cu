// Fused level-wise sparse attend (decode and causal prefill).
//
// Recursive Sparse Attention, abstract: each level above the tokens keeps at most k
// candidates, so a query reads O(log L) entries; the summaries of the candidates it
// does not keep share one softmax with the exact tokens; every entry is RoPE-rotated
// at its index among the candidates of its level.
//
// One tile = one (sequence, query, KV group) and is processed by a cluster of CS
// CTAs (CS = 1, 2 or 4).  Every CTA holds the same candidate list of the current
// level in shared memory and scores its own contiguous slice of it:
//   1. rotate the G query heads at position n (the level's candidate count);
//   2. gather the slice's 256-byte bf16 key rows with bulk (TMA) copies into shared
//      memory, rotate each at its candidate index and score it against the G heads;
//      the group score S (sum over heads) goes to every CTA of the cluster (DSMEM);
//   3. after a cluster barrier every CTA computes the same top-k (S descending,
//      lower index first) and the same next candidate list (children of the kept
//      nodes, plus the forced partial node in causal mode), in node order;
//   4. each CTA gathers the value rows of its unselected candidates and folds them
//      into per-warp fp32 online-softmax states;
// and at the token level every candidate is scored and folded.  The per-warp states
// are merged in the CTA, then across the cluster, and the output row is written.
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "recsa_device.cuh"
#include "recsa_internal.h"

namespace cg = cooperative_groups;

namespace recsa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr uint32_t kForced = 0x80000000u;  // candidate is a forced partial node
constexpr uint32_t kKept = 0x40000000u;    // candidate kept by top-k
constexpr uint32_t kNodeMask = 0x3fffffffu;

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
  int32_t max_cand;  // candidate buffer rows (multiple of 32)
  int32_t own_max;   // logits buffer rows per CTA
  int32_t chunk;     // rows per gather pass
  float scale;
};

struct Layout {
  int bar, misc, q, qrot, cand, skey, rank, slog, kbuf, vbuf, red, clm, total;
};

__host__ __device__ inline int align128(int x) { return (x + 127) & ~127; }

__host__ __device__ inline Layout make_layout(int G, int CS, int max_cand, int own_max, int chunk) {
  Layout L;
  int o = 0;
  auto take = [&o](int bytes) {
    int r = o;
    o = align128(o + bytes);
    return r;
  };
  L.bar = take(64);
  L.misc = take(64);
  L.q = take(G * kD * 4);
  L.qrot = take(G * kD * 4);
  L.cand = take(2 * max_cand * 4);
  L.skey = take((CS > 1 ? 2 : 1) * max_cand * 4);
  L.rank = take(max_cand * 4 + 64);
  L.slog = take(G * own_max * 4);
  L.kbuf = take(chunk * kRowBytes);
  L.vbuf = take(chunk * kRowBytes);
  const int red_bytes = kWarps * G * (kD + 2) * 4;
  if (2 * chunk * kRowBytes >= red_bytes)
    L.red = L.kbuf;  // the merge runs after the last gather
  else
    L.red = take(red_bytes);
  L.clm = CS > 1 ? take(CS * G * (kD + 2) * 4) : 0;
  L.total = o;
  return L;
}

__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Sum of 8 lanes (lane bits 0..2) of G per-head partials; afterwards the lane holds
// the full sum of head (j >> (3 - log2 G)).
template <int G>
__device__ __forceinline__ float reduce8(const float (&v)[G], int j) {
  if constexpr (G == 1) {
    float x = v[0];
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x;
  } else if constexpr (G == 2) {
    const bool b2 = j & 4;
    float x = (b2 ? v[1] : v[0]) + __shfl_xor_sync(0xffffffffu, b2 ? v[0] : v[1], 4);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x;
  } else if constexpr (G == 4) {
    const bool b2 = j & 4, b1 = j & 2;
    const float k0 = (b2 ? v[2] : v[0]) + __shfl_xor_sync(0xffffffffu, b2 ? v[0] : v[2], 4);
    const float k1 = (b2 ? v[3] : v[1]) + __shfl_xor_sync(0xffffffffu, b2 ? v[1] : v[3], 4);
    float x = (b1 ? k1 : k0) + __shfl_xor_sync(0xffffffffu, b1 ? k0 : k1, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x;
  } else {
    static_assert(G == 8, "G must be 1, 2, 4 or 8");
    const bool b2 = j & 4, b1 = j & 2, b0 = j & 1;
    float k[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) k[i] = (b2 ? v[i + 4] : v[i]) + __shfl_xor_sync(0xffffffffu, b2 ? v[i] : v[i + 4], 4);
    const float m0 = (b1 ? k[2] : k[0]) + __shfl_xor_sync(0xffffffffu, b1 ? k[0] : k[2], 2);
    const float m1 = (b1 ? k[3] : k[1]) + __shfl_xor_sync(0xffffffffu, b1 ? k[1] : k[3], 2);
    return (b0 ? m1 : m0) + __shfl_xor_sync(0xffffffffu, b0 ? m0 : m1, 1);
  }
}

template <int G>
__host__ __device__ constexpr int log2g() {
  return G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : 3;
}

// Exclusive scan of arr[0..n) in place (all threads of the block call it); returns the total.
__device__ int block_exclusive_scan(int *arr, int n, int *wsum) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int carry = 0;
  for (int base = 0; base < n; base += kThreads) {
    const int i = base + tid;
    const int v = i < n ? arr[i] : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = lane < kWarps ? wsum[lane] : 0;
#pragma unroll
      for (int o = 1; o < kWarps; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      if (lane < kWarps) wsum[lane] = w;
    }
    __syncthreads();
    const int before = warp ? wsum[warp - 1] : 0;
    if (i < n) arr[i] = carry + before + x - v;
    const int tile_total = wsum[kWarps - 1];
    __syncthreads();
    carry += tile_total;
  }
  return carry;
}

template <int G, int CS>
__global__ void __launch_bounds__(kThreads, 1) attend_kernel(const AttendArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const Layout Ls = make_layout(G, CS, a.max_cand, a.own_max, a.chunk);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Ls.bar);  // [0] keys, [1] values
  int *misc = reinterpret_cast<int *>(smem + Ls.misc);           // [0..1] candidate counts, [2] bad ws
  float *qraw = reinterpret_cast<float *>(smem + Ls.q);
  float *qrot = reinterpret_cast<float *>(smem + Ls.qrot);
  uint32_t *cand = reinterpret_cast<uint32_t *>(smem + Ls.cand);
  uint32_t *skey = reinterpret_cast<uint32_t *>(smem + Ls.skey);
  int *rank = reinterpret_cast<int *>(smem + Ls.rank);
  int *wsum = rank + a.max_cand;
  float *slog = reinterpret_cast<float *>(smem + Ls.slog);
  uint16_t *kbuf = reinterpret_cast<uint16_t *>(smem + Ls.kbuf);
  uint16_t *vbuf = reinterpret_cast<uint16_t *>(smem + Ls.vbuf);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j8 = lane & 7;  // lane within an 8-lane row group
  int crank = 0;
  if constexpr (CS > 1) crank = (int)cg::this_cluster().block_rank();
  const int tile = blockIdx.x / CS;
  const int qi = tile % a.nq;
  const int sg = tile / a.nq;
  const int g = sg % a.hkv;
  const int s = sg / a.hkv;
  const int64_t p = a.causal ? a.length + qi : a.length;
  const int64_t bh = (int64_t)s * a.hkv + g;
  uint32_t *err = &a.hdr->err;

  // levels above the tokens visible to this query
  int T = 0;
  {
    int64_t n = p;
    while (n > a.b) {
      n = (n + a.b - 1) / a.b;
      ++T;
    }
  }

  // The workspace must hold an initialised RoPE table for this call.
  if (tid == 0) {
    const uint32_t magic = a.hdr->magic;
    const int rows = a.hdr->table_rows;
    misc[2] = (magic != kWsMagic || rows < a.table_rows_needed) ? 1 : 0;
    if (misc[2]) atomicOr(err, kErrWs);
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  float *out_f = reinterpret_cast<float *>(a.out);
  uint16_t *out_h = reinterpret_cast<uint16_t *>(a.out);
  const int64_t out_row0 = (((int64_t)s * a.nq + qi) * a.hq + (int64_t)g * G) * kD;
  if (misc[2]) {  // identical decision in every CTA of the cluster: exit before any cluster barrier
    if (crank == 0)
      for (int e = tid; e < G * kD; e += kThreads) {
        if (a.out_fp32) out_f[out_row0 + e] = 0.f;
        else out_h[out_row0 + e] = 0;
      }
    return;
  }

  // query rows of the group (pre-RoPE) -> fp32
  {
    const uint16_t *qg = a.q + (((int64_t)s * a.nq + qi) * a.hq + (int64_t)g * G) * kD;
    for (int e = tid; e < G * kD / 2; e += kThreads) {
      const uint32_t u = reinterpret_cast<const uint32_t *>(qg)[e];
      qraw[2 * e] = bf16_lo(u);
      qraw[2 * e + 1] = bf16_hi(u);
    }
  }
  // top-level candidates
  int n;
  {
    if (T == 0) {
      n = (int)p;
      for (int i = tid; i < n; i += kThreads) cand[i] = (uint32_t)i;
    } else if (!a.causal) {
      n = (int)((a.length + a.span[T] - 1) / a.span[T]);
      for (int i = tid; i < n; i += kThreads) cand[i] = (uint32_t)i;
    } else {
      const int full = (int)(p / a.span[T]);
      const bool part = (p % a.span[T]) != 0;
      n = full + (part ? 1 : 0);
      for (int i = tid; i < n; i += kThreads) cand[i] = (uint32_t)i | ((part && i == full) ? kForced : 0u);
    }
  }
  if constexpr (CS > 1) cluster_barrier();  // peers are running before any DSMEM store
  __syncthreads();

  // per-warp online softmax state: lane owns dims 4*lane .. 4*lane+3 of every head
  float m_w[G], l_w[G], acc[G][4];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m_w[h] = -INFINITY;
    l_w[h] = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[h][i] = 0.f;
  }
  uint32_t kphase = 0, vphase = 0;
  int keys_read = 0, values_read = 0;
  int cur = 0;

  // Fold the entries of own rows [c0, c0 + cn) whose values sit in vbuf rows 0..cn-1.
  // `is_entry(i)` says whether row i is an entry; logits live at slog[h][c0 - lo + i].
  auto fold = [&](int c0, int cn, int lo, auto is_entry) {
    float mx[G];
#pragma unroll
    for (int h = 0; h < G; ++h) mx[h] = -INFINITY;
    for (int r = lane; r * kWarps + warp < cn; r += 32) {
      const int i = r * kWarps + warp;
      if (is_entry(i)) {
#pragma unroll
        for (int h = 0; h < G; ++h) mx[h] = fmaxf(mx[h], slog[h * a.own_max + c0 - lo + i]);
      }
    }
    float mnew[G], alpha[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      mx[h] = warp_max(mx[h]);
      mnew[h] = fmaxf(m_w[h], mx[h]);
      alpha[h] = (mnew[h] == -INFINITY) ? 1.f : expf(m_w[h] - mnew[h]);
    }
    float ls[G];
#pragma unroll
    for (int h = 0; h < G; ++h) ls[h] = 0.f;
    for (int r = lane; r * kWarps + warp < cn; r += 32) {
      const int i = r * kWarps + warp;
      if (is_entry(i)) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float *sl = &slog[h * a.own_max + c0 - lo + i];
          const float pr = expf(*sl - mnew[h]);
          *sl = pr;
          ls[h] += pr;
        }
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      l_w[h] = l_w[h] * alpha[h] + warp_sum(ls[h]);
      m_w[h] = mnew[h];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[h][i] *= alpha[h];
    }
    __syncwarp();
    for (int i = warp; i < cn; i += kWarps) {
      if (!is_entry(i)) continue;
      const uint2 vu = *reinterpret_cast<const uint2 *>(vbuf + i * kD + lane * 4);
      const float v0 = bf16_lo(vu.x), v1 = bf16_hi(vu.x), v2 = bf16_lo(vu.y), v3 = bf16_hi(vu.y);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float pr = slog[h * a.own_max + c0 - lo + i];
        acc[h][0] = fmaf(pr, v0, acc[h][0]);
        acc[h][1] = fmaf(pr, v1, acc[h][1]);
        acc[h][2] = fmaf(pr, v2, acc[h][2]);
        acc[h][3] = fmaf(pr, v3, acc[h][3]);
      }
    }
  };

  for (int lvl = T; lvl >= 0; --lvl) {
    uint32_t *cl = cand + cur * a.max_cand;
    uint32_t *sk = skey + ((CS > 1) ? (lvl & 1) * a.max_cand : 0);
    if (n > a.table_rows_needed - 1) {  // cannot happen for a valid launch; guards the table read
      if (tid == 0) atomicOr(err, kErrCount);
      n = a.table_rows_needed - 1;
    }
    // 1. query heads rotated at position n (the level's candidate count)
    for (int e = tid; e < G * kHalf; e += kThreads) {
      const int h = e / kHalf, i = e % kHalf;
      const float2 cs = __ldg(&a.table[(int64_t)n * kHalf + i]);
      const float lo = qraw[h * kD + i], hi = qraw[h * kD + i + kHalf];
      qrot[h * kD + i] = lo * cs.x - hi * cs.y;
      qrot[h * kD + i + kHalf] = hi * cs.x + lo * cs.y;
    }
    __syncthreads();
    float qlo[G][8], qhi[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float4 *r = reinterpret_cast<const float4 *>(qrot + h * kD);
      const float4 x0 = r[2 * j8], x1 = r[2 * j8 + 1], y0 = r[16 + 2 * j8], y1 = r[16 + 2 * j8 + 1];
      qlo[h][0] = x0.x; qlo[h][1] = x0.y; qlo[h][2] = x0.z; qlo[h][3] = x0.w;
      qlo[h][4] = x1.x; qlo[h][5] = x1.y; qlo[h][6] = x1.z; qlo[h][7] = x1.w;
      qhi[h][0] = y0.x; qhi[h][1] = y0.y; qhi[h][2] = y0.z; qhi[h][3] = y0.w;
      qhi[h][4] = y1.x; qhi[h][5] = y1.y; qhi[h][6] = y1.z; qhi[h][7] = y1.w;
    }
    const int per = (n + CS - 1) / CS;
    const int lo_r = min(n, crank * per);
    const int hi_r = min(n, lo_r + per);
    const uint16_t *kbase = (lvl == 0) ? a.k_tok + bh * a.cap * kD : a.k_node + (a.row_off[lvl] + bh * a.slots[lvl]) * kD;
    const uint16_t *vbase = (lvl == 0) ? a.v_tok + bh * a.cap * kD : a.v_node + (a.row_off[lvl] + bh * a.slots[lvl]) * kD;
    const int64_t nrows = (lvl == 0) ? a.cap : a.slots[lvl];

    // 2. score own slice, chunk by chunk (and fold it at the token level)
    for (int c0 = lo_r; c0 < hi_r; c0 += a.chunk) {
      const int cn = min(a.chunk, hi_r - c0);
      if (warp == 0) {
        int cnt = 0;
        for (int i = lane; i < cn; i += 32) {
          const uint32_t c = cl[c0 + i];
          if (!(c & kForced) && (int64_t)(c & kNodeMask) < nrows) cnt += (lvl == 0) ? 2 : 1;
        }
        cnt = warp_sum_int(cnt);
        fence_proxy_async();
        if (lane == 0) mbar_arrive_expect_tx(&bars[0], (uint32_t)cnt * kRowBytes);
        __syncwarp();
        for (int i = lane; i < cn; i += 32) {
          const uint32_t c = cl[c0 + i];
          if (c & kForced) continue;
          const int64_t node = c & kNodeMask;
          if (node >= nrows) {
            atomicOr(err, kErrIndex);
            continue;
          }
          bulk_g2s(kbuf + i * kD, kbase + node * kD, kRowBytes, &bars[0]);
          if (lvl == 0) bulk_g2s(vbuf + i * kD, vbase + node * kD, kRowBytes, &bars[0]);
        }
      }
      mbar_wait(&bars[0], kphase, err);
      kphase ^= 1u;
      for (int i0 = 0; i0 < cn; i0 += 32) {
        const int i = i0 + warp * 4 + (lane >> 3);
        const bool valid = i < cn;
        const uint32_t c = valid ? cl[c0 + i] : kForced;
        const bool scorable = valid && !(c & kForced);
        float part[G];
#pragma unroll
        for (int h = 0; h < G; ++h) part[h] = 0.f;
        if (scorable) {
          const int pos = c0 + i;  // RoPE position = rank among the level's candidates
          const uint4 klo = *reinterpret_cast<const uint4 *>(kbuf + i * kD + 8 * j8);
          const uint4 khi = *reinterpret_cast<const uint4 *>(kbuf + i * kD + kHalf + 8 * j8);
          const float4 *tb = reinterpret_cast<const float4 *>(a.table + (int64_t)pos * kHalf + 8 * j8);
          const float4 t0 = __ldg(tb), t1 = __ldg(tb + 1), t2 = __ldg(tb + 2), t3 = __ldg(tb + 3);
          const float cs_c[8] = {t0.x, t0.z, t1.x, t1.z, t2.x, t2.z, t3.x, t3.z};
          const float cs_s[8] = {t0.y, t0.w, t1.y, t1.w, t2.y, t2.w, t3.y, t3.w};
          const uint32_t lw[4] = {klo.x, klo.y, klo.z, klo.w};
          const uint32_t hw[4] = {khi.x, khi.y, khi.z, khi.w};
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const float xl = (t & 1) ? bf16_hi(lw[t >> 1]) : bf16_lo(lw[t >> 1]);
            const float xh = (t & 1) ? bf16_hi(hw[t >> 1]) : bf16_lo(hw[t >> 1]);
            const float rl = xl * cs_c[t] - xh * cs_s[t];
            const float rh = xh * cs_c[t] + xl * cs_s[t];
#pragma unroll
            for (int h = 0; h < G; ++h) part[h] = fmaf(qlo[h][t], rl, fmaf(qhi[h][t], rh, part[h]));
          }
        }
        float x = reduce8<G>(part, j8) * a.scale;  // logit of head hsel
        const int hsel = j8 >> (3 - log2g<G>());
        float S = x;
#pragma unroll
        for (int st = 0, o = 4; st < log2g<G>(); ++st, o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
        if (scorable) {
          if ((j8 & ((1 << (3 - log2g<G>())) - 1)) == 0) slog[hsel * a.own_max + (c0 - lo_r) + i] = x;
          if (lvl > 0 && j8 == 0) {
            const uint32_t key = order_key(S);
            const int pos = c0 + i;
            if constexpr (CS > 1) {
              cg::cluster_group cluster = cg::this_cluster();
#pragma unroll
              for (int r = 0; r < CS; ++r) cluster.map_shared_rank(sk, r)[pos] = key;
            } else {
              sk[pos] = key;
            }
          }
        }
      }
      __syncthreads();
      if (lvl == 0) {
        fold(c0, cn, lo_r, [&](int i) { return true; });
        __syncthreads();
      }
    }
    if (lvl == 0) {
      keys_read += n;
      values_read += n;
      break;
    }
    if constexpr (CS > 1) cluster_barrier();
    __syncthreads();

    // 3. top-k over the whole level (same in every CTA)
    int nforced = 0;
    if (a.causal && n > 0 && (cl[n - 1] & kForced)) nforced = 1;  // only the trailing node can be partial
    const int m = n - nforced;
    const bool keep_all = a.top_k >= m;
    if (!keep_all) {
      for (int c = tid; c < n; c += kThreads) rank[c] = 0;
      __syncthreads();
      const int nseg = (m + 63) / 64;
      const int items = n * nseg;
      for (int it = tid; it < items; it += kThreads) {
        const int c = it % n, seg = it / n;
        if (cl[c] & kForced) continue;
        const uint32_t kc = sk[c];
        const int e0 = seg * 64, e1 = min(m, e0 + 64);
        int cntb = 0;
        for (int e = e0; e < e1; ++e) {
          const uint32_t ke = sk[e];
          cntb += (ke > kc || (ke == kc && e < c)) ? 1 : 0;
        }
        if (cntb) atomicAdd(&rank[c], cntb);
      }
      __syncthreads();
    }
    for (int c = tid; c < n; c += kThreads) {
      const uint32_t v = cl[c];
      if (!(v & kForced) && (keep_all || rank[c] < a.top_k)) cl[c] = v | kKept;
    }
    __syncthreads();
    keys_read += m;
    values_read += m - min(a.top_k, m);

    // 4. fold own unselected candidates
    for (int c0 = lo_r; c0 < hi_r; c0 += a.chunk) {
      const int cn = min(a.chunk, hi_r - c0);
      if (warp == 0) {
        int cnt = 0;
        for (int i = lane; i < cn; i += 32) {
          const uint32_t c = cl[c0 + i];
          if (!(c & (kForced | kKept)) && (int64_t)(c & kNodeMask) < nrows) ++cnt;
        }
        cnt = warp_sum_int(cnt);
        fence_proxy_async();
        if (lane == 0) mbar_arrive_expect_tx(&bars[1], (uint32_t)cnt * kRowBytes);
        __syncwarp();
        for (int i = lane; i < cn; i += 32) {
          const uint32_t c = cl[c0 + i];
          if (c & (kForced | kKept)) continue;
          const int64_t node = c & kNodeMask;
          if (node >= nrows) continue;
          bulk_g2s(vbuf + i * kD, vbase + node * kD, kRowBytes, &bars[1]);
        }
      }
      mbar_wait(&bars[1], vphase, err);
      vphase ^= 1u;
      fold(c0, cn, lo_r, [&](int i) { return !(cl[c0 + i] & (kForced | kKept)); });
      __syncthreads();
    }

    // 5. next level's candidates: children of kept (and forced) nodes, in node order
    const int64_t span_below = a.span[lvl - 1];
    const int64_t n_below = a.causal ? 0 : (a.length + span_below - 1) / span_below;
    for (int c = tid; c < n; c += kThreads) {
      const uint32_t v = cl[c];
      int nch = 0;
      if (v & (kKept | kForced)) {
        const int64_t node = v & kNodeMask;
        if (!a.causal) {
          nch = (int)min((int64_t)a.b, n_below - node * a.b);
        } else if (v & kForced) {
          const int64_t first = node * a.b;  // first child; visible children start before p
          nch = (int)min((int64_t)a.b, (p - first * span_below + span_below - 1) / span_below);
        } else {
          nch = a.b;
        }
        nch = max(nch, 0);
      }
      rank[c] = nch;
    }
    __syncthreads();
    int total = block_exclusive_scan(rank, n, wsum);
    uint32_t *nx = cand + (cur ^ 1) * a.max_cand;
    for (int c = tid; c < n; c += kThreads) {
      const uint32_t v = cl[c];
      if (!(v & (kKept | kForced))) continue;
      const int64_t node = v & kNodeMask;
      const int off = rank[c];
      const int nch = (c + 1 < n ? rank[c + 1] : total) - off;
      for (int t = 0; t < nch; ++t) {
        if (off + t >= a.max_cand) {
          atomicOr(err, kErrCount);
          break;
        }
        const int64_t child = node * a.b + t;
        const bool fc = a.causal && (v & kForced) && t == nch - 1 && (child + 1) * span_below > p;
        nx[off + t] = (uint32_t)child | (fc ? kForced : 0u);
      }
    }
    if (a.sel_idx != nullptr && crank == 0 && lvl <= a.sel_levels) {
      // kept nodes of this level in ascending order (positions are in node order)
      int32_t *dst = a.sel_idx + ((int64_t)tile * a.sel_levels + (lvl - 1)) * a.top_k;
      __syncthreads();
      for (int c = tid; c < n; c += kThreads) rank[c] = (cl[c] & kKept) ? 1 : 0;
      __syncthreads();
      const int nk = block_exclusive_scan(rank, n, wsum);
      for (int c = tid; c < n; c += kThreads)
        if ((cl[c] & kKept) && rank[c] < a.top_k) dst[rank[c]] = (int32_t)(cl[c] & kNodeMask);
      for (int t = nk + tid; t < a.top_k; t += kThreads) dst[t] = -1;
    }
    if (total > a.max_cand) total = a.max_cand;
    n = total;
    cur ^= 1;
    __syncthreads();
  }

  if (a.entries != nullptr && crank == 0 && tid == 0) {
    a.entries[2 * (int64_t)tile] = keys_read;
    a.entries[2 * (int64_t)tile + 1] = values_read;
  }

  // merge the per-warp states in the CTA
  float *red = reinterpret_cast<float *>(smem + Ls.red);  // [warp][h][130]: m, l, acc[128]
  __syncthreads();
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float *r = red + (warp * G + h) * (kD + 2);
    if (lane == 0) {
      r[0] = m_w[h];
      r[1] = l_w[h];
    }
    *reinterpret_cast<float2 *>(r + 2 + lane * 4) = make_float2(acc[h][0], acc[h][1]);
    *reinterpret_cast<float2 *>(r + 4 + lane * 4) = make_float2(acc[h][2], acc[h][3]);
  }
  __syncthreads();
  float *clm = reinterpret_cast<float *>(smem + Ls.clm);  // [rank][h][130] on cluster rank 0
  for (int e = tid; e < G * kD; e += kThreads) {
    const int h = e / kD, d = e % kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red[(w * G + h) * (kD + 2)]);
    float l = 0.f, o = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float *r = red + (w * G + h) * (kD + 2);
        const float f = (r[0] == -INFINITY) ? 0.f : expf(r[0] - M);
        l += f * r[1];
        o += f * r[2 + d];
      }
    }
    if constexpr (CS == 1) {
      const float y = l > 0.f ? o / l : 0.f;
      if (a.out_fp32) out_f[out_row0 + e] = y;
      else out_h[out_row0 + e] = (uint16_t)f32_to_bf16_bits(y);
    } else {
      cg::cluster_group cluster = cg::this_cluster();
      float *dst = cluster.map_shared_rank(clm, 0) + (crank * G + h) * (kD + 2);
      if (d == 0) {
        dst[0] = M;
        dst[1] = l;
      }
      dst[2 + d] = o;
    }
  }
  if constexpr (CS > 1) {
    cluster_barrier();
    if (crank == 0) {
      for (int e = tid; e < G * kD; e += kThreads) {
        const int h = e / kD, d = e % kD;
        float M = -INFINITY;
#pragma unroll
        for (int r = 0; r < CS; ++r) M = fmaxf(M, clm[(r * G + h) * (kD + 2)]);
        float l = 0.f, o = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int r = 0; r < CS; ++r) {
            const float *x = clm + (r * G + h) * (kD + 2);
            const float f = (x[0] == -INFINITY) ? 0.f : expf(x[0] - M);
            l += f * x[1];
            o += f * x[2 + d];
          }
        }
        const float y = l > 0.f ? o / l : 0.f;
        if (a.out_fp32) out_f[out_row0 + e] = y;
        else out_h[out_row0 + e] = (uint16_t)f32_to_bf16_bits(y);
      }
    }
  }
}

template <int G, int CS>
int launch_one(const AttendArgs &args, int tiles, const Layout &L, cudaStream_t stream) {
  auto kern = attend_kernel<G, CS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
  if (e != cudaSuccess) return (int)e;
  if constexpr (CS == 1) {
    kern<<<tiles, kThreads, L.total, stream>>>(args);
    return (int)cudaGetLastError();
  } else {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles * CS));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)L.total;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, args);
    if (e != cudaSuccess) return (int)e;
    return (int)cudaGetLastError();
  }
}

template <int G>
int launch_g(const AttendArgs &args, int tiles, int CS, int max_cand, cudaStream_t stream, int *smem_out) {
  int own = ((max_cand + CS - 1) / CS + 31) / 32 * 32;
  int chunk = std::min(own, 128);
  AttendArgs a2 = args;
  a2.own_max = own;
  a2.chunk = chunk;
  const Layout L = make_layout(G, CS, max_cand, own, chunk);
  *smem_out = L.total;
  if (L.total > 227 * 1024) return -1;
  switch (CS) {
    case 1: return launch_one<G, 1>(a2, tiles, L, stream);
    case 2: return launch_one<G, 2>(a2, tiles, L, stream);
    case 4: return launch_one<G, 4>(a2, tiles, L, stream);
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
  const int tiles = l.geom.batch * l.geom.hkv * l.num_queries;
  int CS = l.cluster_size;
  if (CS == 0) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    CS = (tiles * 4 <= sms) ? 4 : (tiles * 2 <= sms) ? 2 : 1;
  }
  int smem = 0;
  int rc;
  switch (l.group) {
    case 1: rc = launch_g<1>(a, tiles, CS, l.max_cand, (cudaStream_t)stream, &smem); break;
    case 2: rc = launch_g<2>(a, tiles, CS, l.max_cand, (cudaStream_t)stream, &smem); break;
    case 4: rc = launch_g<4>(a, tiles, CS, l.max_cand, (cudaStream_t)stream, &smem); break;
    case 8: rc = launch_g<8>(a, tiles, CS, l.max_cand, (cudaStream_t)stream, &smem); break;
    default: rc = -2;
  }
  if (rc == -1) set_error("attend needs %d bytes of shared memory (limit 232448)", smem);
  if (rc == -2) set_error("unsupported group size %d or cluster size %d", l.group, CS);
  return rc;
}

}  // namespace recsa
