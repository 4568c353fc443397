// Tree build (one level per launch), chunk append and RoPE table kernels.
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
  const float *pooler;    // [128][128] row-major W
};

// One CTA handles blocks of 64 nodes: each warp streams the children of 8 nodes
// (lane = 4 consecutive dims, one 256-byte row per warp load), forms the child
// means in fp32, writes the value rows, then applies W to its own 8 key means (W^T
// resident in shared memory, 8 nodes x 4 outputs per lane).  Warps share only W^T, so
// they never wait for one another after it is loaded.
template <int NPW>
__global__ void __launch_bounds__(kBuildThreads, 2) build_level_kernel(const BuildArgs a) {
  constexpr int kNodesPerBlock = kBuildWarps * NPW;
  extern __shared__ __align__(16) float smem_f[];
  float *Wt = smem_f;               // Wt[k][o] = W[o][k]
  float *Mean = smem_f + kD * kD;   // [64][128] key means
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  for (int e = tid; e < kD * kD; e += kBuildThreads) {
    const int o = e >> 7, k = e & 127;
    Wt[k * kD + o] = a.pooler[e];
  }
  __syncthreads();

  const int64_t total = (int64_t)a.bh * a.nj;
  for (int64_t base = (int64_t)blockIdx.x * kNodesPerBlock; base < total;
       base += (int64_t)gridDim.x * kNodesPerBlock) {
    for (int t = 0; t < NPW; ++t) {
      const int nl = warp * NPW + t;
      const int64_t id = base + nl;
      float2 ks2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};  // dims (0,1), (2,3) of the lane's 4
      float2 vs2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      float ks[4] = {0.f, 0.f, 0.f, 0.f}, vs[4] = {0.f, 0.f, 0.f, 0.f};
      if (id < total) {
        const int64_t bhi = id / a.nj;
        const int64_t j = a.j0 + id % a.nj;
        const int64_t c0 = j * a.b;
        const int64_t c1 = min(c0 + (int64_t)a.b, a.n_prev);
        const uint16_t *kb = a.src_k + (a.src_row_off + bhi * a.src_slots) * kD + lane * 4;
        const uint16_t *vb = a.src_v + (a.src_row_off + bhi * a.src_slots) * kD + lane * 4;
        // Every child but the level's last covers span_prev tokens, so the value mean
        // sums the children with weight 1 and then gives the last child, if it covers
        // fewer tokens, its share f = tokens / span_prev.
#pragma unroll 16  // a whole node's children (b = 16) in flight at once
        for (int64_t c = c0; c < c1; ++c) {
          const uint2 ku = __ldg(reinterpret_cast<const uint2 *>(kb + c * kD));
          const uint2 vu = __ldg(reinterpret_cast<const uint2 *>(vb + c * kD));
          ks2[0] = __fadd2_rn(ks2[0], make_float2(bf16_lo(ku.x), bf16_hi(ku.x)));
          ks2[1] = __fadd2_rn(ks2[1], make_float2(bf16_lo(ku.y), bf16_hi(ku.y)));
          vs2[0] = __fadd2_rn(vs2[0], make_float2(bf16_lo(vu.x), bf16_hi(vu.x)));
          vs2[1] = __fadd2_rn(vs2[1], make_float2(bf16_lo(vu.y), bf16_hi(vu.y)));
        }
        ks[0] = ks2[0].x, ks[1] = ks2[0].y, ks[2] = ks2[1].x, ks[3] = ks2[1].y;
        vs[0] = vs2[0].x, vs[1] = vs2[0].y, vs[2] = vs2[1].x, vs[3] = vs2[1].y;
        const float nch = (float)(c1 - c0);
        float wsum = nch;
        if (c1 == a.n_prev && c1 > c0) {
          const int64_t last_tokens = a.length - (c1 - 1) * a.span_prev;
          if (last_tokens < a.span_prev) {
            const float f1 = (float)last_tokens / (float)a.span_prev - 1.f;
            const uint2 vu = __ldg(reinterpret_cast<const uint2 *>(vb + (c1 - 1) * kD));
            vs[0] += f1 * bf16_lo(vu.x);
            vs[1] += f1 * bf16_hi(vu.x);
            vs[2] += f1 * bf16_lo(vu.y);
            vs[3] += f1 * bf16_hi(vu.y);
            wsum += f1;
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          ks[i] = ks[i] / nch;
          vs[i] = vs[i] / wsum;
        }
        uint2 vo;
        vo.x = pack_bf16x2(vs[0], vs[1]);
        vo.y = pack_bf16x2(vs[2], vs[3]);
        *reinterpret_cast<uint2 *>(a.dst_v + (a.dst_row_off + bhi * a.dst_slots + j) * kD + lane * 4) = vo;
      }
      *reinterpret_cast<float4 *>(Mean + nl * kD + lane * 4) = make_float4(ks[0], ks[1], ks[2], ks[3]);
    }
    __syncwarp();  // a warp applies W to its own 8 nodes only: warps run out of step, so some
                   // stream children while others compute

    // key = W @ mean for this warp's 8 nodes; lane owns outputs 4*lane .. 4*lane+3, as the
    // pairs (4l, 4l+1) and (4l+2, 4l+3) of packed fp32 FMAs (each output's terms in k order)
    float2 acc2[NPW][2];
#pragma unroll
    for (int n = 0; n < NPW; ++n) acc2[n][0] = acc2[n][1] = make_float2(0.f, 0.f);
    const float4 *Wt4 = reinterpret_cast<const float4 *>(Wt);
    const float4 *M4 = reinterpret_cast<const float4 *>(Mean);
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
        const float4 m = M4[(warp * NPW + n) * 32 + (k >> 2)];
        const float mt[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float2 mm = make_float2(mt[t], mt[t]);
          acc2[n][0] = __ffma2_rn(mm, w[t][0], acc2[n][0]);
          acc2[n][1] = __ffma2_rn(mm, w[t][1], acc2[n][1]);
        }
      }
    }
    float acc[NPW][4];
#pragma unroll
    for (int n = 0; n < NPW; ++n) {
      acc[n][0] = acc2[n][0].x;
      acc[n][1] = acc2[n][0].y;
      acc[n][2] = acc2[n][1].x;
      acc[n][3] = acc2[n][1].y;
    }
#pragma unroll
    for (int n = 0; n < NPW; ++n) {
      const int64_t id = base + warp * NPW + n;
      if (id < total) {
        const int64_t bhi = id / a.nj;
        const int64_t j = a.j0 + id % a.nj;
        uint2 ko;
        ko.x = pack_bf16x2(acc[n][0], acc[n][1]);
        ko.y = pack_bf16x2(acc[n][2], acc[n][3]);
        *reinterpret_cast<uint2 *>(a.dst_k + (a.dst_row_off + bhi * a.dst_slots + j) * kD + lane * 4) = ko;
      }
    }
    __syncwarp();  // this warp's Mean rows are rewritten next
  }
}

// k_new / v_new [B][C][Hkv][128] -> token caches [B][Hkv][capacity][128] at slot `at + i`.
__global__ void append_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new, uint16_t *k_tok,
                              uint16_t *v_tok, int64_t capacity, int64_t at, int chunk, int hkv, int64_t rows) {
  const int64_t n16 = rows * 16;  // 16-byte pieces
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n16; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = e >> 4;
    const int part = (int)(e & 15);
    const int h = (int)(row % hkv);
    const int64_t bi_i = row / hkv;
    const int64_t i = bi_i % chunk;
    const int64_t bi = bi_i / chunk;
    const int64_t dst = ((bi * hkv + h) * capacity + at + i) * kD + part * 8;
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
  a.pooler = t.pooler;
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(build_level_kernel<kNodesPerWarp>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)build_smem(kNodesPerWarp));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(build_level_kernel<kFewNodes>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)build_smem(kFewNodes));
    if (e != cudaSuccess) return (int)e;
    configured_device = dev;
  }
  const int64_t nodes = (int64_t)a.bh * a.nj;
  const int64_t full_grid = (int64_t)sm_count() * 2;
  if (nodes <= full_grid * kBuildWarps * kFewNodes) {  // fits one pass of warps with a node each
    const int64_t grid = ceil_div(nodes, kBuildWarps * kFewNodes);
    build_level_kernel<kFewNodes><<<(unsigned)grid, kBuildThreads, build_smem(kFewNodes), (cudaStream_t)stream>>>(a);
  } else {
    const int64_t grid = std::min<int64_t>(ceil_div(nodes, kBuildWarps * kNodesPerWarp), full_grid);
    build_level_kernel<kNodesPerWarp>
        <<<(unsigned)grid, kBuildThreads, build_smem(kNodesPerWarp), (cudaStream_t)stream>>>(a);
  }
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
      rows);
  return (int)cudaGetLastError();
}

}  // namespace recsa
