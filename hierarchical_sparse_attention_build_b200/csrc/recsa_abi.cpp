// Host side of the C ABI: argument validation, tree layout, workspace sizing and
// the sequence of kernel launches behind each call.  No call allocates, frees or
// synchronises, except recsa_check_device_errors.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "recsa.h"
#include "recsa_internal.h"

namespace recsa {

namespace {
thread_local char g_last_error[512] = "";
}

void set_error(const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
  va_end(ap);
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

int levels_for(int64_t length, int b) {
  int T = 0;
  int64_t n = length;
  while (n > b) {
    n = ceil_div(n, b);
    ++T;
  }
  return T;
}

}  // namespace recsa

using namespace recsa;

namespace {

recsa_status fail(recsa_status s, const char *fmt, ...) {
  char buf[480];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  set_error("%s: %s", recsa_status_string(s), buf);
  return s;
}

recsa_status cuda_fail(int rc, const char *what) {
  if (rc < 0) return RECSA_ERR_UNSUPPORTED;  // message already set by the launcher
  set_error("RECSA_ERR_CUDA: %s: %s", what, cudaGetErrorString((cudaError_t)rc));
  return RECSA_ERR_CUDA;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

recsa_status check_params(const recsa_params *p) {
  if (!p) return fail(RECSA_ERR_INVALID_ARGUMENT, "params is NULL");
  if (p->head_dim != kD) return fail(RECSA_ERR_UNSUPPORTED, "head_dim %d (only 128)", p->head_dim);
  if (p->num_kv_heads < 1) return fail(RECSA_ERR_INVALID_ARGUMENT, "num_kv_heads %d", p->num_kv_heads);
  if (p->num_q_heads < 1 || p->num_q_heads % p->num_kv_heads != 0)
    return fail(RECSA_ERR_INVALID_ARGUMENT, "num_q_heads %d is not a multiple of num_kv_heads %d", p->num_q_heads,
                p->num_kv_heads);
  const int G = p->num_q_heads / p->num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return fail(RECSA_ERR_UNSUPPORTED, "query heads per KV group %d (1, 2, 4 or 8)", G);
  if (p->branching < 2) return fail(RECSA_ERR_INVALID_ARGUMENT, "branching %d < 2", p->branching);
  if (p->branching > 4096) return fail(RECSA_ERR_UNSUPPORTED, "branching %d > 4096", p->branching);
  if (p->top_k < 0) return fail(RECSA_ERR_INVALID_ARGUMENT, "top_k %d < 0", p->top_k);
  if (!(p->rope_base > 0.f) || !std::isfinite(p->rope_base))
    return fail(RECSA_ERR_INVALID_ARGUMENT, "rope_base %g", (double)p->rope_base);
  if (!(p->softmax_scale >= 0.f) || !std::isfinite(p->softmax_scale))
    return fail(RECSA_ERR_INVALID_ARGUMENT, "softmax_scale %g", (double)p->softmax_scale);
  return RECSA_OK;
}

recsa_status make_geom(const recsa_params *p, int32_t batch, int64_t capacity, TreeGeom *g) {
  if (batch < 1) return fail(RECSA_ERR_INVALID_ARGUMENT, "batch %d < 1", batch);
  if (capacity < 1) return fail(RECSA_ERR_INVALID_ARGUMENT, "capacity %lld < 1", (long long)capacity);
  if (capacity > ((int64_t)1 << 30))
    return fail(RECSA_ERR_UNSUPPORTED, "capacity %lld > 2^30 tokens", (long long)capacity);
  std::memset(g, 0, sizeof *g);
  g->batch = batch;
  g->hkv = p->num_kv_heads;
  g->b = p->branching;
  g->capacity = capacity;
  const int T = levels_for(capacity, p->branching);
  if (T > kMaxLevels) return fail(RECSA_ERR_UNSUPPORTED, "%d levels > %d", T, kMaxLevels);
  g->levels_cap = T;
  g->slots[0] = capacity;
  g->span[0] = 1;
  int64_t off = 0;
  for (int l = 1; l <= kMaxLevels; ++l) {
    g->span[l] = g->span[l - 1] > (((int64_t)1 << 62) / p->branching) ? ((int64_t)1 << 62)
                                                                         : g->span[l - 1] * p->branching;
    if (l <= T) {
      g->slots[l] = ceil_div(g->slots[l - 1], p->branching);
      g->row_off[l] = off;
      off += (int64_t)batch * p->num_kv_heads * g->slots[l];
    }
  }
  g->row_off[0] = 0;
  return RECSA_OK;
}

// Largest candidate count of any level for a cache of `length` tokens.
int64_t max_candidates(const recsa_params *p, int64_t length, bool causal) {
  const int64_t kk = (int64_t)p->top_k + (causal ? 1 : 0);
  const int64_t b = p->branching;
  const int64_t m = std::min(kk * b, length);
  return std::max(b, m);
}

int64_t table_rows_for(const recsa_params *p, int64_t capacity) {
  const int64_t m = std::min<int64_t>(max_candidates(p, capacity, true), kMaxCand);
  return m + 1;
}

size_t workspace_bytes(const recsa_params *p, int64_t capacity) {
  return kWsHeader + (size_t)table_rows_for(p, capacity) * kHalf * sizeof(float) * 2;
}

recsa_status check_tree(const recsa_params *p, const recsa_tree *t, TreeGeom *g) {
  if (!t) return fail(RECSA_ERR_INVALID_ARGUMENT, "tree is NULL");
  recsa_status s = make_geom(p, t->batch, t->capacity, g);
  if (s != RECSA_OK) return s;
  if (t->length < 0 || t->length > t->capacity)
    return fail(RECSA_ERR_INVALID_ARGUMENT, "length %lld outside [0, capacity %lld]", (long long)t->length,
                (long long)t->capacity);
  const void *ptrs[5] = {t->k_tok, t->v_tok, t->k_node, t->v_node, t->pooler};
  const char *names[5] = {"k_tok", "v_tok", "k_node", "v_node", "pooler"};
  for (int i = 0; i < 5; ++i) {
    if (!ptrs[i]) return fail(RECSA_ERR_INVALID_ARGUMENT, "tree->%s is NULL", names[i]);
    if (!aligned16(ptrs[i])) return fail(RECSA_ERR_INVALID_ARGUMENT, "tree->%s is not 16-byte aligned", names[i]);
  }
  if (t->seq_len && reinterpret_cast<uintptr_t>(t->seq_len) % 8 != 0)
    return fail(RECSA_ERR_INVALID_ARGUMENT, "tree->seq_len is not 8-byte aligned");
  if (t->page_table) {
    const int32_t P = t->page_size;
    if (P < 1 || P > 65536 || (P & (P - 1)) != 0)
      return fail(RECSA_ERR_INVALID_ARGUMENT, "page_size %d is not a power of two in 1 .. 65536", P);
    if (t->capacity % P != 0)
      return fail(RECSA_ERR_INVALID_ARGUMENT, "capacity %lld is not a multiple of page_size %d",
                  (long long)t->capacity, P);
    if (t->num_pages < 1) return fail(RECSA_ERR_INVALID_ARGUMENT, "num_pages %d < 1", t->num_pages);
    if (reinterpret_cast<uintptr_t>(t->page_table) % 4 != 0)
      return fail(RECSA_ERR_INVALID_ARGUMENT, "tree->page_table is not 4-byte aligned");
    if ((int64_t)t->num_pages * g->hkv * P > ((int64_t)1 << 40))
      return fail(RECSA_ERR_UNSUPPORTED, "a page pool of %d pages", t->num_pages);
  }
  return RECSA_OK;
}

recsa_status check_ws(const recsa_params *p, const recsa_tree *t, const void *ws, size_t ws_bytes) {
  if (!ws) return fail(RECSA_ERR_INVALID_ARGUMENT, "workspace is NULL");
  if (!aligned16(ws)) return fail(RECSA_ERR_INVALID_ARGUMENT, "workspace is not 16-byte aligned");
  const size_t need = workspace_bytes(p, t->capacity);
  if (ws_bytes < need)
    return fail(RECSA_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes < %zu needed", ws_bytes, need);
  return RECSA_OK;
}

recsa_status check_debug(const recsa_params *p, const recsa_debug *d) {
  if (!d) return RECSA_OK;
  if (d->sel_idx && (p->top_k > kDebugMaxK || p->top_k < 1 || d->sel_levels < 1))
    return fail(RECSA_ERR_INVALID_ARGUMENT, "sel_idx needs 1 <= top_k <= %d and sel_levels >= 1", kDebugMaxK);
  if (d->cluster_size != 0 && d->cluster_size != 1 && d->cluster_size != 2 && d->cluster_size != 4)
    return fail(RECSA_ERR_INVALID_ARGUMENT, "cluster_size %d (0, 1, 2 or 4)", d->cluster_size);
  if (d->kernel < 0 || d->kernel > 4) return fail(RECSA_ERR_INVALID_ARGUMENT, "kernel %d (0 .. 4)", d->kernel);
  return RECSA_OK;
}

recsa_status build_range(const TreeGeom &g, const recsa_tree &t, int64_t length, int64_t old_length,
                         bool extension, void *stream) {
  const int T_new = levels_for(length, g.b);
  const int T_old = extension ? levels_for(old_length, g.b) : 0;
  for (int l = 1; l <= T_new; ++l) {
    const int64_t j0 = (extension && l <= T_old) ? old_length / g.span[l] : 0;
    const int64_t j1 = ceil_div(length, g.span[l]);
    const int rc = launch_build_level(g, t, l, length, j0, j1, stream);
    if (rc != 0) return cuda_fail(rc, "build level");
  }
  return RECSA_OK;
}

// Appends `chunk` tokens at L (at each sequence's own length when the tree has per-sequence
// lengths) and rebuilds every node whose span meets them.  When the chunk is short and each
// level has at most kPathNodes such nodes per (sequence, head) (a decode step's token, a
// short prefill chunk), or when the sequences have their own lengths, one launch appends
// and walks the ancestor path, a CTA per (sequence, head); otherwise the tokens are copied
// and each level is rebuilt by its own launch, wide over the level's nodes.
constexpr int64_t kPathNodes = 4;
constexpr int kPathTokens = 64;
recsa_status extend_tree(const TreeGeom &g, const recsa_tree &t, const void *k_new, const void *v_new, int64_t L,
                         int chunk, void *stream) {
  const int64_t L2 = L + chunk;
  const int T_new = levels_for(L2, g.b);
  const int T_old = levels_for(L, g.b);
  int64_t most = 0;
  for (int l = 1; l <= T_new; ++l)
    most = std::max(most, ceil_div(L2, g.span[l]) - (l <= T_old ? L / g.span[l] : 0));
  if (t.seq_len || (chunk <= kPathTokens && most <= kPathNodes)) {
    const int rc = launch_extend(g, t, k_new, v_new, L, chunk, T_new, stream);
    return rc != 0 ? cuda_fail(rc, "append and path update") : RECSA_OK;
  }
  const int rc = launch_append(g, t, k_new, v_new, L, chunk, stream);
  if (rc != 0) return cuda_fail(rc, "append");
  return build_range(g, t, L2, L, true, stream);
}

// Every check of a decode call and the launch it becomes (nothing is queued here).
recsa_status decode_launch(const recsa_params *params, const recsa_tree *tree, const void *q, int32_t num_queries,
                           void *out, int32_t out_is_fp32, void *ws, size_t ws_bytes, const recsa_debug *debug,
                           AttendLaunch *l) {
  recsa_status s = check_params(params);
  if (s != RECSA_OK) return s;
  TreeGeom g;
  s = check_tree(params, tree, &g);
  if (s != RECSA_OK) return s;
  if (tree->length < 1) return fail(RECSA_ERR_INVALID_ARGUMENT, "decode needs length >= 1");
  if (num_queries < 1) return fail(RECSA_ERR_INVALID_ARGUMENT, "num_queries %d < 1", num_queries);
  if (!q || !out) return fail(RECSA_ERR_INVALID_ARGUMENT, "q or out is NULL");
  if (!aligned16(q) || !aligned16(out)) return fail(RECSA_ERR_INVALID_ARGUMENT, "q or out is not 16-byte aligned");
  s = check_ws(params, tree, ws, ws_bytes);
  if (s != RECSA_OK) return s;
  s = check_debug(params, debug);
  if (s != RECSA_OK) return s;
  const int64_t mc = max_candidates(params, tree->length, false);
  if (mc > kMaxCand)
    return fail(RECSA_ERR_UNSUPPORTED, "up to %lld candidates per level > %d", (long long)mc, kMaxCand);
  const int64_t tiles = (int64_t)tree->batch * params->num_kv_heads * num_queries;
  if (tiles > 0x7fffffff / 4) return fail(RECSA_ERR_UNSUPPORTED, "%lld tiles", (long long)tiles);
  l->geom = g;
  l->tree = *tree;
  l->q = q;
  l->out = out;
  l->out_fp32 = out_is_fp32 ? 1 : 0;
  l->num_queries = num_queries;
  l->length = tree->length;
  l->causal = 0;
  l->group = params->num_q_heads / params->num_kv_heads;
  l->top_k = params->top_k;
  l->scale = params->softmax_scale > 0.f ? params->softmax_scale : 1.0f / std::sqrt((float)kD);
  l->ws = ws;
  l->table_rows_needed = (int)mc + 1;
  l->max_cand = (int)((mc + 31) / 32 * 32);
  l->cluster_size = debug ? debug->cluster_size : 0;
  l->kernel = debug ? debug->kernel : 0;
  l->debug = debug;
  return RECSA_OK;
}

}  // namespace

extern "C" {

RECSA_API const char *recsa_status_string(recsa_status s) {
  switch (s) {
    case RECSA_OK: return "RECSA_OK";
    case RECSA_ERR_INVALID_ARGUMENT: return "RECSA_ERR_INVALID_ARGUMENT";
    case RECSA_ERR_UNSUPPORTED: return "RECSA_ERR_UNSUPPORTED";
    case RECSA_ERR_WORKSPACE_TOO_SMALL: return "RECSA_ERR_WORKSPACE_TOO_SMALL";
    case RECSA_ERR_CAPACITY: return "RECSA_ERR_CAPACITY";
    case RECSA_ERR_CUDA: return "RECSA_ERR_CUDA";
    case RECSA_ERR_DEVICE_CHECK: return "RECSA_ERR_DEVICE_CHECK";
    case RECSA_ERR_TIMEOUT: return "RECSA_ERR_TIMEOUT";
  }
  return "RECSA_ERR_UNKNOWN";
}

RECSA_API const char *recsa_last_error(void) { return g_last_error; }

RECSA_API recsa_status recsa_tree_layout(const recsa_params *params, int32_t batch, int64_t capacity,
                                         int64_t *node_rows_out, int32_t *num_levels_out,
                                         int64_t level_row_offsets_out[RECSA_MAX_LEVELS + 1]) {
  recsa_status s = check_params(params);
  if (s != RECSA_OK) return s;
  TreeGeom g;
  s = make_geom(params, batch, capacity, &g);
  if (s != RECSA_OK) return s;
  int64_t rows = 0;
  for (int l = 1; l <= g.levels_cap; ++l) rows += (int64_t)batch * params->num_kv_heads * g.slots[l];
  if (node_rows_out) *node_rows_out = rows;
  if (num_levels_out) *num_levels_out = g.levels_cap;
  if (level_row_offsets_out)
    for (int l = 0; l <= RECSA_MAX_LEVELS; ++l) level_row_offsets_out[l] = (l <= g.levels_cap) ? g.row_off[l] : 0;
  return RECSA_OK;
}

RECSA_API recsa_status recsa_workspace_size(const recsa_params *params, int64_t capacity, size_t *bytes_out) {
  recsa_status s = check_params(params);
  if (s != RECSA_OK) return s;
  if (capacity < 1) return fail(RECSA_ERR_INVALID_ARGUMENT, "capacity %lld < 1", (long long)capacity);
  if (!bytes_out) return fail(RECSA_ERR_INVALID_ARGUMENT, "bytes_out is NULL");
  *bytes_out = workspace_bytes(params, capacity);
  return RECSA_OK;
}

RECSA_API recsa_status recsa_workspace_init(const recsa_params *params, int64_t capacity, void *ws, size_t ws_bytes,
                                            recsa_stream_t stream) {
  recsa_status s = check_params(params);
  if (s != RECSA_OK) return s;
  if (capacity < 1) return fail(RECSA_ERR_INVALID_ARGUMENT, "capacity %lld < 1", (long long)capacity);
  if (!ws || !aligned16(ws)) return fail(RECSA_ERR_INVALID_ARGUMENT, "workspace is NULL or not 16-byte aligned");
  const size_t need = workspace_bytes(params, capacity);
  if (ws_bytes < need) return fail(RECSA_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes < %zu needed", ws_bytes, need);
  const int rc = launch_rope_table(ws, (int)table_rows_for(params, capacity), (double)params->rope_base, stream);
  if (rc != 0) return cuda_fail(rc, "rope table");
  return RECSA_OK;
}

RECSA_API recsa_status recsa_build_tree(const recsa_params *params, const recsa_tree *tree, recsa_stream_t stream) {
  recsa_status s = check_params(params);
  if (s != RECSA_OK) return s;
  TreeGeom g;
  s = check_tree(params, tree, &g);
  if (s != RECSA_OK) return s;
  return build_range(g, *tree, tree->length, 0, false, stream);
}

RECSA_API recsa_status recsa_decode(const recsa_params *params, const recsa_tree *tree, const void *q,
                                    int32_t num_queries, void *out, int32_t out_is_fp32, void *ws, size_t ws_bytes,
                                    const recsa_debug *debug, recsa_stream_t stream) {
  AttendLaunch l;
  const recsa_status s = decode_launch(params, tree, q, num_queries, out, out_is_fp32, ws, ws_bytes, debug, &l);
  if (s != RECSA_OK) return s;
  const int rc = launch_attend(l, stream);
  if (rc != 0) return cuda_fail(rc, "decode attend");
  return RECSA_OK;
}

RECSA_API recsa_status recsa_decode_host(const recsa_params *params, const recsa_tree *tree, const void *q_host,
                                         int32_t num_queries, void *out_host, int32_t out_is_fp32, void *q_dev,
                                         void *out_dev, void *ws, size_t ws_bytes, const recsa_debug *debug,
                                         recsa_stream_t stream) {
  if (!q_host || !out_host) return fail(RECSA_ERR_INVALID_ARGUMENT, "q_host or out_host is NULL");
  if (!aligned16(q_host) || !aligned16(out_host))
    return fail(RECSA_ERR_INVALID_ARGUMENT, "q_host or out_host is not 16-byte aligned");
  AttendLaunch l;  // every check, on the staging buffers, before any CUDA call
  const recsa_status s = decode_launch(params, tree, q_dev, num_queries, out_dev, out_is_fp32, ws, ws_bytes, debug, &l);
  if (s != RECSA_OK) return s;
  // Pinned host memory is mapped into the device's address space: the kernel then reads
  // the queries and writes the outputs across the host link itself (no staging copy).
  // Pageable memory goes through the staging buffers.
  auto mapped = [](const void *host) -> void * {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, host) != cudaSuccess) {
      cudaGetLastError();  // a pointer the runtime does not know: not an error of this call
      return nullptr;
    }
    return at.type == cudaMemoryTypeHost ? at.devicePointer : nullptr;
  };
  void *q_map = mapped(q_host), *out_map = mapped(out_host);
  if (q_map) l.q = q_map;
  if (out_map) l.out = out_map;
  const size_t q_bytes = (size_t)tree->batch * num_queries * params->num_q_heads * kD * 2;
  const size_t out_bytes = q_bytes * (out_is_fp32 ? 2 : 1);
  if (!q_map) {
    const cudaError_t e = cudaMemcpyAsync(q_dev, q_host, q_bytes, cudaMemcpyHostToDevice, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail((int)e, "copy of the queries to the device");
  }
  const int rc = launch_attend(l, stream);
  if (rc != 0) return cuda_fail(rc, "decode attend");
  if (!out_map) {
    const cudaError_t e = cudaMemcpyAsync(out_host, out_dev, out_bytes, cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail((int)e, "copy of the output to the host");
  }
  return RECSA_OK;
}

RECSA_API recsa_status recsa_append(const recsa_params *params, recsa_tree *tree, const void *k_new,
                                    const void *v_new, int32_t count, recsa_stream_t stream) {
  recsa_status s = check_params(params);
  if (s != RECSA_OK) return s;
  TreeGeom g;
  s = check_tree(params, tree, &g);
  if (s != RECSA_OK) return s;
  if (count < 1) return fail(RECSA_ERR_INVALID_ARGUMENT, "count %d < 1", count);
  if (!k_new || !v_new) return fail(RECSA_ERR_INVALID_ARGUMENT, "k_new or v_new is NULL");
  if (!aligned16(k_new) || !aligned16(v_new))
    return fail(RECSA_ERR_INVALID_ARGUMENT, "k_new or v_new is not 16-byte aligned");
  const int64_t L = tree->length;
  if (L + count > tree->capacity)
    return fail(RECSA_ERR_CAPACITY, "length %lld + count %d > capacity %lld", (long long)L, count,
                (long long)tree->capacity);
  s = extend_tree(g, *tree, k_new, v_new, L, count, stream);
  if (s != RECSA_OK) return s;
  if (tree->seq_len) {
    const int rc = launch_advance_lengths(tree->seq_len, tree->batch, count, L + count, stream);
    if (rc != 0) return cuda_fail(rc, "advance of the sequence lengths");
  }
  tree->length = L + count;
  return RECSA_OK;
}

RECSA_API recsa_status recsa_decode_step(const recsa_params *params, const recsa_tree *tree, const void *k_new,
                                         const void *v_new, const void *q, void *out, int32_t out_is_fp32, void *ws,
                                         size_t ws_bytes, recsa_stream_t stream) {
  recsa_status s = check_params(params);
  if (s != RECSA_OK) return s;
  TreeGeom g;
  s = check_tree(params, tree, &g);
  if (s != RECSA_OK) return s;
  if (!tree->seq_len) return fail(RECSA_ERR_INVALID_ARGUMENT, "a decode step needs per-sequence lengths (tree->seq_len)");
  if (!k_new || !v_new || !q || !out) return fail(RECSA_ERR_INVALID_ARGUMENT, "k_new, v_new, q or out is NULL");
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(q) || !aligned16(out))
    return fail(RECSA_ERR_INVALID_ARGUMENT, "k_new, v_new, q or out is not 16-byte aligned");
  s = check_ws(params, tree, ws, ws_bytes);
  if (s != RECSA_OK) return s;
  // every bound comes from the capacity, none from the current lengths
  const int64_t cap = tree->capacity;
  const int64_t mc = max_candidates(params, cap, false);
  if (mc > kMaxCand)
    return fail(RECSA_ERR_UNSUPPORTED, "up to %lld candidates per level > %d", (long long)mc, kMaxCand);
  uint32_t *err = &reinterpret_cast<WsHeader *>(ws)->err;
  int rc = launch_extend(g, *tree, k_new, v_new, cap - 1, 1, levels_for(cap, g.b), stream, err);
  if (rc != 0) return cuda_fail(rc, "append and path update");
  rc = launch_advance_lengths(tree->seq_len, tree->batch, 1, cap, stream);
  if (rc != 0) return cuda_fail(rc, "advance of the sequence lengths");
  AttendLaunch l;
  l.geom = g;
  l.tree = *tree;
  l.q = q;
  l.out = out;
  l.out_fp32 = out_is_fp32 ? 1 : 0;
  l.num_queries = 1;
  l.length = cap;
  l.causal = 0;
  l.group = params->num_q_heads / params->num_kv_heads;
  l.top_k = params->top_k;
  l.scale = params->softmax_scale > 0.f ? params->softmax_scale : 1.0f / std::sqrt((float)kD);
  l.ws = ws;
  l.table_rows_needed = (int)mc + 1;
  l.max_cand = (int)((mc + 31) / 32 * 32);
  l.cluster_size = 0;
  l.kernel = 0;
  l.debug = nullptr;
  rc = launch_attend(l, stream);
  return rc != 0 ? cuda_fail(rc, "decode attend") : RECSA_OK;
}

RECSA_API recsa_status recsa_prefill_chunk(const recsa_params *params, recsa_tree *tree, const void *k_new,
                                           const void *v_new, const void *q, int32_t chunk, void *out,
                                           int32_t out_is_fp32, void *ws, size_t ws_bytes, const recsa_debug *debug,
                                           recsa_stream_t stream) {
  recsa_status s = check_params(params);
  if (s != RECSA_OK) return s;
  TreeGeom g;
  s = check_tree(params, tree, &g);
  if (s != RECSA_OK) return s;
  if (chunk < 1) return fail(RECSA_ERR_INVALID_ARGUMENT, "chunk %d < 1", chunk);
  if (!k_new || !v_new || !q || !out) return fail(RECSA_ERR_INVALID_ARGUMENT, "k_new, v_new, q or out is NULL");
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(q) || !aligned16(out))
    return fail(RECSA_ERR_INVALID_ARGUMENT, "k_new, v_new, q or out is not 16-byte aligned");
  const int64_t L = tree->length;
  const int64_t L2 = L + chunk;
  if (L2 > tree->capacity)
    return fail(RECSA_ERR_CAPACITY, "length %lld + chunk %d > capacity %lld", (long long)L, chunk,
                (long long)tree->capacity);
  s = check_ws(params, tree, ws, ws_bytes);
  if (s != RECSA_OK) return s;
  s = check_debug(params, debug);
  if (s != RECSA_OK) return s;
  const int64_t mc = max_candidates(params, L2, true);
  if (mc > kMaxCand)
    return fail(RECSA_ERR_UNSUPPORTED, "up to %lld candidates per level > %d", (long long)mc, kMaxCand);
  const int64_t tiles = (int64_t)tree->batch * params->num_kv_heads * chunk;
  if (tiles > 0x7fffffff / 4) return fail(RECSA_ERR_UNSUPPORTED, "%lld tiles", (long long)tiles);

  s = extend_tree(g, *tree, k_new, v_new, L, chunk, stream);
  if (s != RECSA_OK) return s;
  AttendLaunch l;
  l.geom = g;
  l.tree = *tree;
  l.q = q;
  l.out = out;
  l.out_fp32 = out_is_fp32 ? 1 : 0;
  l.num_queries = chunk;
  l.length = L;
  l.causal = 1;
  l.group = params->num_q_heads / params->num_kv_heads;
  l.top_k = params->top_k;
  l.scale = params->softmax_scale > 0.f ? params->softmax_scale : 1.0f / std::sqrt((float)kD);
  l.ws = ws;
  l.table_rows_needed = (int)mc + 1;
  l.max_cand = (int)((mc + 31) / 32 * 32);
  l.cluster_size = debug ? debug->cluster_size : 0;
  l.kernel = debug ? debug->kernel : 0;
  l.debug = debug;
  int rc = launch_attend(l, stream);
  if (rc != 0) return cuda_fail(rc, "prefill attend");
  if (tree->seq_len) {
    rc = launch_advance_lengths(tree->seq_len, tree->batch, chunk, L2, stream);
    if (rc != 0) return cuda_fail(rc, "advance of the sequence lengths");
  }
  tree->length = L2;
  return RECSA_OK;
}

RECSA_API recsa_status recsa_check_device_errors(void *ws, recsa_stream_t stream) {
  if (!ws) return fail(RECSA_ERR_INVALID_ARGUMENT, "workspace is NULL");
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail((int)e, "synchronize");
  uint32_t word = 0, build_word = 0;
  e = cudaMemcpy(&word, ws, sizeof word, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail((int)e, "read error word");
  const int rc = read_build_errors(&build_word);  // the build kernels' word (they take no workspace)
  if (rc != 0) return cuda_fail(rc, "read the build error word");
  word |= build_word;
  if (word == 0) return RECSA_OK;
  const uint32_t zero = 0;
  e = cudaMemcpy(ws, &zero, sizeof zero, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail((int)e, "clear error word");
  if (word & kErrTimeout) return fail(RECSA_ERR_TIMEOUT, "a bounded device wait ran out (0x%x)", word);
  return fail(RECSA_ERR_DEVICE_CHECK, "device check failed (0x%x: %s%s%s)", word,
              (word & kErrIndex) ? "index " : "", (word & kErrWs) ? "workspace " : "",
              (word & kErrCount) ? "candidate-count" : "");
}

}  // extern "C"
