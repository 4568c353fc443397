/*
 * recsa.h - C ABI of the RecSA (Recursive Sparse Attention) tree build and
 * level-wise sparse attend for NVIDIA B200 (sm_100a).
 *
 * Method: "Recursive Sparse Attention: Million-Token Length Extrapolation at
 * Logarithmic Cost" (arXiv 2611.07232), abstract.  A tree is built over the KV
 * cache; every node summarises its subtree with one key (a per-layer pooler that
 * all levels share) and one mean-pooled value.  A query descends the tree one
 * level at a time, keeping at most k candidates per level above the tokens; the
 * summaries of the candidates it does not keep share one softmax with the exact
 * tokens under the kept leaves, and every entry is RoPE-rotated at its index among
 * the candidates of its level.
 *
 * Readings this library implements where the abstract is silent:
 *   - pooler: parent key = W @ (mean of the children's stored pre-RoPE keys), W a
 *     caller-supplied fp32 128x128 row-major matrix, applied at every level;
 *   - parent value = token-count-weighted mean of the children's values (= mean of
 *     the subtree's tokens); node rows are stored as bf16 (round to nearest even);
 *   - levels: n_0 = L, n_{l+1} = ceil(n_l / b) while n_l > b (the top level has at
 *     most b nodes; L <= b means plain attention over the tokens);
 *   - selection ranks candidates by the sum, over the query heads of a KV group
 *     (heads g*G .. g*G+G-1), of the scaled logits; ties go to the lower node index;
 *   - the RoPE position of a candidate is its rank among its level's candidates in
 *     node order and the query's position is that level's candidate count;
 *     rotate-half RoPE over dims (i, i+64), angle pos * base^(-2i/128);
 *   - a query at position p sees tokens [0, p): decode queries sit at p = L; query i
 *     of a prefill chunk appended at L sits at p = L + i.  In prefill the partial
 *     trailing node of each level is not scored, takes no top-k slot, holds a
 *     position and is always expanded;
 *   - a query with nothing visible (prefill query 0 of an empty cache) outputs zeros.
 *
 * Conventions for every call:
 *   - data pointers are DEVICE pointers (CUDA global memory of the current device)
 *     unless stated; bf16 tensors are IEEE bfloat16, contiguous, row-major, and
 *     every base pointer must be 16-byte aligned;
 *   - the caller owns every buffer and keeps it alive until the work queued on
 *     `stream` has finished; no call allocates or frees device memory;
 *   - calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and never synchronise, except recsa_check_device_errors;
 *   - argument errors are reported synchronously with a status and nothing is
 *     launched; a failed launch returns RECSA_ERR_CUDA; recsa_last_error() gives a
 *     thread-local description of the most recent failure;
 *   - the library holds no device state of its own; calls on different streams
 *     with disjoint outputs may run concurrently.
 */
#ifndef RECSA_H
#define RECSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(_WIN32)
#define RECSA_API
#else
#define RECSA_API __attribute__((visibility("default")))
#endif

typedef struct CUstream_st *recsa_stream_t; /* ABI-identical to cudaStream_t */

typedef enum recsa_status {
  RECSA_OK = 0,
  RECSA_ERR_INVALID_ARGUMENT = 1,    /* null/misaligned pointer, bad size or shape  */
  RECSA_ERR_UNSUPPORTED = 2,         /* valid but outside what the kernels handle   */
  RECSA_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes below recsa_workspace_size()       */
  RECSA_ERR_CAPACITY = 4,            /* length + chunk exceeds the cache capacity   */
  RECSA_ERR_CUDA = 5,                /* a CUDA runtime call or launch failed        */
  RECSA_ERR_DEVICE_CHECK = 6,        /* a kernel found an out-of-range index or a
                                        workspace that was not initialised          */
  RECSA_ERR_TIMEOUT = 7              /* a bounded device-side wait ran out          */
} recsa_status;

#define RECSA_HEAD_DIM 128
#define RECSA_TOPK_ALL 0x7fffffff /* keep every candidate (full expansion) */
#define RECSA_MAX_LEVELS 40       /* levels above the tokens a tree may have */
#define RECSA_MAX_CANDIDATES 4096 /* per level and query group (see recsa_decode) */

/* Per-layer attention shape and method parameters. */
typedef struct recsa_params {
  int32_t head_dim;     /* must be 128                                              */
  int32_t num_kv_heads; /* Hkv >= 1                                                 */
  int32_t num_q_heads;  /* Hq = G * Hkv with G (query heads per KV group) 1, 2, 4, 8 */
  int32_t branching;    /* b >= 2 children per node                                 */
  int32_t top_k;        /* k >= 0 kept per level above the tokens, or RECSA_TOPK_ALL */
  float rope_base;      /* > 0, e.g. 1e6                                            */
  float softmax_scale;  /* > 0, or 0 for 1/sqrt(128)                                */
} recsa_params;

/* One layer's KV cache and its summary tree.
 *   k_tok, v_tok : bf16 [batch][Hkv][capacity][128], pre-RoPE token keys / values;
 *                  slots [0, length) are valid.
 *   k_node, v_node: bf16 node arena, each [node_rows][128] with the layout that
 *                  recsa_tree_layout() returns for (batch, capacity); level l,
 *                  sequence s, KV head h, node j sits at row
 *                  level_row_offsets[l] + (s*Hkv + h) * ceil(capacity / b^l) + j.
 *   pooler       : fp32 [128][128] row-major W (node key = W @ mean of child keys).
 *   seq_len      : NULL when every sequence holds `length` tokens.  Otherwise a device
 *                  array int64 [batch], 8-byte aligned, owned by the caller: sequence s
 *                  holds seq_len[s] tokens, 0 <= seq_len[s] <= length, and `length` is
 *                  the longest (the host-side bound every size check uses).  Each
 *                  sequence then has its own tree over its own tokens (levels, node
 *                  counts, query positions).  recsa_append and recsa_prefill_chunk append
 *                  at each sequence's own end and advance seq_len on the device (queued
 *                  after their kernels) as they advance `length` on the host.  The
 *                  kernels clamp an entry outside [0, length] into it; decode and prefill
 *                  calls also flag one in the workspace error word
 *                  (RECSA_ERR_DEVICE_CHECK from recsa_check_device_errors).
 *   page_table   : NULL for the contiguous caches above.  Otherwise the token caches are
 *                  a paged pool: k_tok, v_tok are bf16 [num_pages][Hkv][page_size][128],
 *                  and page_table is a device array int32 [batch][capacity / page_size],
 *                  4-byte aligned, owned by the caller: token t of sequence s sits in
 *                  page page_table[s][t / page_size], row t % page_size.  page_size is a
 *                  power of two (1 .. 65536) dividing capacity; num_pages >= 1.  Every
 *                  call reads the same rows as with contiguous caches (the results are
 *                  identical); appends write into the pages the table names, so the
 *                  caller maps a sequence's pages before its tokens reach them.  A table
 *                  entry outside [0, num_pages) is never dereferenced: the attend kernels
 *                  skip the row and flag it (RECSA_ERR_DEVICE_CHECK), the build and append
 *                  kernels skip it (such a tree holds undefined rows). */
typedef struct recsa_tree {
  int32_t batch;
  int32_t reserved;
  int64_t capacity;
  int64_t length;
  void *k_tok;
  void *v_tok;
  void *k_node;
  void *v_node;
  const float *pooler;
  int64_t *seq_len;
  const int32_t *page_table;
  int32_t page_size;
  int32_t num_pages;
} recsa_tree;

/* Optional diagnostics and launch-shape overrides of recsa_decode / recsa_prefill_chunk
 * (pass NULL for none).  A "tile" is one (sequence, query, KV group); tiles are
 * numbered ((s * Hkv + g) * num_queries + query).
 *   sel_idx  : int32 [tiles][sel_levels][top_k]; slot (l-1) receives the node indices
 *              kept at level l (ascending, -1 padded).  Needs top_k <= 64.
 *   entries  : int32 [tiles][2]; keys scored and values folded by the tile (rows read).
 *   kernel   : 0 = automatic (3 while tiles <= SM count, 4 up to 4 x SM count tiles,
 *              2 beyond); 1 = one CTA (or a cluster of cluster_size CTAs) per tile;
 *              2 = one warp per tile, the throughput shape for many tiles; 3 = one
 *              cluster of 2 or 4 CTAs per tile in which every CTA ranks all of a
 *              level's scores (one cluster and one block barrier per level), where a
 *              level's candidates fit its registers, else shape 1; 4 = one CTA per
 *              tile with two CTAs sharing an SM (fewer rows in flight per CTA), where
 *              the group has at most 4 query heads and two CTAs' shared memory fits,
 *              else shape 1 with one CTA per tile.  Results agree up to fp32 rounding.
 *   cluster_size: with kernel 1 or 3: 0 = automatic, or 1, 2, 4 CTAs per tile. */
typedef struct recsa_debug {
  int32_t *sel_idx;
  int32_t *entries;
  int32_t sel_levels;
  int32_t kernel;
  int32_t cluster_size;
  int32_t reserved;
} recsa_debug;

/* Arena layout of a tree of `capacity` token slots (host only, no CUDA call).
 * Writes the total node rows (per K and per V arena), the number of levels above
 * the tokens for a cache filled to capacity, and level_row_offsets[0..levels]
 * (entry 0 is 0 and unused).  The arena size in bytes is node_rows * 256. */
RECSA_API recsa_status recsa_tree_layout(const recsa_params *params, int32_t batch, int64_t capacity,
                                         int64_t *node_rows_out, int32_t *num_levels_out,
                                         int64_t level_row_offsets_out[RECSA_MAX_LEVELS + 1]);

/* Bytes of the workspace that recsa_decode / recsa_prefill_chunk need for trees of
 * up to `capacity` tokens with these params (host only).  The workspace holds the
 * RoPE cos/sin table and the device error word. */
RECSA_API recsa_status recsa_workspace_size(const recsa_params *params, int64_t capacity, size_t *bytes_out);

/* Fill a workspace of ws_bytes >= recsa_workspace_size(params, capacity) bytes
 * (device pointer, 16-byte aligned): computes the RoPE table in fp64 and clears the
 * error word.  Call once per (params, capacity) before the first attend call that
 * uses this workspace; its contents then stay valid for every later call. */
RECSA_API recsa_status recsa_workspace_init(const recsa_params *params, int64_t capacity, void *ws,
                                            size_t ws_bytes, recsa_stream_t stream);

/* Build every level of the tree over the first tree->length tokens (abstract: each
 * node summarises its subtree with one pooled key and one mean-pooled value).
 * Overwrites the node arena rows of levels 1..T(length). */
RECSA_API recsa_status recsa_build_tree(const recsa_params *params, const recsa_tree *tree,
                                        recsa_stream_t stream);

/* Decode attention of num_queries independent queries per sequence, all at position
 * L = tree->length, over a tree built by recsa_build_tree (abstract: level-wise
 * selection of at most k candidates, unselected summaries sharing one softmax with
 * the exact tokens).
 *   q   : bf16 [batch][num_queries][Hq][128], pre-RoPE.
 *   out : [batch][num_queries][Hq][128], fp32 if out_is_fp32 else bf16.
 *   ws  : an initialised workspace (recsa_workspace_init) for >= tree->capacity.
 * Needs length >= 1 and at most RECSA_MAX_CANDIDATES candidates per level
 * (max(b, min(k*b, L)) here), else RECSA_ERR_UNSUPPORTED. */
RECSA_API recsa_status recsa_decode(const recsa_params *params, const recsa_tree *tree, const void *q,
                                    int32_t num_queries, void *out, int32_t out_is_fp32, void *ws,
                                    size_t ws_bytes, const recsa_debug *debug, recsa_stream_t stream);

/* recsa_decode on host buffers: one call takes a batch of queries in host memory to
 * attention outputs in host memory, queued on `stream`.  A pinned (page-locked) host
 * buffer is read or written by the decode kernel itself through its device mapping; a
 * pageable one is copied through the staging buffer (q_host -> q_dev before the decode,
 * out_dev -> out_host after it).  Not in the abstract: the plumbing a host-side caller
 * needs around recsa_decode.
 *   q_host   : host bf16 [batch][num_queries][Hq][128], 16-byte aligned.
 *   out_host : host output of the same shape, fp32 if out_is_fp32 else bf16, 16-byte aligned.
 *   q_dev, out_dev : device staging buffers of those sizes (16-byte aligned), owned by the
 *              caller (untouched when the host buffer is pinned).
 * The host buffers must stay untouched until the stream passes this call (out_host holds
 * the result after that).  Every argument is checked, as recsa_decode checks its own,
 * before anything is queued; a failed copy returns RECSA_ERR_CUDA. */
RECSA_API recsa_status recsa_decode_host(const recsa_params *params, const recsa_tree *tree, const void *q_host,
                                         int32_t num_queries, void *out_host, int32_t out_is_fp32, void *q_dev,
                                         void *out_dev, void *ws, size_t ws_bytes, const recsa_debug *debug,
                                         recsa_stream_t stream);

/* Append `count` tokens to every sequence and update the tree over them (abstract:
 * trees over the KV cache; the incremental update is not specified there): k_new /
 * v_new go to token slots L .. L+count-1 (L = tree->length), and every node whose span
 * meets those slots is rebuilt from its children -- the new tokens' ancestors, O(T)
 * nodes per (sequence, head) for one token -- plus any level that becomes new.  The
 * result equals recsa_build_tree over L + count tokens bit for bit (both form a key
 * with the same split-bf16 tensor-core product of the pooler).  This is the cache update of a
 * decode loop: append the step's token, then recsa_decode its query at the new length.
 * On success tree->length becomes L + count (host-side update; the device work is
 * still queued).
 *   k_new, v_new: bf16 [batch][count][Hkv][128] (device, 16-byte aligned).
 * Needs count >= 1 and L + count <= capacity (else RECSA_ERR_CAPACITY); nothing is
 * queued when a check fails. */
RECSA_API recsa_status recsa_append(const recsa_params *params, recsa_tree *tree, const void *k_new,
                                    const void *v_new, int32_t count, recsa_stream_t stream);

/* One decode step of a serving loop whose lengths live on the device: for every sequence s,
 * append one token (k_new, v_new: bf16 [batch][1][Hkv][128]) at slot seq_len[s] and update
 * the tree over it (as recsa_append), advance seq_len[s] by one, and decode that token's
 * query (q: bf16 [batch][1][Hq][128]; out as in recsa_decode) over its seq_len[s] tokens.
 * Not in the abstract: the plumbing of a decode loop.  Every kernel parameter comes from
 * the tree's capacity and its arrays, none from the current lengths, so the call can be
 * captured once into a CUDA graph and the graph replayed step after step (the caller writes
 * each step's k_new, v_new and q into the same buffers before a replay).  Needs
 * tree->seq_len (else RECSA_ERR_INVALID_ARGUMENT); tree->length is neither read nor
 * written.  A sequence with no room left (seq_len[s] == capacity) is not appended to, keeps
 * its length, and is flagged in the workspace error word (RECSA_ERR_DEVICE_CHECK); its query
 * is decoded over its tokens as they are. */
RECSA_API recsa_status recsa_decode_step(const recsa_params *params, const recsa_tree *tree, const void *k_new,
                                         const void *v_new, const void *q, void *out, int32_t out_is_fp32,
                                         void *ws, size_t ws_bytes, recsa_stream_t stream);

/* Causal prefill of a chunk of `chunk` tokens at positions L .. L+chunk-1
 * (L = tree->length): appends k_new / v_new to the token caches, rebuilds the tree
 * nodes those tokens touch (and any level that becomes new), then attends query i
 * at p = L + i.  On success tree->length becomes L + chunk (host-side update; the
 * device work is still queued).
 *   k_new, v_new: bf16 [batch][chunk][Hkv][128]; q: bf16 [batch][chunk][Hq][128];
 *   out: [batch][chunk][Hq][128] (fp32 or bf16).
 * Needs L + chunk <= capacity (else RECSA_ERR_CAPACITY) and at most
 * RECSA_MAX_CANDIDATES candidates per level (max(b, min((k+1)*b, L+chunk))). */
RECSA_API recsa_status recsa_prefill_chunk(const recsa_params *params, recsa_tree *tree, const void *k_new,
                                           const void *v_new, const void *q, int32_t chunk, void *out,
                                           int32_t out_is_fp32, void *ws, size_t ws_bytes,
                                           const recsa_debug *debug, recsa_stream_t stream);

/* Decode without any device allocation.  The RecSA paper has no counterpart to this
 * call; it exists for callers that cannot allocate device memory for a workspace:
 * hosts that give the library a fixed memory budget and own every allocation, serving
 * loops that forbid allocation after warm-up, or code that must not touch the
 * allocator while other work holds it.  Same inputs, outputs and results as
 * recsa_decode (no debug outputs); the RoPE table and error word live in a fixed
 * 256 KiB device array of the library, which every GPU that loads the library holds
 * until the process exits.
 *   - The first call made with a device current looks the array's address up on that
 *     device (and again after the device's context was re-created, e.g. by a reset);
 *     make that first call before any stream capture.
 *   - Every call rewrites the array (table for its own parameters, error word cleared),
 *     so calls whose GPU work overlaps (other streams, other threads) race: order them
 *     on one stream.
 *   - The array holds RoPE positions 0..510: configurations whose candidate lists can
 *     exceed 510 entries ((top_k + 1) * branching, bounded by the capacity) return
 *     RECSA_ERR_UNSUPPORTED with nothing launched.
 *   - Device-side checks are not reported: the error word is cleared by the next call. */
RECSA_API recsa_status recsa_decode_no_alloc(const recsa_params *params, const recsa_tree *tree, const void *q,
                                             int32_t num_queries, void *out, int32_t out_is_fp32,
                                             recsa_stream_t stream);

/* Synchronise `stream`, then read and clear the workspace's device error word and the
 * library's own word for the build and append kernels (which take no workspace).
 * Returns RECSA_OK, RECSA_ERR_DEVICE_CHECK (an index out of range, or a workspace
 * that was not initialised for the call), RECSA_ERR_TIMEOUT (a bounded wait ran
 * out: the attend kernels' none, the build and append kernels' wait on a tensor-core
 * product of the pooler, after which those keys are left unwritten), or
 * RECSA_ERR_CUDA. */
RECSA_API recsa_status recsa_check_device_errors(void *ws, recsa_stream_t stream);

/* Static name of a status code. */
RECSA_API const char *recsa_status_string(recsa_status status);

/* Thread-local description of the most recent failure in this thread ("" if none). */
RECSA_API const char *recsa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* RECSA_H */
