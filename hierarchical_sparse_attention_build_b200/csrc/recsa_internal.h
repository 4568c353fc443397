// Internal declarations shared by the host entry points (recsa_abi.cpp) and the
// kernel launchers (*.cu).  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>

#include "recsa.h"

namespace recsa {

constexpr int kD = RECSA_HEAD_DIM;     // head dim
constexpr int kHalf = kD / 2;          // RoPE pairs (i, i + 64)
constexpr int kRowBytes = kD * 2;      // one bf16 row
constexpr int kMaxLevels = RECSA_MAX_LEVELS;
constexpr int kMaxCand = RECSA_MAX_CANDIDATES;
constexpr int kDebugMaxK = 64;

// Workspace layout: a 256-byte header, then the RoPE table float2[rows][64].
constexpr size_t kWsHeader = 256;
constexpr uint32_t kWsMagic = 0x52534131u;  // "RSA1"
struct WsHeader {
  uint32_t err;         // device error bits (kErr*)
  uint32_t magic;       // kWsMagic once initialised
  int32_t table_rows;   // positions 0 .. table_rows-1
  float rope_base;      // base the table was computed for
};
constexpr uint32_t kErrIndex = 1u;    // an index fell outside its level
constexpr uint32_t kErrWs = 2u;       // workspace not initialised for this call
constexpr uint32_t kErrTimeout = 4u;  // a bounded wait ran out
constexpr uint32_t kErrCount = 8u;    // a candidate list outgrew its buffer

// Geometry of one tree (host-computed, passed by value to kernels).
struct TreeGeom {
  int32_t batch, hkv, b;
  int32_t levels_cap;                    // levels above the tokens at capacity
  int64_t capacity;
  int64_t slots[kMaxLevels + 1];         // nodes per (sequence, head) at level l for capacity (slots[0] = capacity)
  int64_t row_off[kMaxLevels + 1];       // arena row offset of level l
  int64_t span[kMaxLevels + 1];          // b^l, saturated at 2^62
};

struct Status {
  recsa_status code;
};

// Host helpers (recsa_abi.cpp)
void set_error(const char *fmt, ...);
int64_t ceil_div(int64_t a, int64_t b);
int levels_for(int64_t length, int b);  // T(length)

// Launchers (return cudaError_t as int; 0 = success)
int launch_rope_table(void *ws, int rows, double base, void *stream);
// Read and clear the build kernels' device error word (kErrTimeout when a wait on the tensor
// cores gave up); returns a cudaError_t.
int read_build_errors(uint32_t *bits);
int launch_build_level(const TreeGeom &g, const recsa_tree &t, int level, int64_t length, int64_t j0, int64_t j1,
                       void *stream);
int launch_append(const TreeGeom &g, const recsa_tree &t, const void *k_new, const void *v_new, int64_t at,
                  int chunk, void *stream);
// Append `chunk` tokens at slot `at` (at t.seq_len[s] when the tree has per-sequence lengths)
// and rebuild the nodes over them, all levels in one launch (a CTA per (sequence, head)
// walks up the levels).  levels = T of the longest new length.
int launch_extend(const TreeGeom &g, const recsa_tree &t, const void *k_new, const void *v_new, int64_t at,
                  int chunk, int levels, void *stream, uint32_t *err = nullptr);
// seq_len[s] += count for every sequence whose new length stays within `limit` (queued after
// the kernels that read the old lengths).
int launch_advance_lengths(int64_t *seq_len, int batch, int64_t count, int64_t limit, void *stream);

struct AttendLaunch {
  TreeGeom geom;
  recsa_tree tree;
  const void *q;
  void *out;
  int out_fp32;
  int num_queries;     // queries per sequence (decode) or chunk length (prefill)
  int64_t length;      // decode: L (queries at p = L); prefill: L before the chunk (query i at L + i)
  int causal;
  int group;           // G
  int top_k;
  float scale;
  void *ws;
  int table_rows_needed;
  int max_cand;        // candidate buffer size per level (multiple of 32)
  int cluster_size;    // 0 = automatic
  int kernel;          // 0 = automatic, 1 = CTA/cluster per tile, 2 = warp per tile
  const recsa_debug *debug;
};
int launch_attend(const AttendLaunch &a, void *stream);

}  // namespace recsa
