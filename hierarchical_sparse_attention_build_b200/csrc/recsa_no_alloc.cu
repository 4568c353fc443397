// Decode for callers that cannot allocate device memory.
//
// recsa_decode takes its scratch (the RoPE cos/sin table and the device error word)
// from a workspace the caller allocates.  Some callers cannot do that: a host that
// hands the library a fixed memory budget and owns every allocation itself, a
// serving loop that forbids allocation once it has warmed up, or code that must not
// touch the allocator while other work holds it.  recsa_decode_no_alloc keeps that
// scratch in a fixed array of this file instead, so the call needs nothing beyond
// the caller's inputs and outputs.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "recsa.h"
#include "recsa_internal.h"

namespace recsa {
namespace {

// 256 KiB: a 256-byte header plus RoPE rows for positions 0..510 (512 bytes each).
constexpr size_t kStaticScratchBytes = 256 * 1024;

// Device scratch shared by every recsa_decode_no_alloc call on a device; it lives
// until the process exits.  Host code must not use this name as an address.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 128;
void *g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Unique id of the calling thread's current CUDA context (0 when there is none, or when
// the driver cannot say).  A device reset destroys the context, and the array with it;
// the next context gets a new id, so an address kept from the old one is never reused.
unsigned long long current_context_id() {
  using GetCurrent = int (*)(void **);
  using GetId = int (*)(void *, unsigned long long *);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(f);
  });
  void *ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != 0 || ctx == nullptr ||
      get_id(ctx, &id) != 0)
    return 0;
  return id;
}

// Device address of g_static_scratch for the current device, looked up with
// cudaGetSymbolAddress on the first call made with that device current and again only
// when the device's context has changed since (a reset).  Without a context id the
// address is looked up on every call.
recsa_status static_scratch(void **out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_error("RECSA_ERR_CUDA: cudaGetDevice: %s", cudaGetErrorString(e));
    return RECSA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    set_error("RECSA_ERR_UNSUPPORTED: device %d >= %d", dev, kMaxDevices);
    return RECSA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  const unsigned long long ctx = current_context_id();
  if (g_scratch_ptr[dev] == nullptr || ctx == 0 || g_scratch_ctx[dev] != ctx) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);  // also creates the context on a first call
    if (e != cudaSuccess || p == nullptr) {
      g_scratch_ptr[dev] = nullptr;
      set_error("RECSA_ERR_CUDA: cudaGetSymbolAddress of the static scratch: %s", cudaGetErrorString(e));
      return RECSA_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = current_context_id();
  }
  *out = g_scratch_ptr[dev];
  return RECSA_OK;
}

}  // namespace
}  // namespace recsa

extern "C" RECSA_API recsa_status recsa_decode_no_alloc(const recsa_params *params, const recsa_tree *tree,
                                                       const void *q, int32_t num_queries, void *out,
                                                       int32_t out_is_fp32, recsa_stream_t stream) {
  using namespace recsa;
  if (tree == nullptr) {
    set_error("RECSA_ERR_INVALID_ARGUMENT: tree is NULL");
    return RECSA_ERR_INVALID_ARGUMENT;
  }
  size_t need = 0;
  recsa_status s = recsa_workspace_size(params, tree->capacity, &need);  // validates params
  if (s != RECSA_OK) return s;
  if (need > kStaticScratchBytes) {
    set_error("RECSA_ERR_UNSUPPORTED: decode without allocation needs %zu bytes of scratch for this top_k, "
              "branching and capacity; the fixed scratch holds %zu (RoPE positions up to %zu)",
              need, kStaticScratchBytes, (kStaticScratchBytes - kWsHeader) / (kHalf * 8) - 1);
    return RECSA_ERR_UNSUPPORTED;
  }
  if (q == nullptr || out == nullptr || num_queries < 1 || tree->length < 1) {
    set_error("RECSA_ERR_INVALID_ARGUMENT: q or out is NULL, num_queries < 1 or length < 1");
    return RECSA_ERR_INVALID_ARGUMENT;
  }
  void *scratch = nullptr;
  s = static_scratch(&scratch);
  if (s != RECSA_OK) return s;
  // Every call rewrites the table and clears the error word for its own parameters:
  // the array keeps whatever the previous call left.
  const int rows = (int)((need - kWsHeader) / (kHalf * 8));
  const int rc = launch_rope_table(scratch, rows, (double)params->rope_base, stream);
  if (rc != 0) {
    set_error("RECSA_ERR_CUDA: rope table: %s", cudaGetErrorString((cudaError_t)rc));
    return RECSA_ERR_CUDA;
  }
  return recsa_decode(params, tree, q, num_queries, out, out_is_fp32, scratch, need, nullptr, stream);
}
