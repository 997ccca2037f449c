// Decode attention for callers that cannot allocate device memory.
//
// Some callers may not call cudaMalloc at all: code running inside a
// framework that owns every device allocation through its own pool, plugins
// loaded into a host process whose memory budget is fixed up front, or code
// paths that must not add an allocation (and its possible implicit
// synchronisation) to a latency-critical loop.  They still pass their own
// inputs and outputs, but cannot provide the split-K workspace that
// kvc_decode_attention_paged needs.  This entry point uses instead a
// file-scope device array of fixed size, which the library holds on every
// GPU that loads it until the process exits.
#include <mutex>

#include "kvc_internal.cuh"

namespace {

constexpr size_t kScratchBytes = KVC_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// The scratch itself.  In host code `g_scratch` names a host-side stand-in
// for this symbol, not a device address: kernels must be given the address
// obtained from cudaGetSymbolAddress below.
__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device, looked up once per
// device (with that device current) and cached.
kvc_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVC_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return KVC_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return KVC_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return KVC_OK;
}

}  // namespace

extern "C" {

kvc_status kvc_decode_attention_paged_noalloc(const void* q_bf16, const kvc_paged_cache* cache,
                                              const int32_t* block_table, const uint8_t* older_fmt,
                                              const int32_t* context_lens, int batch, int n_q_heads,
                                              int n_kv_heads, int head_dim, int page_size,
                                              int max_pages, int sink_tokens, int window_tokens,
                                              kvc_format hp_mode, float softmax_scale, float* out,
                                              kvc_stream_t stream) {
  // Validate every argument before anything is enqueued: with no workspace
  // the regular entry point checks them all and then reports only the
  // missing workspace (or returns KVC_OK at once for an empty batch).
  kvc_status st = kvc_decode_attention_paged(q_bf16, cache, block_table, older_fmt, context_lens,
                                             batch, n_q_heads, n_kv_heads, head_dim, page_size,
                                             max_pages, sink_tokens, window_tokens, hp_mode,
                                             softmax_scale, out, nullptr, 0, stream);
  if (st != KVC_ERR_WORKSPACE) return st;
  size_t need = 0;
  st = kvc_decode_workspace_size(batch, n_q_heads, n_kv_heads, head_dim, max_pages, &need);
  if (st != KVC_OK) return st;
  if (need > kScratchBytes) return KVC_ERR_WORKSPACE;   // shapes too large for the fixed scratch
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != KVC_OK) return st;
  // The scratch keeps whatever the previous call left; the regular entry
  // point clears the error word and the merge tickets on every call (one
  // cudaMemsetAsync on `stream`) and rewrites the partial states.
  return kvc_decode_attention_paged(q_bf16, cache, block_table, older_fmt, context_lens, batch,
                                    n_q_heads, n_kv_heads, head_dim, page_size, max_pages,
                                    sink_tokens, window_tokens, hp_mode, softmax_scale, out,
                                    scratch, kScratchBytes, stream);
}

}  // extern "C"
