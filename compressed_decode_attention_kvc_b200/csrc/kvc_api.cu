// The extern "C" boundary of libkvc: argument validation, the host page
// planner, the decode workspace layout and kernel dispatch.  No entry point
// allocates memory or synchronises (except kvc_decode_read_error, whose job
// is to read a device flag).
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "kvc_internal.cuh"

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool head_dim_ok(int d) { return d == 64 || d == 128 || d == 256; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

kvc_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KVC_OK : KVC_ERR_CUDA; }

// Shape checks common to the page codecs.
kvc_status check_codec(const void* src, const void* dst, int n, int page_size, int hkv, int d,
                       kvc_format mode, const float* scale) {
  if (n < 0 || hkv < 1) return KVC_ERR_INVALID_ARG;
  if (page_size != KVC_PAGE_SIZE || !head_dim_ok(d)) return KVC_ERR_UNSUPPORTED;
  if (mode != KVC_FMT_BF16 && mode != KVC_FMT_FP8_E4M3 && mode != KVC_FMT_TERNARY2)
    return KVC_ERR_INVALID_ARG;
  if (n == 0) return KVC_OK;
  if (!src || !dst) return KVC_ERR_INVALID_ARG;
  if (!aligned(src, 16) || !aligned(dst, 16)) return KVC_ERR_INVALID_ARG;
  if (mode != KVC_FMT_BF16 && (!scale || !aligned(scale, 4))) return KVC_ERR_INVALID_ARG;
  return KVC_OK;
}

}  // namespace

namespace kvc {

// The tensor-memory (tcgen05) decode kernel is the alternative
// implementation, measured slower than the register-sourced one on every
// workload here; it runs only when the environment variable
// KVC_DECODE_KERNEL is "tcgen05" (read once per process).
static bool umma_selected() {
  static const bool on = [] {
    const char* v = getenv("KVC_DECODE_KERNEL");
    return v != nullptr && strcmp(v, "tcgen05") == 0;
  }();
  return on;
}

// Ternary P.V of the tensor-core kernel at GQA <= 4: int8 MMAs with P in two
// exact digits, full entries with one softmax maximum test per entry (2,
// the default); the same per page pair (1, "pair"); or f16 MMAs with P as an
// f16 hi + lo pair (0, "f16").  Environment variable KVC_DECODE_TERNARY_PV,
// read once per process.
static int ternary_pv_mode() {
  static const int mode = [] {
    const char* v = getenv("KVC_DECODE_TERNARY_PV");
    if (v != nullptr && strcmp(v, "f16") == 0) return 0;
    if (v != nullptr && strcmp(v, "pair") == 0) return 1;
    return 2;
  }();
  return mode;
}

// Failure-detection tests: with KVC_TEST_DECODE_TIMEOUT=1 (read once per
// process) the tensor-core decode kernel arms its first ring slot for bytes
// no copy delivers, so its bounded waits run out and it sets device flag 8
// (read by kvc_decode_read_error); nothing faults or hangs, and the context
// stays usable.
static bool test_timeout() {
  static const bool on = [] {
    const char* v = getenv("KVC_TEST_DECODE_TIMEOUT");
    return v != nullptr && strcmp(v, "1") == 0;
  }();
  return on;
}

cudaError_t decode_plan(int batch, int hq, int hkv, int d, int max_pages, DecodePlan* plan) {
  const long long bg = (long long)batch * hkv;
  const int G = hq / hkv;
  const size_t record = (size_t)G * (d + 2) * sizeof(float);
  plan->chunk = 0;
  plan->ticket_offset = 256;
  plan->partial_offset = round_up(256 + (size_t)bg * 4, 256);
  if (umma_selected() && umma_supported(batch, d, hkv, max_pages)) {
    // persistent grid, one CTA of two warpgroup workers per SM; two records
    // (ternary, high precision) per (worker, pair) boundary
    int grid = 0;
    cudaError_t e = umma_grid(batch, d, hq, hkv, &grid);
    if (e != cudaSuccess) return e;
    plan->kernel = kDecodeUmma;
    plan->grid = grid;
    plan->n_splits = 2 * grid * umma_heads_per_cta(hkv);   // two warpgroup workers per CTA
    plan->pages_per_split = 0;
    plan->bytes = plan->partial_offset + 2 * ((size_t)plan->n_splits + (size_t)bg) * record;
    return cudaSuccess;
  }
  const int chunk = tc_chunk(hkv, max_pages);
  if (chunk >= 1) {
    // persistent grid, every warp a stream-K worker; one partial state per
    // (warp, pair) boundary: at most warps + pairs records per launch.  A
    // batch larger than `chunk` runs as consecutive launches that reuse the
    // records (each has its own tickets).
    const int per_launch = std::min(batch, chunk);
    int grid = 0;
    cudaError_t e = tc_grid(per_launch, d, hq, hkv, &grid);
    if (e != cudaSuccess) return e;
    plan->kernel = kDecodeTc;
    plan->grid = grid;
    plan->chunk = chunk;
    plan->n_splits = grid * tc_warps_per_cta(hkv);
    plan->pages_per_split = 0;
    plan->bytes = plan->partial_offset + ((size_t)plan->n_splits + (size_t)per_launch * hkv) * record;
    return cudaSuccess;
  }
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  // Split each (sequence, KV head) over pages so that about four CTAs per SM
  // are in flight, with at least 16 pages per split.
  long long splits = bg > 0 ? (4ll * sms + bg - 1) / bg : 1;
  const long long max_splits = std::max(1, (max_pages + 15) / 16);
  splits = std::max(1ll, std::min(splits, max_splits));
  const int pps = max_pages > 0 ? (int)((max_pages + splits - 1) / splits) : 1;
  splits = max_pages > 0 ? (max_pages + pps - 1) / pps : 1;
  plan->kernel = kDecodeSimple;
  plan->grid = 0;
  plan->n_splits = (int)splits;
  plan->pages_per_split = pps;
  plan->bytes = plan->partial_offset + (size_t)bg * splits * record;
  return cudaSuccess;
}

cudaError_t launch_decode(const DecodeParams& p, int head_dim, const DecodePlan& plan, cudaStream_t s) {
  if (plan.kernel == kDecodeUmma) return launch_decode_umma(p, head_dim, plan.grid, s);
  if (plan.kernel == kDecodeTc) return launch_decode_tc(p, head_dim, plan.grid, plan.chunk, s);
  return launch_decode_simple(p, head_dim, s);
}

}  // namespace kvc

extern "C" {

const char* kvc_status_string(kvc_status status) {
  switch (status) {
    case KVC_OK: return "ok";
    case KVC_ERR_INVALID_ARG: return "invalid argument";
    case KVC_ERR_UNSUPPORTED: return "unsupported shape";
    case KVC_ERR_WORKSPACE: return "workspace missing or too small";
    case KVC_ERR_CUDA: return "CUDA error";
    case KVC_ERR_DEVICE_CHECK: return "device-side check failed";
    case KVC_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

int kvc_layout_version(void) { return KVC_LAYOUT_VERSION; }

kvc_status kvc_quantize_pack_pages(const void* src_bf16, const int32_t* page_ids, int n,
                                   int page_size, int n_kv_heads, int head_dim, kvc_format mode,
                                   void* dst, float* dst_scale, int64_t n_src_pages,
                                   uint32_t* device_flags, kvc_stream_t stream) {
  kvc_status st = check_codec(src_bf16, dst, n, page_size, n_kv_heads, head_dim, mode, dst_scale);
  if (st != KVC_OK || n == 0) return st;
  if (n_src_pages < 1 || (!page_ids && n_src_pages < n)) return KVC_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (mode) {
    case KVC_FMT_TERNARY2:
      return from_cuda(kvc::launch_quant_ternary(src_bf16, page_ids, n_src_pages, device_flags, n, n_kv_heads,
                                                 head_dim, dst, dst_scale, s));
    case KVC_FMT_FP8_E4M3:
      return from_cuda(kvc::launch_quant_fp8(src_bf16, page_ids, n_src_pages, device_flags, n, n_kv_heads, head_dim,
                                             dst, dst_scale, s));
    default:
      return from_cuda(kvc::launch_copy_pages(src_bf16, page_ids, n_src_pages, device_flags, n,
                                              (size_t)n_kv_heads * KVC_PAGE_SIZE * head_dim * 2, dst, s));
  }
}

kvc_status kvc_dequantize_pages(const void* src, const float* src_scale, const int32_t* page_ids,
                                int n, int page_size, int n_kv_heads, int head_dim,
                                kvc_format mode, void* dst_bf16, int64_t n_src_pages, uint32_t* device_flags,
                                kvc_stream_t stream) {
  kvc_status st = check_codec(src, dst_bf16, n, page_size, n_kv_heads, head_dim, mode, src_scale);
  if (st != KVC_OK || n == 0) return st;
  if (n_src_pages < 1 || (!page_ids && n_src_pages < n)) return KVC_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (mode) {
    case KVC_FMT_TERNARY2:
      return from_cuda(kvc::launch_dequant_ternary(src, src_scale, page_ids, n_src_pages, device_flags, n, n_kv_heads,
                                                   head_dim, dst_bf16, s));
    case KVC_FMT_FP8_E4M3:
      return from_cuda(kvc::launch_dequant_fp8(src, src_scale, page_ids, n_src_pages, device_flags, n, n_kv_heads,
                                               head_dim, dst_bf16, s));
    default:
      return from_cuda(kvc::launch_copy_pages(src, page_ids, n_src_pages, device_flags, n,
                                              (size_t)n_kv_heads * KVC_PAGE_SIZE * head_dim * 2, dst_bf16, s));
  }
}

kvc_status kvc_append_retier(const void* k_new_bf16, const void* v_new_bf16,
                             const kvc_paged_cache* cache, int32_t* block_table, uint8_t* older_fmt,
                             const int32_t* context_lens, const int32_t* ternary_slot,
                             int32_t* freed_hp_slot, uint32_t* device_flags, int batch, int n_kv_heads,
                             int head_dim, int page_size, int max_pages, int sink_tokens,
                             int window_tokens, kvc_format hp_mode, kvc_stream_t stream) {
  if (batch < 0 || n_kv_heads < 1 || max_pages < 1 || sink_tokens < 0 || window_tokens < 1)
    return KVC_ERR_INVALID_ARG;
  if (page_size != KVC_PAGE_SIZE || !head_dim_ok(head_dim)) return KVC_ERR_UNSUPPORTED;
  if (hp_mode != KVC_FMT_BF16 && hp_mode != KVC_FMT_FP8_E4M3) return KVC_ERR_INVALID_ARG;
  if (!cache) return KVC_ERR_INVALID_ARG;
  if (batch == 0) return KVC_OK;
  if (!k_new_bf16 || !v_new_bf16 || !block_table || !context_lens || !ternary_slot || !freed_hp_slot)
    return KVC_ERR_INVALID_ARG;
  if (!aligned(k_new_bf16, 16) || !aligned(v_new_bf16, 16)) return KVC_ERR_INVALID_ARG;
  const bool bf = hp_mode == KVC_FMT_BF16;
  const void* hk = bf ? cache->k_bf16 : cache->k_fp8;
  const void* hv = bf ? cache->v_bf16 : cache->v_fp8;
  if (!hk || !hv || !aligned(hk, 16) || !aligned(hv, 16)) return KVC_ERR_INVALID_ARG;
  if (!bf && (!cache->k_fp8_scale || !cache->v_fp8_scale)) return KVC_ERR_INVALID_ARG;
  if (cache->n_pages[2] > 0 &&
      (!cache->k_tern || !cache->v_tern || !cache->k_gamma || !cache->v_gamma ||
       !aligned(cache->k_tern, 16) || !aligned(cache->v_tern, 16)))
    return KVC_ERR_INVALID_ARG;
  return from_cuda(kvc::launch_append_retier(k_new_bf16, v_new_bf16, *cache, block_table, older_fmt,
                                             context_lens, ternary_slot, freed_hp_slot, device_flags,
                                             batch, n_kv_heads, head_dim, max_pages, sink_tokens,
                                             window_tokens, hp_mode,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

kvc_status kvc_promote_pages(const kvc_paged_cache* cache, int32_t* block_table, uint8_t* older_fmt,
                             const int32_t* context_lens, const int32_t* req_seq, const int32_t* req_page,
                             const int32_t* anchor_slot, int n_requests, int32_t* freed_ternary_slot,
                             uint32_t* device_flags, int batch, int n_kv_heads, int head_dim, int page_size,
                             int max_pages, int sink_tokens, int window_tokens, kvc_format hp_mode,
                             kvc_format anchor_fmt, kvc_stream_t stream) {
  if (n_requests < 0 || batch < 0 || n_kv_heads < 1 || max_pages < 1 || sink_tokens < 0 || window_tokens < 0)
    return KVC_ERR_INVALID_ARG;
  if (page_size != KVC_PAGE_SIZE || !head_dim_ok(head_dim)) return KVC_ERR_UNSUPPORTED;
  if (hp_mode != KVC_FMT_BF16 && hp_mode != KVC_FMT_FP8_E4M3) return KVC_ERR_INVALID_ARG;
  if (anchor_fmt != KVC_FMT_BF16 && anchor_fmt != KVC_FMT_FP8_E4M3) return KVC_ERR_INVALID_ARG;
  if (!cache) return KVC_ERR_INVALID_ARG;
  if (n_requests == 0) return KVC_OK;
  if ((long long)batch * max_pages > 0x7fffffffll) return KVC_ERR_UNSUPPORTED;
  if (!block_table || !older_fmt || !context_lens || !req_seq || !req_page || !anchor_slot ||
      !freed_ternary_slot)
    return KVC_ERR_INVALID_ARG;
  const bool bf = anchor_fmt == KVC_FMT_BF16;
  const void* ak = bf ? cache->k_bf16 : cache->k_fp8;
  const void* av = bf ? cache->v_bf16 : cache->v_fp8;
  if (cache->n_pages[anchor_fmt] > 0 && (!ak || !av || !aligned(ak, 16) || !aligned(av, 16)))
    return KVC_ERR_INVALID_ARG;
  if (!bf && cache->n_pages[anchor_fmt] > 0 && (!cache->k_fp8_scale || !cache->v_fp8_scale))
    return KVC_ERR_INVALID_ARG;
  if (cache->n_pages[KVC_FMT_TERNARY2] > 0 &&
      (!cache->k_tern || !cache->v_tern || !cache->k_gamma || !cache->v_gamma ||
       !aligned(cache->k_tern, 16) || !aligned(cache->v_tern, 16)))
    return KVC_ERR_INVALID_ARG;
  return from_cuda(kvc::launch_promote(*cache, block_table, older_fmt, context_lens, req_seq, req_page,
                                       anchor_slot, freed_ternary_slot, device_flags, n_requests, batch,
                                       n_kv_heads, head_dim, max_pages, sink_tokens, window_tokens, hp_mode,
                                       anchor_fmt, reinterpret_cast<cudaStream_t>(stream)));
}

// values of one page of one pool, or -1 when outside the codec's range
static long long exans_group_elems(int page_size, int n_kv_heads, int head_dim) {
  if (page_size != KVC_PAGE_SIZE || !head_dim_ok(head_dim) || n_kv_heads < 1) return -1;
  const long long n = (long long)n_kv_heads * KVC_PAGE_SIZE * head_dim;
  return n <= (1ll << 22) ? n : -1;
}

kvc_status kvc_exans_workspace_size(int n, int page_size, int n_kv_heads, int head_dim, size_t* bytes) {
  if (!bytes || n < 0) return KVC_ERR_INVALID_ARG;
  const long long N = exans_group_elems(page_size, n_kv_heads, head_dim);
  if (N < 0) return KVC_ERR_UNSUPPORTED;
  *bytes = (size_t)n * (size_t)kvc::exans_slot_bytes(N);
  return KVC_OK;
}

kvc_status kvc_exans_encode(const void* src_bf16, const int32_t* page_ids, int n, int page_size,
                            int n_kv_heads, int head_dim, void* workspace, size_t workspace_bytes, void* dst,
                            size_t dst_bytes, int64_t* offsets, int64_t n_src_pages, uint32_t* device_flags,
                            kvc_stream_t stream) {
  if (n < 0 || n > (1 << 24)) return KVC_ERR_INVALID_ARG;
  const long long N = exans_group_elems(page_size, n_kv_heads, head_dim);
  if (N < 0) return KVC_ERR_UNSUPPORTED;
  if (!offsets) return KVC_ERR_INVALID_ARG;
  if (n == 0) return from_cuda(cudaMemsetAsync(offsets, 0, sizeof(int64_t), reinterpret_cast<cudaStream_t>(stream)));
  if (!src_bf16 || !dst || !aligned(src_bf16, 16) || !aligned(dst, 16) || !aligned(offsets, 8))
    return KVC_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 16) || workspace_bytes < (size_t)n * (size_t)kvc::exans_slot_bytes(N))
    return KVC_ERR_WORKSPACE;
  if (dst_bytes < (size_t)n * (size_t)(64 + 2 * N)) return KVC_ERR_INVALID_ARG;
  if (n_src_pages < 1 || (!page_ids && n_src_pages < n)) return KVC_ERR_INVALID_ARG;
  return from_cuda(kvc::launch_exans_encode(src_bf16, page_ids, n_src_pages, device_flags, n, N, workspace,
                                            reinterpret_cast<long long*>(offsets), dst,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

kvc_status kvc_exans_decode(const void* src, size_t src_bytes, const int64_t* offsets, int n_blobs,
                            const int32_t* blob_ids, int n, int page_size, int n_kv_heads, int head_dim,
                            void* dst_bf16, uint32_t* device_flags, kvc_stream_t stream) {
  if (n < 0 || n_blobs < 0) return KVC_ERR_INVALID_ARG;
  const long long N = exans_group_elems(page_size, n_kv_heads, head_dim);
  if (N < 0) return KVC_ERR_UNSUPPORTED;
  if (n == 0) return KVC_OK;
  if (!src || !offsets || !dst_bf16 || !aligned(src, 16) || !aligned(dst_bf16, 16) || !aligned(offsets, 8))
    return KVC_ERR_INVALID_ARG;
  return from_cuda(kvc::launch_exans_decode(src, (long long)src_bytes, reinterpret_cast<const long long*>(offsets),
                                            n_blobs, blob_ids, n, N, dst_bf16, device_flags,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

kvc_status kvc_plan_paged_cache(const int32_t* context_lens, int batch, int max_pages,
                                int page_size, int sink_tokens, int window_tokens,
                                kvc_format hp_mode, const uint8_t* older_fmt,
                                const float* slot_key, int32_t* block_table, uint8_t* page_fmt,
                                int32_t* pool_pages, int32_t* pool_src_ids) {
  if (batch < 0 || max_pages < 0 || sink_tokens < 0 || window_tokens < 0) return KVC_ERR_INVALID_ARG;
  if (page_size != KVC_PAGE_SIZE) return KVC_ERR_UNSUPPORTED;
  if (hp_mode != KVC_FMT_BF16 && hp_mode != KVC_FMT_FP8_E4M3) return KVC_ERR_INVALID_ARG;
  if (!pool_pages) return KVC_ERR_INVALID_ARG;
  const long long total = (long long)batch * max_pages;
  if (total > 0x7fffffffll) return KVC_ERR_UNSUPPORTED;
  if (total > 0 && (!context_lens || !block_table || !page_fmt || !pool_src_ids))
    return KVC_ERR_INVALID_ARG;
  for (int b = 0; b < batch; ++b)
    if (context_lens[b] < 0 || (long long)context_lens[b] > (long long)max_pages * KVC_PAGE_SIZE)
      return KVC_ERR_INVALID_ARG;
  if (older_fmt)
    for (long long i = 0; i < total; ++i)
      if (older_fmt[i] > KVC_FMT_TERNARY2) return KVC_ERR_INVALID_ARG;

  std::vector<int32_t> members[3];
  for (long long i = 0; i < total; ++i) {
    block_table[i] = 0;
    page_fmt[i] = 255;
  }
  for (int b = 0; b < batch; ++b) {
    const int L = context_lens[b];
    const int np = (L + KVC_PAGE_SIZE - 1) / KVC_PAGE_SIZE;
    for (int j = 0; j < np; ++j) {
      const int32_t id = b * max_pages + j;
      const int older = older_fmt ? older_fmt[id] : KVC_FMT_TERNARY2;
      const int f = kvc::page_format(j, L, sink_tokens, window_tokens, hp_mode, older);
      page_fmt[id] = (uint8_t)f;
      members[f].push_back(id);
    }
  }
  int32_t offset = 0;
  for (int f = 0; f < 3; ++f) {
    std::vector<int32_t>& m = members[f];
    if (slot_key)
      std::stable_sort(m.begin(), m.end(), [slot_key](int32_t a, int32_t c) {
        return slot_key[a] < slot_key[c];
      });
    for (size_t slot = 0; slot < m.size(); ++slot) {
      block_table[m[slot]] = (int32_t)slot;
      pool_src_ids[offset + slot] = m[slot];
    }
    pool_pages[f] = (int32_t)m.size();
    offset += (int32_t)m.size();
  }
  return KVC_OK;
}

kvc_status kvc_decode_workspace_size(int batch, int n_q_heads, int n_kv_heads, int head_dim,
                                     int max_pages, size_t* bytes) {
  if (!bytes || batch < 0 || max_pages < 0 || n_kv_heads < 1 || n_q_heads < 1) return KVC_ERR_INVALID_ARG;
  if (n_q_heads % n_kv_heads) return KVC_ERR_INVALID_ARG;
  if (!head_dim_ok(head_dim) || n_q_heads / n_kv_heads > 8) return KVC_ERR_UNSUPPORTED;
  kvc::DecodePlan plan;
  cudaError_t e = kvc::decode_plan(batch, n_q_heads, n_kv_heads, head_dim, max_pages, &plan);
  if (e != cudaSuccess) return KVC_ERR_CUDA;
  *bytes = plan.bytes;
  return KVC_OK;
}

kvc_status kvc_decode_plan_info(int batch, int n_q_heads, int n_kv_heads, int head_dim, int max_pages,
                                int32_t* kernel, int32_t* launches) {
  if (!kernel || !launches || batch < 0 || max_pages < 0 || n_kv_heads < 1 || n_q_heads < 1)
    return KVC_ERR_INVALID_ARG;
  if (n_q_heads % n_kv_heads) return KVC_ERR_INVALID_ARG;
  if (!head_dim_ok(head_dim) || n_q_heads / n_kv_heads > 8) return KVC_ERR_UNSUPPORTED;
  kvc::DecodePlan plan;
  if (kvc::decode_plan(batch, n_q_heads, n_kv_heads, head_dim, max_pages, &plan) != cudaSuccess)
    return KVC_ERR_CUDA;
  *kernel = plan.kernel == kvc::kDecodeUmma ? KVC_DECODE_KERNEL_TCGEN05
            : plan.kernel == kvc::kDecodeTc ? KVC_DECODE_KERNEL_MMA : KVC_DECODE_KERNEL_CUDA_CORE;
  if (batch == 0) *launches = 0;
  else if (plan.kernel == kvc::kDecodeTc) *launches = (batch + plan.chunk - 1) / plan.chunk;
  else *launches = 1;
  return KVC_OK;
}

kvc_status kvc_decode_attention_paged(const void* q_bf16, const kvc_paged_cache* cache,
                                      const int32_t* block_table, const uint8_t* older_fmt,
                                      const int32_t* context_lens, int batch, int n_q_heads,
                                      int n_kv_heads, int head_dim, int page_size, int max_pages,
                                      int sink_tokens, int window_tokens, kvc_format hp_mode,
                                      float softmax_scale, float* out, void* workspace,
                                      size_t workspace_bytes, kvc_stream_t stream) {
  return kvc_decode_attention_paged_layers(q_bf16, cache, block_table, older_fmt, context_lens, 1, batch,
                                           n_q_heads, n_kv_heads, head_dim, page_size, max_pages,
                                           sink_tokens, window_tokens, hp_mode, softmax_scale, out,
                                           workspace, workspace_bytes, stream);
}

kvc_status kvc_decode_attention_paged_layers(const void* q_bf16, const kvc_paged_cache* cache,
                                             const int32_t* block_table, const uint8_t* older_fmt,
                                             const int32_t* context_lens, int n_layers, int batch,
                                             int n_q_heads, int n_kv_heads, int head_dim, int page_size,
                                             int max_pages, int sink_tokens, int window_tokens,
                                             kvc_format hp_mode, float softmax_scale, float* out,
                                             void* workspace, size_t workspace_bytes, kvc_stream_t stream) {
  if (batch < 0 || max_pages < 0 || n_kv_heads < 1 || n_q_heads < 1 || sink_tokens < 0 ||
      window_tokens < 0 || n_layers < 1)
    return KVC_ERR_INVALID_ARG;
  if ((long long)n_layers * batch > (1ll << 30)) return KVC_ERR_INVALID_ARG;
  const int seqs = batch;        // per layer
  batch = n_layers * batch;      // virtual sequences (layer-major)
  if (n_q_heads % n_kv_heads) return KVC_ERR_INVALID_ARG;
  if (page_size != KVC_PAGE_SIZE || !head_dim_ok(head_dim) || n_q_heads / n_kv_heads > 8)
    return KVC_ERR_UNSUPPORTED;
  if (hp_mode != KVC_FMT_BF16 && hp_mode != KVC_FMT_FP8_E4M3) return KVC_ERR_INVALID_ARG;
  if (batch == 0) return KVC_OK;
  if (!q_bf16 || !cache || !block_table || !context_lens || !out) return KVC_ERR_INVALID_ARG;
  if (!aligned(q_bf16, 16) || !aligned(out, 16)) return KVC_ERR_INVALID_ARG;
  for (int f = 0; f < 3; ++f) {
    if (cache->n_pages[f] < 0) return KVC_ERR_INVALID_ARG;
    // group indices (layer * n_pages + slot) * Hkv + head are 32-bit in the kernels
    if ((long long)n_layers * cache->n_pages[f] * n_kv_heads >= (1ll << 31)) return KVC_ERR_UNSUPPORTED;
  }
  if (cache->n_pages[KVC_FMT_BF16] > 0 &&
      (!cache->k_bf16 || !cache->v_bf16 || !aligned(cache->k_bf16, 16) || !aligned(cache->v_bf16, 16)))
    return KVC_ERR_INVALID_ARG;
  if (cache->n_pages[KVC_FMT_FP8_E4M3] > 0 &&
      (!cache->k_fp8 || !cache->v_fp8 || !cache->k_fp8_scale || !cache->v_fp8_scale ||
       !aligned(cache->k_fp8, 16) || !aligned(cache->v_fp8, 16)))
    return KVC_ERR_INVALID_ARG;
  if (cache->n_pages[KVC_FMT_TERNARY2] > 0 &&
      (!cache->k_tern || !cache->v_tern || !cache->k_gamma || !cache->v_gamma ||
       !aligned(cache->k_tern, 16) || !aligned(cache->v_tern, 16)))
    return KVC_ERR_INVALID_ARG;

  kvc::DecodePlan plan;
  if (kvc::decode_plan(batch, n_q_heads, n_kv_heads, head_dim, max_pages, &plan) != cudaSuccess)
    return KVC_ERR_CUDA;
  if (!workspace || workspace_bytes < plan.bytes || !aligned(workspace, 256)) return KVC_ERR_WORKSPACE;
  // error word and merge tickets start at zero on every call, so a call that
  // gave up on a wait (and left tickets behind) cannot poison the next one
  if (cudaMemsetAsync(workspace, 0, plan.partial_offset, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KVC_ERR_CUDA;

  kvc::DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(q_bf16);
  p.cache = *cache;
  p.block_table = block_table;
  p.older_fmt = older_fmt;
  p.ctx = context_lens;
  p.B = batch;
  p.Bseq = seqs;
  p.b_base = 0;
  p.Hq = n_q_heads;
  p.Hkv = n_kv_heads;
  p.G = n_q_heads / n_kv_heads;
  p.max_pages = max_pages;
  p.sink = sink_tokens;
  p.window = window_tokens;
  p.hp = hp_mode;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)head_dim);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.tern_int = kvc::ternary_pv_mode();
  p.test_timeout = kvc::test_timeout() ? 1 : 0;
  p.n_splits = plan.n_splits;
  p.pages_per_split = plan.pages_per_split;
  p.out = out;
  char* ws = static_cast<char*>(workspace);
  p.err = reinterpret_cast<uint32_t*>(ws);
  p.tickets = reinterpret_cast<uint32_t*>(ws + plan.ticket_offset);
  p.partials = reinterpret_cast<float*>(ws + plan.partial_offset);
  return from_cuda(kvc::launch_decode(p, head_dim, plan, reinterpret_cast<cudaStream_t>(stream)));
}

kvc_status kvc_decode_read_error(void* workspace, int batch, int n_q_heads, int n_kv_heads,
                                 int head_dim, int max_pages, uint32_t* flags,
                                 kvc_stream_t stream) {
  (void)batch; (void)n_q_heads; (void)n_kv_heads; (void)head_dim; (void)max_pages;
  if (!workspace || !flags) return KVC_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return KVC_ERR_CUDA;
  if (cudaMemcpy(flags, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
    return KVC_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), s) != cudaSuccess) return KVC_ERR_CUDA;
  return from_cuda(cudaStreamSynchronize(s));
}

}  // extern "C"
