// Internal declarations shared by the CUDA translation units of libkvc.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "kvc.h"

namespace kvc {

constexpr int kPage = KVC_PAGE_SIZE;   // tokens per page

// Device error flags (bit mask written with atomicOr into the workspace).
constexpr uint32_t kErrBlockTable = 1u;
constexpr uint32_t kErrFormat = 2u;
constexpr uint32_t kErrContext = 4u;
constexpr uint32_t kErrTimeout = 8u;
constexpr uint32_t kErrRange = 16u;   // a query value outside the f16 range met an FP8 page

// Format of logical page j (length-L sequence): the high-precision format
// if the page holds any of the first `sink` tokens or any of the last
// `window` tokens, else the caller's tag for that older page.  Used by the
// host planner and by the decode kernels, so both always agree.
__host__ __device__ __forceinline__ int page_format(int j, int L, int sink, int window,
                                                    int hp, int older) {
  const int first = j * kPage;
  const int last_valid = ((j + 1) * kPage < L ? (j + 1) * kPage : L) - 1;
  return (first < sink || last_valid >= L - window) ? hp : older;
}

// ---------------------------------------------------------------- quantise
// page_ids[i] (or i when page_ids is NULL) names the source page of output
// page i; ids outside [0, n_src) skip that output page and set bit 1 of
// *flags (when flags is not NULL).
cudaError_t launch_quant_ternary(const void* src, const int32_t* page_ids, long long n_src, uint32_t* flags, int n,
                                 int hkv, int d, void* dst, float* gamma, cudaStream_t s);
cudaError_t launch_quant_fp8(const void* src, const int32_t* page_ids, long long n_src, uint32_t* flags, int n,
                             int hkv, int d, void* dst, float* scale, cudaStream_t s);
cudaError_t launch_copy_pages(const void* src, const int32_t* page_ids, long long n_src, uint32_t* flags, int n,
                              size_t page_bytes, void* dst, cudaStream_t s);
cudaError_t launch_dequant_ternary(const void* src, const float* gamma, const int32_t* page_ids, long long n_src,
                                   uint32_t* flags, int n, int hkv, int d, void* dst, cudaStream_t s);
cudaError_t launch_dequant_fp8(const void* src, const float* scale, const int32_t* page_ids, long long n_src,
                               uint32_t* flags, int n, int hkv, int d, void* dst, cudaStream_t s);

// exponent-split lossless codec of BF16 pages (exans.cu)
long long exans_slot_bytes(long long group_elems);
cudaError_t launch_exans_encode(const void* src, const int32_t* page_ids, long long n_src, uint32_t* flags, int n,
                                long long group_elems, void* ws, long long* offsets, void* dst, cudaStream_t s);
cudaError_t launch_exans_decode(const void* src, long long src_bytes, const long long* offsets, int n_blobs,
                                const int32_t* ids, int n, long long group_elems, void* dst, uint32_t* flags,
                                cudaStream_t s);
cudaError_t launch_promote(const kvc_paged_cache& cache, int32_t* block_table, uint8_t* older_fmt,
                           const int32_t* ctx, const int32_t* req_seq, const int32_t* req_page,
                           const int32_t* anchor_slot, int32_t* freed, uint32_t* flags, int n, int batch,
                           int hkv, int d, int max_pages, int sink, int window, int hp, int anchor,
                           cudaStream_t s);
cudaError_t launch_append_retier(const void* k_new, const void* v_new, const kvc_paged_cache& cache,
                                int32_t* block_table, uint8_t* older_fmt, const int32_t* ctx,
                                const int32_t* tern_slot, int32_t* freed, uint32_t* flags, int batch,
                                int hkv, int d, int max_pages, int sink, int window, int hp,
                                cudaStream_t s);

// ------------------------------------------------------------------ decode
struct DecodeParams {
  const __nv_bfloat16* q;
  kvc_paged_cache cache;
  const int32_t* block_table;
  const uint8_t* older_fmt;
  const int32_t* ctx;
  int B, Hq, Hkv, G, max_pages;
  int Bseq;                  // sequences per layer; B = layers * Bseq virtual sequences
                             // (virtual sequence b: layer b / Bseq, sequence b % Bseq;
                             // layer l's pool slots start at l * n_pages[format])
  int b_base;                // virtual sequence of this launch's entry 0, when a batch
                             // is decoded in several launches (q, out and tickets
                             // then point at that entry's rows)
  int sink, window, hp;
  float scale_log2;          // softmax_scale * log2(e)
  int tern_int;              // tensor-core kernel, GQA <= 4: ternary P.V on int8 MMAs
                             // (1: softmax per page pair; 2: per full entry), 0: f16
  int test_timeout;          // tensor-core kernel: make the first slot wait run out (failure tests)
  int n_splits, pages_per_split;
  float* out;
  uint32_t* err;             // device error word
  uint32_t* tickets;         // [B][Hkv] merge tickets
  float* partials;           // [B][Hkv][n_splits][G][D + 2]
};

struct DecodePlan {
  int kernel;                // kDecodeSimple, kDecodeTc or kDecodeUmma
  int n_splits;              // simple: splits per (sequence, KV head); tc: warps in the grid
  int pages_per_split;       // simple only
  int grid;                  // tc only: persistent CTAs
  int chunk;                 // tc only: virtual sequences per launch
  size_t ticket_offset, partial_offset, bytes;
};

constexpr int kDecodeSimple = 0, kDecodeTc = 1, kDecodeUmma = 2;

// Kernel choice, split-K plan and workspace layout for these shapes on the
// current device.
cudaError_t decode_plan(int batch, int hq, int hkv, int d, int max_pages, DecodePlan* plan);

cudaError_t launch_decode(const DecodeParams& p, int head_dim, const DecodePlan& plan, cudaStream_t s);
cudaError_t launch_decode_simple(const DecodeParams& p, int head_dim, cudaStream_t s);

// tensor-core kernel (decode_tc.cu)
// virtual sequences one launch of the tensor-core kernel takes (a larger
// batch is decoded in consecutive launches); 0 when these shapes do not fit
int tc_chunk(int hkv, int max_pages);
cudaError_t tc_grid(int batch, int d, int hq, int hkv, int* grid);
int tc_warps_per_cta(int hkv);
cudaError_t launch_decode_tc(const DecodeParams& p, int head_dim, int grid, int chunk, cudaStream_t s);

// tensor-memory (tcgen05) kernel (decode_umma.cu): two partial records per
// (CTA, sequence, KV head)
bool umma_supported(int batch, int d, int hkv, int max_pages);
int umma_heads_per_cta(int hkv);
cudaError_t umma_grid(int batch, int d, int hq, int hkv, int* grid);
cudaError_t launch_decode_umma(const DecodeParams& p, int head_dim, int grid, cudaStream_t s);

}  // namespace kvc
