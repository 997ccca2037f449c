// Page codecs: ternary quantise+pack, FP8 e4m3 page quantise, BF16 page
// copy, and the two dequantisers.
//
// Ternary follows "Show HN: Vantage-V-AI" (newshot.cc), section "Core
// architecture": ternary {-1, 0, +1} codes with the absmean scale
// gamma = mean(|X|) (BitNet b1.58), 4 codes per byte; here gamma is taken per
// (page, KV head) group.  FP8 follows the same page's FP8 streaming mode
// (section "Quick start", quant_mode = "fp8") and Minima-KV's FP8 recent tier
// ("Recent, Anchor and Stale"), with one scale per page.
//
// All kernels are HBM-streaming kernels: 16-byte loads and stores, one warp
// per (page, head) group for the ternary codec so that a group's gamma is a
// warp reduction held entirely in registers.
#include "kvc_internal.cuh"

namespace kvc {
namespace {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Read-once streaming load (no L1 allocation).
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float abs_sum8(const uint4& v) {
  // pairwise tree over the 8 values of one 16-byte chunk
  const float a0 = fabsf(bf16_lo(v.x)), a1 = fabsf(bf16_hi(v.x));
  const float a2 = fabsf(bf16_lo(v.y)), a3 = fabsf(bf16_hi(v.y));
  const float a4 = fabsf(bf16_lo(v.z)), a5 = fabsf(bf16_hi(v.z));
  const float a6 = fabsf(bf16_lo(v.w)), a7 = fabsf(bf16_hi(v.w));
  return ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
}

// 2-bit field of one value: 01 if x > t, 11 if x < -t, else 00.
__device__ __forceinline__ uint32_t tern_field(float x, float t) {
  return x > t ? 1u : (x < -t ? 3u : 0u);
}

__device__ __forceinline__ uint32_t tern_word16(const uint4& v, float t) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    out |= tern_field(bf16_lo(w[k]), t) << (4 * k);
    out |= tern_field(bf16_hi(w[k]), t) << (4 * k + 2);
  }
  return out;
}

// One warp per (page, head) group of 16*D bf16 values = 2*D chunks of 16 B;
// at head_dim 256 four warps share a group (each holds 2 KB in registers:
// more, smaller parts keep more loads in flight per SM, 72 -> 76 % of HBM
// measured) and add their partial sums through shared memory.  Lane l owns
// chunks l, l+32, ... of its warp's part: every load and store instruction
// of the warp is contiguous.  gamma is a pairwise tree (per chunk, across the
// lane's chunks, across lanes, across the parts): depth log2(16*D) <= 12, so
// its float32 relative error stays below 12 * 2^-24.
// Source page of output page i, or -1 when page_ids[i] lies outside
// [0, n_src): the caller skips that output page and flag 1 is raised.
__device__ __forceinline__ long long src_page(const int32_t* __restrict__ ids, long long i, long long n_src,
                                              uint32_t* flags) {
  const long long sp = ids ? (long long)__ldg(ids + i) : i;
  if (sp < 0 || sp >= n_src) {
    if (flags) atomicOr(flags, 1u);
    return -1;
  }
  return sp;
}

template <int D>
__global__ void __launch_bounds__(256) quant_ternary_kernel(const uint4* __restrict__ src,
                                                            const int32_t* __restrict__ page_ids,
                                                            long long n_src, uint32_t* flags,
                                                            long long n_groups, int hkv,
                                                            uint16_t* __restrict__ dst,
                                                            float* __restrict__ gamma) {
  constexpr int WPG = D > 128 ? 4 : 1;      // warps per group
  constexpr int NC = D / 16 / WPG;          // chunks per lane
  __shared__ float red[8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int part = warp % WPG;
  const long long grp = (long long)blockIdx.x * (8 / WPG) + warp / WPG;
  bool valid = grp < n_groups;
  const uint4* s = src;
  if (valid) {
    const long long i = grp / hkv;
    const int h = (int)(grp - i * hkv);
    const long long sp = src_page(page_ids, i, n_src, flags);
    valid = sp >= 0;
    s = src + (sp * hkv + h) * (2 * D) + part * (NC * 32);
  }

  uint4 v[NC];
  float sum = 0.f;
  if (valid) {
#pragma unroll
    for (int c = 0; c < NC; ++c) v[c] = ld_stream(s + c * 32 + lane);
    float pt[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) pt[c] = abs_sum8(v[c]);
#pragma unroll
    for (int w = 1; w < NC; w <<= 1)
#pragma unroll
      for (int c = 0; c + w < NC; c += 2 * w) pt[c] += pt[c + w];
    sum = pt[0];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  }
  if constexpr (WPG > 1) {
    if (lane == 0) red[warp] = sum;
    __syncthreads();
    const int w0 = warp - part;
    sum = (red[w0] + red[w0 + 1]) + (red[w0 + 2] + red[w0 + 3]);   // same order in all four warps
  }
  if (!valid) return;

  const float g = sum * (1.0f / (16 * D));  // exact: a power of two
  const float t = 0.5f * g;
  uint16_t* out = dst + grp * (2 * D) + part * (NC * 32);   // 4*D bytes per group
#pragma unroll
  for (int c = 0; c < NC; ++c) out[c * 32 + lane] = (uint16_t)tern_word16(v[c], t);
  if (lane == 0 && part == 0) gamma[grp] = g;
}

// One CTA per page: amax over the whole page (all heads), then
// e = RNE-satfinite-e4m3(x * (448 / amax)).  The second pass re-reads the
// page from L2 (a page is at most a few hundred KB), so DRAM sees it once.
__global__ void __launch_bounds__(256) quant_fp8_kernel(const uint4* __restrict__ src,
                                                        const int32_t* __restrict__ page_ids,
                                                        long long n_src, uint32_t* flags,
                                                        int chunks_per_page,
                                                        uint2* __restrict__ dst,
                                                        float* __restrict__ scale) {
  __shared__ float red[8];
  const long long i = blockIdx.x;
  const long long sp = src_page(page_ids, i, n_src, flags);
  if (sp < 0) return;                       // uniform over the CTA
  const uint4* s = src + sp * chunks_per_page;
  float amax = 0.f;
  for (int c = threadIdx.x; c < chunks_per_page; c += 256) {
    const uint4 v = __ldg(s + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k)
      amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[k])), fabsf(bf16_hi(w[k]))));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int k = 1; k < 8; ++k) amax = fmaxf(amax, red[k]);

  const float sc = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  const float inv = amax > 0.f ? __fdiv_rn(448.0f, amax) : 1.0f;
  uint2* d = dst + i * chunks_per_page;
  for (int c = threadIdx.x; c < chunks_per_page; c += 256) {
    const uint4 v = __ldg(s + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 y = make_float2(__fmul_rn(bf16_lo(w[k]), inv), __fmul_rn(bf16_hi(w[k]), inv));
      const uint32_t e2 = __nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3);  // .x -> low byte
      packed[k >> 1] |= e2 << (16 * (k & 1));
    }
    d[c] = make_uint2(packed[0], packed[1]);
  }
  if (threadIdx.x == 0) scale[i] = sc;
}

// Single-pass FP8 page quantise for pages of WPP * 32 * CPL chunks (16 B
// each): WPP warps per page, CPL chunks per lane held in registers, so the
// page is read from DRAM once and never re-read; 8 / WPP pages per CTA.  The amax
// is a warp reduction (and a shared-memory one across the page's warps);
// the encode is the same float32 arithmetic as quant_fp8_kernel.
template <int WPP, int CPL>
__global__ void __launch_bounds__(256, 3) quant_fp8_reg_kernel(const uint4* __restrict__ src,
                                                            const int32_t* __restrict__ page_ids,
                                                            long long n_src, uint32_t* flags, int n,
                                                            uint2* __restrict__ dst, float* __restrict__ scale) {
  constexpr int CPP = WPP * 32 * CPL;        // chunks per page
  __shared__ float red[8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int part = warp % WPP;
  const long long i = (long long)blockIdx.x * (8 / WPP) + warp / WPP;
  bool valid = i < n;
  uint4 v[CPL];
  float amax = 0.f;
  const long long sp = valid ? src_page(page_ids, i, n_src, flags) : -1;
  valid = sp >= 0;
  if (valid) {
    const uint4* s = src + sp * CPP + part * (32 * CPL);
#pragma unroll
    for (int c = 0; c < CPL; ++c) v[c] = ld_stream(s + c * 32 + lane);
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      const uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
      for (int k = 0; k < 4; ++k)
        amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[k])), fabsf(bf16_hi(w[k]))));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  }
  if constexpr (WPP > 1) {
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    const int w0 = warp - part;
#pragma unroll
    for (int k = 0; k < WPP; ++k) amax = fmaxf(amax, red[w0 + k]);
  }
  if (!valid) return;
  const float sc = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  const float inv = amax > 0.f ? __fdiv_rn(448.0f, amax) : 1.0f;
  uint2* d = dst + i * CPP + part * (32 * CPL);
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    const uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 y = make_float2(__fmul_rn(bf16_lo(w[k]), inv), __fmul_rn(bf16_hi(w[k]), inv));
      const uint32_t e2 = __nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3);  // .x -> low byte
      packed[k >> 1] |= e2 << (16 * (k & 1));
    }
    d[c * 32 + lane] = make_uint2(packed[0], packed[1]);
  }
  if (lane == 0 && part == 0) scale[i] = sc;
}

__global__ void __launch_bounds__(256) copy_pages_kernel(const uint4* __restrict__ src,
                                                         const int32_t* __restrict__ page_ids,
                                                         long long n_src, uint32_t* flags,
                                                         long long n_chunks, long long cpp,
                                                         uint4* __restrict__ dst) {
  for (long long c = (long long)blockIdx.x * 256 + threadIdx.x; c < n_chunks;
       c += (long long)gridDim.x * 256) {
    const long long i = c / cpp;
    const long long sp = src_page(page_ids, i, n_src, flags);
    if (sp >= 0) dst[c] = ld_stream(src + sp * cpp + (c - i * cpp));
  }
}

// Inverse of the ternary codec: bf16(gamma * c); the product is exact, so
// each value is +-bf16(gamma) or +0.  The unused field 10 reads as 0.
template <int D>
__global__ void __launch_bounds__(256) dequant_ternary_kernel(const uint16_t* __restrict__ src,
                                                              const float* __restrict__ gamma,
                                                              const int32_t* __restrict__ page_ids,
                                                              long long n_src, uint32_t* flags,
                                                              long long n_groups, int hkv,
                                                              uint4* __restrict__ dst) {
  constexpr int NC = D / 16;
  const int lane = threadIdx.x & 31;
  const long long grp = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (grp >= n_groups) return;
  const long long i = grp / hkv;
  const int h = (int)(grp - i * hkv);
  const long long sp = src_page(page_ids, i, n_src, flags);
  if (sp < 0) return;
  const long long sg = sp * hkv + h;
  const uint16_t* s = src + sg * (2 * D);
  const uint32_t pos = __bfloat16_as_ushort(__float2bfloat16_rn(__ldg(gamma + sg)));
  const uint32_t neg = pos | 0x8000u;
  uint32_t w[NC];
#pragma unroll
  for (int c = 0; c < NC; ++c) w[c] = __ldg(s + c * 32 + lane);
  uint4* d = dst + grp * (2 * D);
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t f0 = (w[c] >> (4 * k)) & 3u, f1 = (w[c] >> (4 * k + 2)) & 3u;
      const uint32_t lo = f0 == 1u ? pos : (f0 == 3u ? neg : 0u);
      const uint32_t hi = f1 == 1u ? pos : (f1 == 3u ? neg : 0u);
      o[k] = lo | (hi << 16);
    }
    __stcs(d + c * 32 + lane, make_uint4(o[0], o[1], o[2], o[3]));
  }
}

// FP8 -> bf16: bf16(RN(fl32(s * e))); one thread per 8 values.
__global__ void __launch_bounds__(256) dequant_fp8_kernel(const uint2* __restrict__ src,
                                                          const float* __restrict__ scale,
                                                          const int32_t* __restrict__ page_ids,
                                                          long long n_src, uint32_t* flags,
                                                          long long n_chunks, long long cpp,
                                                          uint4* __restrict__ dst) {
  for (long long c = (long long)blockIdx.x * 256 + threadIdx.x; c < n_chunks;
       c += (long long)gridDim.x * 256) {
    const long long i = c / cpp;
    const long long sp = src_page(page_ids, i, n_src, flags);
    if (sp < 0) continue;
    const float s = __ldg(scale + sp);
    const uint2 e = __ldg(src + sp * cpp + (c - i * cpp));
    const uint32_t ew[2] = {e.x, e.y};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)(ew[k >> 1] >> (16 * (k & 1)));
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
      const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(s, f.x)));
      const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(s, f.y)));
      o[k] = lo | (hi << 16);
    }
    __stcs(dst + c, make_uint4(o[0], o[1], o[2], o[3]));
  }
}

// --------------------------------------------------------- append + retier
// One decode step's cache update, one CTA per sequence b (length L before
// the step; Vantage's sinks stay and the recent window slides, "Core
// architecture"; Minima's recent pages age into the stale tier, "Recent,
// Anchor and Stale"):
//   1. the page j0 that leaves the high-precision window (page-granular:
//      (j0+1)*16 == L - window + 1, never a sink page) and is tagged ternary
//      is quantised to ternary into slot ternary_slot[b] -- from its bf16
//      values, or bf16(s*e) of an FP8 page -- by the same codec as the pack
//      kernel; the block-table entry moves to that slot, the old slot is
//      reported in freed[b];
//   2. token L goes to row L % 16 of page L / 16 (its high-precision slot
//      already in the block table); a page starting at row 0 is zeroed
//      first; FP8 pages are re-quantised as a whole (decode, new row, new
//      amax and scale, encode), in two passes that read the page from L2.
struct AppendParams {
  const uint16_t* k_new;      // [B][Hkv][D] bf16 bits
  const uint16_t* v_new;
  kvc_paged_cache cache;
  int32_t* block_table;       // [B][max_pages]
  uint8_t* older_fmt;         // [B][max_pages] or null
  const int32_t* ctx;         // [B] lengths before the step
  const int32_t* tern_slot;   // [B]
  int32_t* freed;             // [B] out
  uint32_t* flags;            // device error word or null
  int Hkv, max_pages, sink, window, hp;
};

__device__ __forceinline__ void set_flag(const AppendParams& p, uint32_t f) {
  if (p.flags) atomicOr(p.flags, f);
}

// 8 e4m3 bytes -> 8 bf16 of bf16(RN(fl32(s * e))), packed like a 16-byte chunk of bf16.
__device__ __forceinline__ uint4 fp8x8_to_bf16x8(uint2 e, float s) {
  const uint32_t ew[2] = {e.x, e.y};
  uint32_t o[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)(ew[k >> 1] >> (16 * (k & 1)));
    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(s, f.x)));
    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(s, f.y)));
    o[k] = lo | (hi << 16);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Ternary codec of one (page, head) group whose bf16 values come from an
// hp page (BF16 pool, or FP8 pool with scale s): one warp, the same pairwise
// tree as quant_ternary_kernel.
template <int D>
__device__ void retier_group(const void* hp_pool, float s, bool fp8, long long src_grp,
                             uint16_t* tern, float* gamma, long long dst_grp, int lane) {
  constexpr int NC = D / 16;
  uint4 v[NC];
  if (fp8) {
    const uint2* src = static_cast<const uint2*>(hp_pool) + src_grp * (2 * D);
#pragma unroll
    for (int c = 0; c < NC; ++c) v[c] = fp8x8_to_bf16x8(src[c * 32 + lane], s);
  } else {
    const uint4* src = static_cast<const uint4*>(hp_pool) + src_grp * (2 * D);
#pragma unroll
    for (int c = 0; c < NC; ++c) v[c] = src[c * 32 + lane];
  }
  float pt[NC];
#pragma unroll
  for (int c = 0; c < NC; ++c) pt[c] = abs_sum8(v[c]);
#pragma unroll
  for (int w = 1; w < NC; w <<= 1)
#pragma unroll
    for (int c = 0; c + w < NC; c += 2 * w) pt[c] += pt[c + w];
  float sum = pt[0];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float g = sum * (1.0f / (16 * D));
  const float t = 0.5f * g;
  uint16_t* out = tern + dst_grp * (2 * D);
#pragma unroll
  for (int c = 0; c < NC; ++c) out[c * 32 + lane] = (uint16_t)tern_word16(v[c], t);
  if (lane == 0) gamma[dst_grp] = g;
}

// Page value chunk c (8 bf16) after the append: the new row, zero (fresh
// page) or the page's own value.
template <int D>
__device__ __forceinline__ uint4 page_chunk_after(const AppendParams& p, const uint16_t* nw, long long b,
                                                  const void* pool, long long page, float s_old,
                                                  int r, int c) {
  constexpr int CPR = D / 8;                      // chunks per row
  const int h = c / (16 * CPR), rem = c - h * 16 * CPR, row = rem / CPR, dc = rem - row * CPR;
  if (row == r)
    return reinterpret_cast<const uint4*>(nw)[(b * p.Hkv + h) * CPR + dc];
  if (r == 0) return make_uint4(0u, 0u, 0u, 0u);
  if (p.hp == KVC_FMT_FP8_E4M3)
    return fp8x8_to_bf16x8(static_cast<const uint2*>(pool)[page * p.Hkv * 16 * CPR + c], s_old);
  return static_cast<const uint4*>(pool)[page * p.Hkv * 16 * CPR + c];
}

template <int D>
__device__ void append_one(const AppendParams& p, const uint16_t* nw, long long b, void* pool, float* scale,
                           long long page, int r, float* red) {
  constexpr int CPR = D / 8;
  const int nchunks = p.Hkv * 16 * CPR;
  if (p.hp == KVC_FMT_BF16) {
    uint4* dst = static_cast<uint4*>(pool) + page * nchunks;
    for (int c = threadIdx.x; c < nchunks; c += blockDim.x) {
      const int row = (c % (16 * CPR)) / CPR;
      if (row == r || r == 0) dst[c] = page_chunk_after<D>(p, nw, b, pool, page, 0.f, r, c);
    }
    return;
  }
  // FP8: pass 1 -- amax of the page after the append
  const float s_old = scale[page];
  float amax = 0.f;
  for (int c = threadIdx.x; c < nchunks; c += blockDim.x) {
    const uint4 v = page_chunk_after<D>(p, nw, b, pool, page, s_old, r, c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[k])), fabsf(bf16_hi(w[k]))));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
  for (int k = 1; k < (int)(blockDim.x >> 5); ++k) amax = fmaxf(amax, red[k]);
  __syncthreads();                                 // red is reused; every read of pass 1 is done
  const float sc = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  const float inv = amax > 0.f ? __fdiv_rn(448.0f, amax) : 1.0f;
  // pass 2 -- each thread re-reads and rewrites only its own chunks
  uint2* dst = static_cast<uint2*>(pool) + page * nchunks;
  for (int c = threadIdx.x; c < nchunks; c += blockDim.x) {
    const uint4 v = page_chunk_after<D>(p, nw, b, pool, page, s_old, r, c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 y = make_float2(__fmul_rn(bf16_lo(w[k]), inv), __fmul_rn(bf16_hi(w[k]), inv));
      const uint32_t e2 = __nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3);
      packed[k >> 1] |= e2 << (16 * (k & 1));
    }
    dst[c] = make_uint2(packed[0], packed[1]);
  }
  __syncthreads();
  if (threadIdx.x == 0) scale[page] = sc;
}

template <int D>
__global__ void __launch_bounds__(256) append_retier_kernel(AppendParams p) {
  __shared__ float red[8];
  const long long b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = p.ctx[b];
  if (L < 0 || L >= p.max_pages * kPage) {
    if (threadIdx.x == 0) {
      set_flag(p, kErrContext);
      p.freed[b] = -1;
    }
    return;
  }
  const long long hp_pages = p.hp == KVC_FMT_BF16 ? p.cache.n_pages[0] : p.cache.n_pages[1];
  void* k_hp = const_cast<void*>(p.hp == KVC_FMT_BF16 ? p.cache.k_bf16 : p.cache.k_fp8);
  void* v_hp = const_cast<void*>(p.hp == KVC_FMT_BF16 ? p.cache.v_bf16 : p.cache.v_fp8);
  float* k_sc = const_cast<float*>(p.cache.k_fp8_scale);
  float* v_sc = const_cast<float*>(p.cache.v_fp8_scale);

  // 1. retier the page that leaves the window
  int j0 = -1;
  if (p.window >= 1) {
    const int x = L - p.window + 1;
    if (x > 0 && x % kPage == 0 && (x / kPage - 1) * kPage >= p.sink) j0 = x / kPage - 1;
  }
  int freed = -1, ts = -1;
  if (j0 >= 0) {
    const long long row = b * p.max_pages + j0;
    const int tag = p.older_fmt ? (int)p.older_fmt[row] : KVC_FMT_TERNARY2;
    const int phys = p.block_table[row];
    ts = p.tern_slot[b];
    if (tag == KVC_FMT_TERNARY2) {
      if (phys < 0 || phys >= hp_pages || ts < 0 || ts >= p.cache.n_pages[2]) {
        if (threadIdx.x == 0) set_flag(p, kErrBlockTable);
      } else {
        const bool fp8 = p.hp == KVC_FMT_FP8_E4M3;
        for (int g = warp; g < 2 * p.Hkv; g += (int)(blockDim.x >> 5)) {
          const bool is_v = g >= p.Hkv;
          const int h = is_v ? g - p.Hkv : g;
          retier_group<D>(is_v ? v_hp : k_hp, fp8 ? (is_v ? v_sc : k_sc)[phys] : 0.f, fp8,
                          (long long)phys * p.Hkv + h,
                          static_cast<uint16_t*>(const_cast<void*>(is_v ? p.cache.v_tern : p.cache.k_tern)),
                          const_cast<float*>(is_v ? p.cache.v_gamma : p.cache.k_gamma),
                          (long long)ts * p.Hkv + h, lane);
        }
        freed = phys;
      }
    } else if (tag != p.hp) {
      if (threadIdx.x == 0) set_flag(p, kErrFormat);   // an anchor in the other high-precision format
    }
  }
  __syncthreads();

  // 2. append token L
  const int j = L / kPage, r = L % kPage;
  const int physn = p.block_table[b * p.max_pages + j];
  if (physn < 0 || physn >= hp_pages || physn == freed) {
    if (threadIdx.x == 0) set_flag(p, kErrBlockTable);
  } else {
    append_one<D>(p, p.k_new, b, k_hp, k_sc, physn, r, red);
    append_one<D>(p, p.v_new, b, v_hp, v_sc, physn, r, red);
  }
  if (threadIdx.x == 0) {
    if (freed >= 0) {
      p.block_table[b * p.max_pages + j0] = ts;
      if (p.older_fmt) p.older_fmt[b * p.max_pages + j0] = KVC_FMT_TERNARY2;
    }
    p.freed[b] = freed;
  }
}

// ------------------------------------------------ stale -> anchor promotion
// Minima-KV, "Recent, Anchor and Stale": critical older pages are kept at
// higher fidelity as anchors while stale pages stay addressable in
// compressed form.  One CTA per request re-expands a stale (ternary) page
// into an anchor slot of the BF16 or FP8 pools: the page's content is
// bf16(gamma * c) per KV head; an FP8 anchor encodes that bf16 page with the
// FP8 page codec (one scale over all KV heads, K and V separately).  The
// block-table entry moves to the anchor slot, the tag becomes the anchor
// format, and the ternary slot is reported as freed.
struct PromoteParams {
  kvc_paged_cache cache;
  int32_t* block_table;       // [batch][max_pages]
  uint8_t* older_fmt;         // [batch][max_pages]
  const int32_t* ctx;         // [batch]
  const int32_t* req_seq;     // [n]
  const int32_t* req_page;    // [n]
  const int32_t* anchor_slot; // [n]
  int32_t* freed;             // [n] out
  uint32_t* flags;            // device error word or null
  int batch, Hkv, max_pages, sink, window, hp, anchor;
};

// bf16 bit patterns of the 8 codes of one 16-bit word (2 bits each, LSB
// first): +1 -> pos, -1 -> neg, 0 and the unused field 10 -> +0.
__device__ __forceinline__ uint4 tern8_to_bf16(uint32_t w, uint32_t pos, uint32_t neg) {
  uint32_t o[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t f0 = (w >> (4 * k)) & 3u, f1 = (w >> (4 * k + 2)) & 3u;
    const uint32_t lo = f0 == 1u ? pos : (f0 == 3u ? neg : 0u);
    const uint32_t hi = f1 == 1u ? pos : (f1 == 3u ? neg : 0u);
    o[k] = lo | (hi << 16);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

template <int D>
__global__ void __launch_bounds__(256) promote_kernel(PromoteParams p) {
  constexpr int NC = D / 16;                 // 16-bit code words per lane per group
  __shared__ uint32_t amax_bits[2];          // K, V: amax of the decoded page (float bits, >= 0)
  const int i = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = p.req_seq[i], j = p.req_page[i];
  uint32_t flag = 0;
  long long row = 0;
  int t = -1, a = -1;
  if (b < 0 || b >= p.batch) {
    flag = kErrContext;
  } else {
    const int L = p.ctx[b];
    if (L < 0 || L > p.max_pages * kPage || j < 0 || j >= (L + kPage - 1) / kPage) {
      flag = kErrContext;
    } else {
      row = (long long)b * p.max_pages + j;
      if (page_format(j, L, p.sink, p.window, p.hp, p.older_fmt[row]) != KVC_FMT_TERNARY2) {
        flag = kErrFormat;
      } else {
        t = p.block_table[row];
        a = p.anchor_slot[i];
        const long long n_anchor = p.anchor == KVC_FMT_BF16 ? p.cache.n_pages[0] : p.cache.n_pages[1];
        if (t < 0 || t >= p.cache.n_pages[2] || a < 0 || a >= n_anchor) flag = kErrBlockTable;
      }
    }
  }
  if (flag) {                                // uniform across the CTA
    if (threadIdx.x == 0) {
      if (p.flags) atomicOr(p.flags, flag);
      p.freed[i] = -1;
    }
    return;
  }
  const int n_groups = 2 * p.Hkv;            // K heads, then V heads
  const bool fp8 = p.anchor == KVC_FMT_FP8_E4M3;
  if (fp8) {
    if (threadIdx.x < 2) amax_bits[threadIdx.x] = 0u;
    __syncthreads();
    // amax of the decoded page: bf16(gamma) of every head with a nonzero code
    for (int g = warp; g < n_groups; g += 8) {
      const bool is_v = g >= p.Hkv;
      const int h = is_v ? g - p.Hkv : g;
      const long long grp = (long long)t * p.Hkv + h;
      const uint16_t* src = static_cast<const uint16_t*>(is_v ? p.cache.v_tern : p.cache.k_tern) + grp * (2 * D);
      uint32_t any = 0;
#pragma unroll
      for (int c = 0; c < NC; ++c) any |= src[c * 32 + lane];
      if (__any_sync(0xffffffffu, (any & 0x5555u) != 0u) && lane == 0) {
        const float gam = (is_v ? p.cache.v_gamma : p.cache.k_gamma)[grp];
        const float x = __bfloat162float(__float2bfloat16_rn(gam));
        atomicMax(&amax_bits[is_v ? 1 : 0], __float_as_uint(fabsf(x)));
      }
    }
    __syncthreads();
  }
  for (int g = warp; g < n_groups; g += 8) {
    const bool is_v = g >= p.Hkv;
    const int h = is_v ? g - p.Hkv : g;
    const long long grp = (long long)t * p.Hkv + h, dgrp = (long long)a * p.Hkv + h;
    const uint16_t* src = static_cast<const uint16_t*>(is_v ? p.cache.v_tern : p.cache.k_tern) + grp * (2 * D);
    const float gam = (is_v ? p.cache.v_gamma : p.cache.k_gamma)[grp];
    const uint32_t pos = __bfloat16_as_ushort(__float2bfloat16_rn(gam));
    const uint32_t neg = pos ^ 0x8000u;
    uint32_t w[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) w[c] = src[c * 32 + lane];
    if (!fp8) {
      uint4* dst = static_cast<uint4*>(const_cast<void*>(is_v ? p.cache.v_bf16 : p.cache.k_bf16)) + dgrp * (2 * D);
#pragma unroll
      for (int c = 0; c < NC; ++c) dst[c * 32 + lane] = tern8_to_bf16(w[c], pos, neg);
    } else {
      // the FP8 page codec on the decoded values: y = fl32(x * fl32(448 / amax)),
      // RNE-satfinite e4m3; a head takes only the values +-bf16(gamma) and +0
      const float amax = __uint_as_float(amax_bits[is_v ? 1 : 0]);
      const float inv = amax > 0.f ? __fdiv_rn(448.0f, amax) : 1.0f;
      const float x = __uint_as_float(pos << 16);
      const float2 y = make_float2(__fmul_rn(x, inv), __fmul_rn(-x, inv));
      const uint32_t e2 = __nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3);
      const uint32_t ep = e2 & 0xFFu, en = (e2 >> 8) & 0xFFu;
      uint2* dst = static_cast<uint2*>(const_cast<void*>(is_v ? p.cache.v_fp8 : p.cache.k_fp8)) + dgrp * (2 * D);
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        uint32_t o[2] = {0u, 0u};
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t f = (w[c] >> (2 * k)) & 3u;
          o[k >> 2] |= (f == 1u ? ep : (f == 3u ? en : 0u)) << (8 * (k & 3));
        }
        dst[c * 32 + lane] = make_uint2(o[0], o[1]);
      }
      if (h == 0 && lane == 0)
        const_cast<float*>(is_v ? p.cache.v_fp8_scale : p.cache.k_fp8_scale)[a] =
            amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    }
  }
  __syncthreads();                           // every thread has read the entry before it changes
  if (threadIdx.x == 0) {
    p.block_table[row] = a;
    p.older_fmt[row] = (uint8_t)p.anchor;
    p.freed[i] = t;
  }
}

int grid_for(long long work, int per_block) {
  long long g = (work + per_block - 1) / per_block;
  if (g > (1ll << 30)) g = 1ll << 30;
  return (int)(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_quant_ternary(const void* src, const int32_t* page_ids, long long n_src, uint32_t* flags, int n, int hkv, int d,
                                 void* dst, float* gamma, cudaStream_t s) {
  const long long groups = (long long)n * hkv;
  const int grid = grid_for(groups, d > 128 ? 2 : 8);      // groups per 256-thread CTA
  auto* in = static_cast<const uint4*>(src);
  auto* out = static_cast<uint16_t*>(dst);
  switch (d) {
    case 64: quant_ternary_kernel<64><<<grid, 256, 0, s>>>(in, page_ids, n_src, flags, groups, hkv, out, gamma); break;
    case 128: quant_ternary_kernel<128><<<grid, 256, 0, s>>>(in, page_ids, n_src, flags, groups, hkv, out, gamma); break;
    case 256: quant_ternary_kernel<256><<<grid, 256, 0, s>>>(in, page_ids, n_src, flags, groups, hkv, out, gamma); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_quant_fp8(const void* src, const int32_t* page_ids, long long n_src, uint32_t* flags, int n, int hkv, int d,
                             void* dst, float* scale, cudaStream_t s) {
  const int cpp = hkv * kPage * d / 8;
  auto* in = static_cast<const uint4*>(src);
  auto* out = static_cast<uint2*>(dst);
  // pages of 512, 1024, 2048 or 4096 chunks (Hkv * D = 256 .. 2048): the
  // register-resident kernel; other sizes: the two-pass one
  switch (cpp) {
    // (measured: 4 warps x 4 chunks per lane for 8 KB pages and 8 x 8 for
    // 32 KB pages beat 2 x 8 / 8 x 2 and 4 x 16)
    case 512: quant_fp8_reg_kernel<4, 4><<<grid_for(n, 2), 256, 0, s>>>(in, page_ids, n_src, flags, n, out, scale); break;
    case 1024: quant_fp8_reg_kernel<4, 8><<<grid_for(n, 2), 256, 0, s>>>(in, page_ids, n_src, flags, n, out, scale); break;
    case 2048: quant_fp8_reg_kernel<8, 8><<<n, 256, 0, s>>>(in, page_ids, n_src, flags, n, out, scale); break;
    case 4096: quant_fp8_reg_kernel<8, 16><<<n, 256, 0, s>>>(in, page_ids, n_src, flags, n, out, scale); break;
    default: quant_fp8_kernel<<<n, 256, 0, s>>>(in, page_ids, n_src, flags, cpp, out, scale); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_copy_pages(const void* src, const int32_t* page_ids, long long n_src, uint32_t* flags, int n, size_t page_bytes,
                              void* dst, cudaStream_t s) {
  const long long cpp = (long long)(page_bytes / 16);
  const long long chunks = cpp * n;
  copy_pages_kernel<<<grid_for(chunks, 256 * 4), 256, 0, s>>>(
      static_cast<const uint4*>(src), page_ids, n_src, flags, chunks, cpp, static_cast<uint4*>(dst));
  return cudaGetLastError();
}

cudaError_t launch_dequant_ternary(const void* src, const float* gamma, const int32_t* page_ids, long long n_src, uint32_t* flags,
                                   int n, int hkv, int d, void* dst, cudaStream_t s) {
  const long long groups = (long long)n * hkv;
  const int grid = grid_for(groups, 8);
  auto* in = static_cast<const uint16_t*>(src);
  auto* out = static_cast<uint4*>(dst);
  switch (d) {
    case 64: dequant_ternary_kernel<64><<<grid, 256, 0, s>>>(in, gamma, page_ids, n_src, flags, groups, hkv, out); break;
    case 128: dequant_ternary_kernel<128><<<grid, 256, 0, s>>>(in, gamma, page_ids, n_src, flags, groups, hkv, out); break;
    case 256: dequant_ternary_kernel<256><<<grid, 256, 0, s>>>(in, gamma, page_ids, n_src, flags, groups, hkv, out); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_append_retier(const void* k_new, const void* v_new, const kvc_paged_cache& cache,
                                int32_t* block_table, uint8_t* older_fmt, const int32_t* ctx,
                                const int32_t* tern_slot, int32_t* freed, uint32_t* flags, int batch,
                                int hkv, int d, int max_pages, int sink, int window, int hp,
                                cudaStream_t s) {
  AppendParams p;
  p.k_new = static_cast<const uint16_t*>(k_new);
  p.v_new = static_cast<const uint16_t*>(v_new);
  p.cache = cache;
  p.block_table = block_table;
  p.older_fmt = older_fmt;
  p.ctx = ctx;
  p.tern_slot = tern_slot;
  p.freed = freed;
  p.flags = flags;
  p.Hkv = hkv;
  p.max_pages = max_pages;
  p.sink = sink;
  p.window = window;
  p.hp = hp;
  switch (d) {
    case 64: append_retier_kernel<64><<<batch, 256, 0, s>>>(p); break;
    case 128: append_retier_kernel<128><<<batch, 256, 0, s>>>(p); break;
    case 256: append_retier_kernel<256><<<batch, 256, 0, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_promote(const kvc_paged_cache& cache, int32_t* block_table, uint8_t* older_fmt,
                           const int32_t* ctx, const int32_t* req_seq, const int32_t* req_page,
                           const int32_t* anchor_slot, int32_t* freed, uint32_t* flags, int n, int batch,
                           int hkv, int d, int max_pages, int sink, int window, int hp, int anchor,
                           cudaStream_t s) {
  PromoteParams p;
  p.cache = cache;
  p.block_table = block_table;
  p.older_fmt = older_fmt;
  p.ctx = ctx;
  p.req_seq = req_seq;
  p.req_page = req_page;
  p.anchor_slot = anchor_slot;
  p.freed = freed;
  p.flags = flags;
  p.batch = batch;
  p.Hkv = hkv;
  p.max_pages = max_pages;
  p.sink = sink;
  p.window = window;
  p.hp = hp;
  p.anchor = anchor;
  switch (d) {
    case 64: promote_kernel<64><<<n, 256, 0, s>>>(p); break;
    case 128: promote_kernel<128><<<n, 256, 0, s>>>(p); break;
    case 256: promote_kernel<256><<<n, 256, 0, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_dequant_fp8(const void* src, const float* scale, const int32_t* page_ids, long long n_src, uint32_t* flags,
                               int n, int hkv, int d, void* dst, cudaStream_t s) {
  const long long cpp = (long long)hkv * kPage * d / 8;
  const long long chunks = cpp * n;
  dequant_fp8_kernel<<<grid_for(chunks, 256 * 4), 256, 0, s>>>(
      static_cast<const uint2*>(src), scale, page_ids, n_src, flags, chunks, cpp, static_cast<uint4*>(dst));
  return cudaGetLastError();
}

}  // namespace kvc
