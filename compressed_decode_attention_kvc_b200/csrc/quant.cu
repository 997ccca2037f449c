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
// at head_dim 256 two warps share a group (each holds 4 KB in registers, so
// enough warps stay resident to keep HBM busy) and add their partial sums
// through shared memory.  Lane l owns chunks l, l+32, ... of its warp's part:
// every load and store instruction of the warp is contiguous.  gamma is a
// pairwise tree (per chunk, across the lane's chunks, across lanes, across the
// two parts): depth log2(16*D) <= 12, so its float32 relative error stays
// below 12 * 2^-24.
template <int D>
__global__ void __launch_bounds__(256) quant_ternary_kernel(const uint4* __restrict__ src,
                                                            const int32_t* __restrict__ page_ids,
                                                            long long n_groups, int hkv,
                                                            uint16_t* __restrict__ dst,
                                                            float* __restrict__ gamma) {
  constexpr int WPG = D > 128 ? 2 : 1;      // warps per group
  constexpr int NC = D / 16 / WPG;          // chunks per lane
  __shared__ float red[8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int part = warp % WPG;
  const long long grp = (long long)blockIdx.x * (8 / WPG) + warp / WPG;
  const bool valid = grp < n_groups;
  const uint4* s = src;
  if (valid) {
    const long long i = grp / hkv;
    const int h = (int)(grp - i * hkv);
    const long long sp = page_ids ? (long long)page_ids[i] : i;
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
    sum = red[w0] + red[w0 + 1];              // same order in both warps
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
                                                        int chunks_per_page,
                                                        uint2* __restrict__ dst,
                                                        float* __restrict__ scale) {
  __shared__ float red[8];
  const long long i = blockIdx.x;
  const long long sp = page_ids ? (long long)page_ids[i] : i;
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

__global__ void __launch_bounds__(256) copy_pages_kernel(const uint4* __restrict__ src,
                                                         const int32_t* __restrict__ page_ids,
                                                         long long n_chunks, long long cpp,
                                                         uint4* __restrict__ dst) {
  for (long long c = (long long)blockIdx.x * 256 + threadIdx.x; c < n_chunks;
       c += (long long)gridDim.x * 256) {
    const long long i = c / cpp;
    const long long sp = page_ids ? (long long)page_ids[i] : i;
    dst[c] = ld_stream(src + sp * cpp + (c - i * cpp));
  }
}

// Inverse of the ternary codec: bf16(gamma * c); the product is exact, so
// each value is +-bf16(gamma) or +0.  The unused field 10 reads as 0.
template <int D>
__global__ void __launch_bounds__(256) dequant_ternary_kernel(const uint16_t* __restrict__ src,
                                                              const float* __restrict__ gamma,
                                                              const int32_t* __restrict__ page_ids,
                                                              long long n_groups, int hkv,
                                                              uint4* __restrict__ dst) {
  constexpr int NC = D / 16;
  const int lane = threadIdx.x & 31;
  const long long grp = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (grp >= n_groups) return;
  const long long i = grp / hkv;
  const int h = (int)(grp - i * hkv);
  const long long sg = (page_ids ? (long long)page_ids[i] : i) * hkv + h;
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
                                                          long long n_chunks, long long cpp,
                                                          uint4* __restrict__ dst) {
  for (long long c = (long long)blockIdx.x * 256 + threadIdx.x; c < n_chunks;
       c += (long long)gridDim.x * 256) {
    const long long i = c / cpp;
    const long long sp = page_ids ? (long long)page_ids[i] : i;
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

int grid_for(long long work, int per_block) {
  long long g = (work + per_block - 1) / per_block;
  if (g > (1ll << 30)) g = 1ll << 30;
  return (int)(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_quant_ternary(const void* src, const int32_t* page_ids, int n, int hkv, int d,
                                 void* dst, float* gamma, cudaStream_t s) {
  const long long groups = (long long)n * hkv;
  const int grid = grid_for(groups, d > 128 ? 4 : 8);      // groups per 256-thread CTA
  auto* in = static_cast<const uint4*>(src);
  auto* out = static_cast<uint16_t*>(dst);
  switch (d) {
    case 64: quant_ternary_kernel<64><<<grid, 256, 0, s>>>(in, page_ids, groups, hkv, out, gamma); break;
    case 128: quant_ternary_kernel<128><<<grid, 256, 0, s>>>(in, page_ids, groups, hkv, out, gamma); break;
    case 256: quant_ternary_kernel<256><<<grid, 256, 0, s>>>(in, page_ids, groups, hkv, out, gamma); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_quant_fp8(const void* src, const int32_t* page_ids, int n, int hkv, int d,
                             void* dst, float* scale, cudaStream_t s) {
  const int cpp = hkv * kPage * d / 8;
  quant_fp8_kernel<<<n, 256, 0, s>>>(static_cast<const uint4*>(src), page_ids, cpp,
                                      static_cast<uint2*>(dst), scale);
  return cudaGetLastError();
}

cudaError_t launch_copy_pages(const void* src, const int32_t* page_ids, int n, size_t page_bytes,
                              void* dst, cudaStream_t s) {
  const long long cpp = (long long)(page_bytes / 16);
  const long long chunks = cpp * n;
  copy_pages_kernel<<<grid_for(chunks, 256 * 4), 256, 0, s>>>(
      static_cast<const uint4*>(src), page_ids, chunks, cpp, static_cast<uint4*>(dst));
  return cudaGetLastError();
}

cudaError_t launch_dequant_ternary(const void* src, const float* gamma, const int32_t* page_ids,
                                   int n, int hkv, int d, void* dst, cudaStream_t s) {
  const long long groups = (long long)n * hkv;
  const int grid = grid_for(groups, 8);
  auto* in = static_cast<const uint16_t*>(src);
  auto* out = static_cast<uint4*>(dst);
  switch (d) {
    case 64: dequant_ternary_kernel<64><<<grid, 256, 0, s>>>(in, gamma, page_ids, groups, hkv, out); break;
    case 128: dequant_ternary_kernel<128><<<grid, 256, 0, s>>>(in, gamma, page_ids, groups, hkv, out); break;
    case 256: dequant_ternary_kernel<256><<<grid, 256, 0, s>>>(in, gamma, page_ids, groups, hkv, out); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_dequant_fp8(const void* src, const float* scale, const int32_t* page_ids,
                               int n, int hkv, int d, void* dst, cudaStream_t s) {
  const long long cpp = (long long)hkv * kPage * d / 8;
  const long long chunks = cpp * n;
  dequant_fp8_kernel<<<grid_for(chunks, 256 * 4), 256, 0, s>>>(
      static_cast<const uint2*>(src), scale, page_ids, chunks, cpp, static_cast<uint4*>(dst));
  return cudaGetLastError();
}

}  // namespace kvc
