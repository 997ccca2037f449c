// Mixed-format paged decode attention, CUDA-core version.
//
// "Minima-KV" (twodots.gr), section "How mixed-format attention works":
// every page is read in its own format (BF16 / FP8 / packed ternary) with no
// dense copy of the cache, each split of a sequence emits a partial state
// (max score, sum of exponentials, output) and the states are merged by an
// online-softmax normalisation.  The ternary format is Vantage's ("Show HN:
// Vantage-V-AI", section "Core architecture"), the sink/window rule its
// attention sinks and recent window.
//
// Work item = (split of pages, KV head, sequence); one CTA of 4 warps per
// item, warps take the item's pages round robin, each lane owns D/32
// contiguous dims.  Scores are warp-wide dot products; this kernel is the
// straightforward path, kept for shapes the tensor-core kernel does not
// take and as an independent second implementation in the tests.
#include "kvc_internal.cuh"

#include <math.h>

namespace kvc {
namespace {

constexpr int kWarps = 4;

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ float e4m3_to_float(uint32_t byte) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)byte, __NV_E4M3);
  return __half2float(*reinterpret_cast<const __half*>(&h));
}

// Decoded K (or V) values of token t, dims [d0, d0 + DPL) of KV head g of
// physical page `phys` in format `fmt`.
template <int D, int DPL>
__device__ __forceinline__ void load_row(const void* bf16_pool, const void* fp8_pool,
                                         const float* fp8_scale, const void* tern_pool,
                                         const float* gamma, int fmt, long long phys, int hkv,
                                         int g, int t, int d0, float (&x)[DPL]) {
  const long long grp = phys * hkv + g;
  if (fmt == KVC_FMT_BF16) {
    const uint16_t* p = static_cast<const uint16_t*>(bf16_pool) + (grp * kPage + t) * D + d0;
#pragma unroll
    for (int i = 0; i < DPL; ++i) x[i] = bf16_bits_to_float(__ldg(p + i));
  } else if (fmt == KVC_FMT_FP8_E4M3) {
    const uint8_t* p = static_cast<const uint8_t*>(fp8_pool) + (grp * kPage + t) * D + d0;
    const float s = __ldg(fp8_scale + phys);
#pragma unroll
    for (int i = 0; i < DPL; ++i) x[i] = s * e4m3_to_float(__ldg(p + i));
  } else {
    const uint8_t* p = static_cast<const uint8_t*>(tern_pool) + grp * (kPage * D / 4);
    const float gm = __ldg(gamma + grp);
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      const int e = t * D + d0 + i;
      const uint32_t f = (__ldg(p + e / 4) >> (2 * (e % 4))) & 3u;
      x[i] = f == 1u ? gm : (f == 3u ? -gm : 0.f);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kWarps * 32) decode_simple_kernel(DecodeParams p) {
  constexpr int DPL = D / 32;
  __shared__ float qs[8][D];
  __shared__ float sm_m[kWarps][8], sm_l[kWarps][8];
  __shared__ float sm_o[kWarps][8][D];
  __shared__ unsigned last_cta;

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G, Hkv = p.Hkv;
  int L = p.ctx[b % p.Bseq];
  const int layer = b / p.Bseq;
  if (L < 0 || L > p.max_pages * kPage) {
    if (threadIdx.x == 0) atomicOr(p.err, kErrContext);
    L = 0;
  }
  const int n_pages = (L + kPage - 1) / kPage;
  const int j0 = split * p.pages_per_split;
  const int j1 = min(j0 + p.pages_per_split, n_pages);

  for (int i = threadIdx.x; i < G * D; i += kWarps * 32) {
    const int r = i / D, d = i - r * D;
    const uint16_t qb = reinterpret_cast<const uint16_t*>(p.q)[((long long)b * p.Hq + g * G + r) * D + d];
    qs[r][d] = bf16_bits_to_float(qb) * p.scale_log2;
  }
  __syncthreads();

  float m[8], l[8], o[8][DPL];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) o[r][i] = 0.f;
  }
  const int d0 = lane * DPL;
  const kvc_paged_cache& c = p.cache;

  for (int j = j0 + warp; j < j1; j += kWarps) {
    const long long row = (long long)(b % p.Bseq) * p.max_pages + j;
    const int older = p.older_fmt ? p.older_fmt[row] : KVC_FMT_TERNARY2;
    const int fmt = page_format(j, L, p.sink, p.window, p.hp, older);
    if (fmt < 0 || fmt > 2) {
      if (lane == 0) atomicOr(p.err, kErrFormat);
      continue;
    }
    long long phys = p.block_table[row];
    if (phys < 0 || phys >= c.n_pages[fmt]) {
      if (lane == 0) atomicOr(p.err, kErrBlockTable);
      continue;
    }
    phys += (long long)layer * c.n_pages[fmt];          // this layer's part of the pool
    const int nt = min(kPage, L - j * kPage);
    for (int t = 0; t < nt; ++t) {
      float kx[DPL], vx[DPL];
      load_row<D, DPL>(c.k_bf16, c.k_fp8, c.k_fp8_scale, c.k_tern, c.k_gamma, fmt, phys, Hkv, g, t, d0, kx);
      load_row<D, DPL>(c.v_bf16, c.v_fp8, c.v_fp8_scale, c.v_tern, c.v_gamma, fmt, phys, Hkv, g, t, d0, vx);
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (r >= G) break;
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) s = fmaf(qs[r][d0 + i], kx[i], s);
#pragma unroll
        for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        const float mn = fmaxf(m[r], s);
        const float corr = exp2f(m[r] - mn);
        const float pe = exp2f(s - mn);
        l[r] = l[r] * corr + pe;
#pragma unroll
        for (int i = 0; i < DPL; ++i) o[r][i] = fmaf(pe, vx[i], o[r][i] * corr);
        m[r] = mn;
      }
    }
  }

  // merge the warps' states into this split's partial state
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    if (r >= G) break;
    if (lane == 0) {
      sm_m[warp][r] = m[r];
      sm_l[warp][r] = l[r];
    }
#pragma unroll
    for (int i = 0; i < DPL; ++i) sm_o[warp][r][d0 + i] = o[r][i];
  }
  __syncthreads();
  const long long bg = (long long)b * Hkv + g;
  float* part = p.partials + (bg * p.n_splits + split) * (long long)(G * (D + 2));
  for (int i = threadIdx.x; i < G * D; i += kWarps * 32) {
    const int r = i / D, d = i - r * D;
    float ms = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) ms = fmaxf(ms, sm_m[w][r]);
    float ov = 0.f, lv = 0.f;
    if (ms != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float f = exp2f(sm_m[w][r] - ms);
        ov = fmaf(sm_o[w][r][d], f, ov);
        lv = fmaf(sm_l[w][r], f, lv);
      }
    }
    part[r * (D + 2) + 2 + d] = ov;
    if (d == 0) {
      part[r * (D + 2)] = ms;
      part[r * (D + 2) + 1] = lv;
    }
  }

  // last split of this (sequence, KV head) to finish merges all splits
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last_cta = atomicAdd(p.tickets + bg, 1u) == (unsigned)(p.n_splits - 1);
  __syncthreads();
  if (!last_cta) return;
  __threadfence();
  const float* all = p.partials + bg * p.n_splits * (long long)(G * (D + 2));
  for (int i = threadIdx.x; i < G * D; i += kWarps * 32) {
    const int r = i / D, d = i - r * D;
    float ms = -INFINITY;
    for (int s = 0; s < p.n_splits; ++s) ms = fmaxf(ms, __ldcg(all + (s * G + r) * (D + 2)));
    float ov = 0.f, lv = 0.f;
    if (ms != -INFINITY) {
      for (int s = 0; s < p.n_splits; ++s) {
        const float* st = all + (s * G + r) * (D + 2);
        const float f = exp2f(__ldcg(st) - ms);
        lv = fmaf(__ldcg(st + 1), f, lv);
        ov = fmaf(__ldcg(st + 2 + d), f, ov);
      }
    }
    p.out[((long long)b * p.Hq + g * G + r) * D + d] = lv > 0.f ? ov / lv : 0.f;
  }
  if (threadIdx.x == 0) p.tickets[bg] = 0u;
}

}  // namespace

cudaError_t launch_decode_simple(const DecodeParams& p, int head_dim, cudaStream_t s) {
  const dim3 grid(p.n_splits, p.Hkv, p.B);
  switch (head_dim) {
    case 64: decode_simple_kernel<64><<<grid, kWarps * 32, 0, s>>>(p); break;
    case 128: decode_simple_kernel<128><<<grid, kWarps * 32, 0, s>>>(p); break;
    case 256: decode_simple_kernel<256><<<grid, kWarps * 32, 0, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace kvc
