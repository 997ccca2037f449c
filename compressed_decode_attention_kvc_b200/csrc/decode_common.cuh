// Pieces shared by the decode-attention kernels (decode_tc.cu, decode_umma.cu):
// PTX wrappers, the stream-K work partition, the page-metadata loader and the
// split-K merge.  Everything here is internal to the library.
//
// Method: "Minima-KV" (twodots.gr), section "How mixed-format attention
// works" - pages are read in their own format as they are loaded, each split
// of a (sequence, KV head) emits a partial state (max score, sum of
// exponentials, output) and one online-softmax normalisation merges them.
#pragma once

#include "kvc_internal.cuh"

#include <math.h>

namespace kvc {
namespace dec {

constexpr uint32_t kSuspendNs = 1000000;   // 1 ms per try
constexpr uint32_t kSpinLimit = 4000;      // ... for at most ~4 s
constexpr int kSkip = 3;                   // entry carrying an unusable page (flagged, no data)
constexpr unsigned kFull = 0xffffffffu;
constexpr int kMaxPages = 8;               // pages per entry

struct Desc {
  int fmt, np, bg, nrows;            // nrows: valid token rows of the entry's last page
  int row0;                          // first page row held (BF16 half pages: 0 or 8)
  int bq;                            // (sequence, KV head group) pair of the entry
  float gvmax;                       // largest V scale of the entry's pages (this head)
  float ks[kMaxPages], vs[kMaxPages];
};

__host__ __device__ constexpr int group_bytes(int fmt, int d) {
  return fmt == KVC_FMT_TERNARY2 ? 4 * d : (fmt == KVC_FMT_FP8_E4M3 ? 16 * d : 32 * d);
}

// ------------------------------------------------------------------ PTX
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
// Raise the bytes a phase waits for, without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
               ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
// try_wait suspends the warp (it issues nothing) until the phase completes
// or the hinted time, in ns, runs out.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs) : "memory");
  return ok != 0;
}
// Bounded wait: false if the phase did not complete within the limit
// (`limit` tries of at most kSuspendNs each).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t limit = kSpinLimit) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}
// try_wait without a suspend hint: returns after a short, system-defined
// time if the phase has not completed.
__device__ __forceinline__ bool mbar_try_wait_short(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
constexpr uint64_t kWaitLimitNs = 4000000000ull;   // 4 s
// Bounded wait for waits that are usually short (tensor-core completions):
// false if the phase did not complete within kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait_spin(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait_short(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait_short(bar, parity))
    if (global_ns() - t0 > kWaitLimitNs) return false;
  return true;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// int8 x int8 -> int32, m16n8k32: four 8-bit k-elements per register
__device__ __forceinline__ void imma16832(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// signed int8 A x unsigned int8 B -> int32, m16n8k32 (ternary codes times
// the non-negative digits of P)
__device__ __forceinline__ void imma16832_su(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movtrans(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  return __byte_perm(a, b, sel);
}
__device__ __forceinline__ uint32_t f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// bf16 x bf16 -> f32, m16n8k16 (BF16 pages: K, V and Q in their given form)
__device__ __forceinline__ void mma16816_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
// y as a bf16 pair (hi, lo) with hi = bf16(y), lo = bf16(y - hi): ~16 bits.
__device__ __forceinline__ uint32_t split_bf16x2(float y) {
  const float hi = __bfloat162float(__float2bfloat16_rn(y));
  return bf16x2(hi, y - hi);
}

// Ternary fields at bit offset o (even, 0..14) of both 16-bit halves -> f16
// pair of 2*code: 01 -> 0x4000 (+2), 11 -> 0xC000 (-2), 00 -> 0 (10 -> -0).
__device__ __forceinline__ uint32_t tern2(uint32_t w, int o) {
  return (o == 14 ? w : (w << (14 - o))) & 0xC000C000u;
}
// Ternary field f (0..3) of each byte of w -> four int8 of 64*code: the
// 2-bit field moved to bits 6..7 of its byte is 01 -> 64, 11 -> -64, 00 -> 0
// (10 -> -128).  One AND (and one shift for f < 3) per four codes.
__device__ __forceinline__ uint32_t tern8(uint32_t w, int f) {
  return (f == 3 ? w : (w << (6 - 2 * f))) & 0xC0C0C0C0u;
}
// y as an f16 pair (hi, lo) with hi = f16(y), lo = f16(y - hi): ~22 bits.
__device__ __forceinline__ uint32_t split_f16x2(float y) {
  const float hi = __half2float(__float2half_rn(y));
  return f16x2(hi, y - hi);
}
// Two e4m3 bytes (low byte -> low half) -> f16x2.
__device__ __forceinline__ uint32_t e4m3x2_f16(uint32_t two_bytes) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two_bytes & 0xFFFFu), __NV_E4M3);
  return (uint32_t)h.x | ((uint32_t)h.y << 16);
}
// bf16x2 -> f16x2 (exact for |x| in the f16 normal range).
__device__ __forceinline__ uint32_t bf16x2_f16(uint32_t u) {
  return f16x2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}
// byte-permute selector taking byte k and k+1 of a, interleaved with b's:
// result bytes (a.k, b.k, a.k+1, b.k+1)
__host__ __device__ constexpr uint32_t sel_pair(int k) {
  return (uint32_t)(k | ((4 + k) << 4) | ((k + 1) << 8) | ((5 + k) << 12));
}

template <typename T>
__device__ __forceinline__ T lds(const unsigned char* p) {
  return *reinterpret_cast<const T*>(p);
}

// ------------------------------------------------------- work partition
// Sequence b contributes (Hkv / HPC) * np(b) units (one page of a group of
// HPC KV heads), ordered (b, q, j).  Each unit carries a weight: the
// high-precision format's cost for sink and window pages, the ternary cost
// for older pages (anchors are counted as ternary).  CTA W of NW owns the
// units whose weighted start lies in [W*C/NW, (W+1)*C/NW), C the total weight.
struct SeqShape {
  int np, ns, jw2, cost;   // pages, sink pages, first window page (>= ns), weight per KV head
};

__device__ __forceinline__ SeqShape seq_shape(int L, int sink, int window, int whp, int wt) {
  SeqShape s;
  s.np = (L + kPage - 1) / kPage;
  s.ns = min(s.np, (sink + kPage - 1) / kPage);
  int jw = s.np;
  if (window > 0) jw = L - window > 0 ? (L - window) / kPage : 0;
  s.jw2 = max(s.ns, min(jw, s.np));
  s.cost = whp * (s.ns + (s.np - s.jw2)) + (s.jw2 - s.ns) * wt;
  return s;
}
// weighted start of page j inside one (sequence, KV head group)
__device__ __forceinline__ int cost_of_page(const SeqShape& s, int j, int whp, int wt) {
  if (j <= s.ns) return whp * j;
  if (j <= s.jw2) return whp * s.ns + wt * (j - s.ns);
  return whp * s.ns + wt * (s.jw2 - s.ns) + whp * (j - s.jw2);
}
// first page whose weighted start is >= c (np when none)
__device__ __forceinline__ int page_of_cost(const SeqShape& s, int c, int whp, int wt) {
  const int a = whp * s.ns;
  if (c <= a) return (c + whp - 1) / whp;
  const int bnd = a + wt * (s.jw2 - s.ns);
  if (c <= bnd) return s.ns + (c - a + wt - 1) / wt;
  return min(s.np, s.jw2 + (c - bnd + whp - 1) / whp);
}

struct Prologue {
  const int* seqP;     // [B + 1] unit prefix
  const int* seqC;     // [B + 1] weight prefix
  const int* seqL;     // [B] validated lengths
  int B, Hkv, sink, window, whp, wt;   // wt: weight of a ternary page
  long long C;         // total weight
  int U;               // total units
  int nwg;             // workers in the partition

  // last b with prefix[b] <= x (prefix nondecreasing, x < prefix[B])
  __device__ __forceinline__ int find(const int* prefix, long long x) const {
    int lo = 0, hi = B;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid] <= x) lo = mid; else hi = mid;
    }
    return lo;
  }
  // first unit whose weighted start is >= c
  __device__ int unit_of_cost(long long c) const {
    if (c >= C) return U;
    const int b = find(seqC, c);
    const SeqShape s = seq_shape(seqL[b], sink, window, whp, wt);
    const int cl = (int)(c - seqC[b]);
    const int q = cl / s.cost;
    const int j = page_of_cost(s, cl - q * s.cost, whp, wt);
    return seqP[b] + q * s.np + j;
  }
  // worker that owns unit x
  __device__ int worker_of(int x) const {
    const int b = find(seqP, x);
    const SeqShape s = seq_shape(seqL[b], sink, window, whp, wt);
    const int off = x - seqP[b];
    const int q = off / s.np;
    const long long cs = seqC[b] + (long long)q * s.cost + cost_of_page(s, off - q * s.np, whp, wt);
    return (int)(((cs + 1) * nwg + C - 1) / C) - 1;
  }
};

// ------------------------------------------------------------- metadata
// Per-lane page metadata.  Phase A (block-table slot, caller tag) is loaded
// one chunk of 32 units ahead; phase B (format, scales) once those loads
// have landed.  Every warp of a CTA decodes the same units (same pages and
// formats) with the scales of its own KV head.  Packed words keep the
// register footprint small (bq: the (sequence, head group) pair):
//   A.info: ntok (5 bits) | is_hp (1) << 5 | g (7) << 6 | bq << 13
//   Meta.m: fmt (2 bits) | ntok (5) << 2 | bq << 7     (m < 0: no unit)
__device__ __forceinline__ int meta_pack(int fmt, int ntok, int bg) { return fmt | (ntok << 2) | (bg << 7); }
__device__ __forceinline__ int meta_fmt(int m) { return m & 3; }
__device__ __forceinline__ int meta_ntok(int m) { return (m >> 2) & 31; }
__device__ __forceinline__ int meta_bg(int m) { return m >> 7; }

struct MetaA {
  int phys, older, info;    // info < 0: no unit
  int layer;                // layer of a stacked batch (pool slots offset by layer * n_pages)
};
struct Meta {
  int m;                    // packed fmt / ntok / bq
  int grp;                  // (page slot) * Hkv + g: index of this warp's (page, head) group
  float ks, vs;             // K / V scale of the page (gamma, s or 1)
};

// Unit x -> (sequence, KV head, page) for the 32 units of a chunk starting at
// x0.  The chunk's first unit is decoded once for the warp; lanes past the
// end of that (sequence, KV head) decode their own unit.
__device__ __forceinline__ void meta_phase_a(const DecodeParams& p, const Prologue& pr, int x0, int u1,
                                             int lane, int hpc, int wi, MetaA& a) {
  a.info = -1;
  a.phys = 0;
  a.layer = 0;
  a.older = KVC_FMT_TERNARY2;
  if (x0 >= u1) return;
  const int b0 = pr.find(pr.seqP, x0);
  const int L0 = pr.seqL[b0];
  const int np0 = (L0 + kPage - 1) / kPage;
  const int off0 = x0 - pr.seqP[b0];
  const int q0 = off0 / np0;
  const int j0 = off0 - q0 * np0;
  const int x = x0 + lane;
  if (x >= u1) return;
  int b = b0, q = q0, j = j0 + lane, L = L0;
  if (j >= np0) {                                  // past the first (sequence, head group)
    b = pr.find(pr.seqP, x);
    L = pr.seqL[b];
    const int np = (L + kPage - 1) / kPage;
    const int off = x - pr.seqP[b];
    q = off / np;
    j = off - q * np;
  }
  const int g = q * hpc + wi;                      // this warp's KV head
  const int bq = b * (p.Hkv / hpc) + q;            // (sequence, head group) pair
  int rb = p.b_base + b;                           // virtual sequence -> row of the shared block table
  if (rb >= p.Bseq) {                              // stacked layers
    a.layer = rb / p.Bseq;
    rb -= a.layer * p.Bseq;
  }
  const long long row = (long long)rb * p.max_pages + j;
  const int last_valid = min((j + 1) * kPage, L) - 1;
  const int is_hp = (j * kPage < p.sink || last_valid >= L - p.window) ? 1 : 0;
  a.info = min(kPage, L - j * kPage) | (is_hp << 5) | (g << 6) | (bq << 13);
  a.phys = __ldg(p.block_table + row);
  a.older = p.older_fmt ? (int)__ldg(p.older_fmt + row) : KVC_FMT_TERNARY2;
}

__device__ __forceinline__ void meta_phase_b(const DecodeParams& p, const MetaA& a, Meta& m) {
  m.ks = m.vs = 0.f;
  m.grp = 0;
  if (a.info < 0) {
    m.m = -1;
    return;
  }
  const int ntok = a.info & 31, g = (a.info >> 6) & 127, bg = a.info >> 13;
  int fmt = (a.info >> 5) & 1 ? p.hp : a.older;
  if (fmt < 0 || fmt > 2) {
    atomicOr(p.err, kErrFormat);
    fmt = kSkip;
  } else if (a.phys < 0 || a.phys >= (fmt == KVC_FMT_BF16 ? p.cache.n_pages[0]
                                       : fmt == KVC_FMT_FP8_E4M3 ? p.cache.n_pages[1] : p.cache.n_pages[2])) {
    atomicOr(p.err, kErrBlockTable);
    fmt = kSkip;
  } else {
    // the layer's pool slots follow the earlier layers'
    const int phys = a.phys + a.layer * (int)(fmt == KVC_FMT_BF16 ? p.cache.n_pages[0]
                                             : fmt == KVC_FMT_FP8_E4M3 ? p.cache.n_pages[1] : p.cache.n_pages[2]);
    m.grp = phys * p.Hkv + g;
    if (fmt == KVC_FMT_TERNARY2) {
      m.ks = __ldg(p.cache.k_gamma + m.grp);
      m.vs = __ldg(p.cache.v_gamma + m.grp);
    } else if (fmt == KVC_FMT_FP8_E4M3) {
      m.ks = __ldg(p.cache.k_fp8_scale + phys);
      m.vs = __ldg(p.cache.v_fp8_scale + phys);
    } else {
      m.ks = m.vs = 1.f;
    }
  }
  m.m = meta_pack(fmt, ntok, bg);
}

// Merge the partial states of one (sequence, KV head) and write its output
// rows.  Records are read with independent loads: per-record weights
// lane-parallel (lane k owns record k of a batch of 32), then float4 rows.
struct MergeArgs {          // what the merge needs, passed by value
  const float* partials;
  float* out;
  uint32_t* tickets;
  int G, Hq, Hkv;
};

// Partial record k of the pair is at index rec0 + k * rstride.
template <int D>
__device__ __noinline__ void merge_partials(MergeArgs p, int bg, int rec0, int rstride, int nrec, int lane) {
  const int G = p.G;
  const int rs = G * (D + 2);
  const int b = bg / p.Hkv, g = bg - b * p.Hkv;
  // row maxima and normalisers
  float ms[8], ls[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) { ms[r] = -INFINITY; ls[r] = 0.f; }
  for (int k0 = 0; k0 < nrec; k0 += 32) {
    const int k = k0 + lane;
    const float* st = p.partials + (long long)(rec0 + k * rstride) * rs;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      float mk = -INFINITY;
      if (r < G && k < nrec) mk = __ldcg(st + r * (D + 2));
#pragma unroll
      for (int o = 16; o; o >>= 1) mk = fmaxf(mk, __shfl_xor_sync(kFull, mk, o));
      ms[r] = fmaxf(ms[r], mk);
    }
  }
  for (int k0 = 0; k0 < nrec; k0 += 32) {
    const int k = k0 + lane;
    const float* st = p.partials + (long long)(rec0 + k * rstride) * rs;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      float lk = 0.f;
      if (r < G && k < nrec && ms[r] != -INFINITY) lk = __ldcg(st + r * (D + 2) + 1) * ex2(__ldcg(st + r * (D + 2)) - ms[r]);
#pragma unroll
      for (int o = 16; o; o >>= 1) lk += __shfl_xor_sync(kFull, lk, o);
      ls[r] += lk;
    }
  }
  // output rows: lane owns D/32 consecutive dims of every row.  Records are
  // the outer loop, so the loads of all rows of a record (and of the next
  // record) are independent and in flight together.
  constexpr int DPL = D / 32;
  float o[8][DPL];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int i = 0; i < DPL; ++i) o[r][i] = 0.f;
  for (int k0 = 0; k0 < nrec; k0 += 32) {
    const int k = k0 + lane;
    float f[8];                                  // weight of record k in each row
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      f[r] = 0.f;
      if (r < G && k < nrec && ms[r] != -INFINITY)
        f[r] = ex2(__ldcg(p.partials + (long long)(rec0 + k * rstride) * rs + r * (D + 2)) - ms[r]);
    }
    const int kn = min(32, nrec - k0);
#pragma unroll 2
    for (int kk = 0; kk < kn; ++kk) {
      const float* base = p.partials + (long long)(rec0 + (k0 + kk) * rstride) * rs + 2 + lane * DPL;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const float fk = __shfl_sync(kFull, f[r], kk);
        if (r < G) {
#pragma unroll
          for (int i = 0; i < DPL; i += 2) {
            const float2 v = __ldcg(reinterpret_cast<const float2*>(base + r * (D + 2) + i));
            o[r][i] = fmaf(fk, v.x, o[r][i]);
            o[r][i + 1] = fmaf(fk, v.y, o[r][i + 1]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    if (r >= G) break;
    const float inv = ls[r] > 0.f ? 1.f / ls[r] : 0.f;
    float* dst = p.out + ((long long)b * p.Hq + g * G + r) * D + lane * DPL;
#pragma unroll
    for (int i = 0; i < DPL; ++i) dst[i] = o[r][i] * inv;
  }
  if (lane == 0) p.tickets[bg] = 0u;
}

}  // namespace dec
}  // namespace kvc
