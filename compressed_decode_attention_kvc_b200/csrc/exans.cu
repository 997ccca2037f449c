// Lossless exponent-split codec for high-precision (BF16) pages.
//
// "ExANS komprimerer KV-cache og goer AI-svar hurtigere paa H100 GPU"
// (ainews.dk, on "ExANS - Lossless KV cache compression at 622 GB/s on
// H100"): each BF16 value splits into an exponent stream and a sign +
// mantissa stream; exponents repeat inside a KV cache, so that stream is
// coded with an asymmetric numeral system around a per-group centre, each
// physical block (one K group and one V group per layer) on its own.
//
// Here a group is one page of one pool ([Hkv][16][D] bf16, N values).  The
// exponent of each value becomes a symbol (exponent - centre + 8 in 0..14,
// else the escape 15, whose exponent byte goes to an escape stream); the
// centre is the group's most frequent exponent.  The symbols are coded with
// byte-wise rANS (32-bit state in [2^23, 2^31), 12-bit frequencies, a static
// table per group) by 32 interleaved states, one per lane of a warp: lane i
// codes elements 128c + 4i + r.  After each symbol the lanes whose state fell
// below 2^23 read one byte each from the shared stream in lane order, then a
// second round likewise, so a warp decodes with ballots and coalesced byte
// reads.  The sign + mantissa bytes stay raw.  A group whose coded blob would
// exceed its raw bytes is stored raw.
//
// Blob (little-endian, 16-byte multiple): u32 total, mode (0 raw, 1 coded),
// N, centre, escapes, stream bytes; 8 zero bytes; u16 f[16]; then either the
// 2N raw bytes, or N sign+mantissa bytes, the escape bytes zero-padded to 16,
// and the rANS stream (32 initial states, then the renormalisation bytes)
// zero-padded to 16.
#include "kvc_internal.cuh"

namespace kvc {
namespace {

constexpr int kExHeader = 64;
constexpr int kExEscape = 15;
constexpr int kExBias = 8;
constexpr uint32_t kExL = 1u << 23;          // state lower bound
constexpr int kExScaleBits = 12;
constexpr uint32_t kExM = 1u << kExScaleBits;
constexpr int kExWarps = 4;                  // groups in flight per CTA
constexpr uint32_t kFull = 0xffffffffu;

__host__ __device__ __forceinline__ long long round16(long long x) { return (x + 15) / 16 * 16; }

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// element r (0..3) of a lane's 4-element quad (two 32-bit words)
__device__ __forceinline__ uint32_t quad_elem(const uint2& v, int r) {
  return ((r < 2 ? v.x : v.y) >> (16 * (r & 1))) & 0xFFFFu;
}

__device__ __forceinline__ int symbol_of(uint32_t exp, int centre) {
  const int d = (int)exp - centre + kExBias;
  return (d >= 0 && d < kExEscape) ? d : kExEscape;
}

// exclusive prefix over lanes and total of per-lane counts in 0..4
__device__ __forceinline__ void count_scan(int cnt, unsigned lt, int& prefix, int& total) {
  const unsigned b0 = __ballot_sync(kFull, cnt & 1), b1 = __ballot_sync(kFull, cnt & 2),
                 b2 = __ballot_sync(kFull, cnt & 4);
  prefix = __popc(b0 & lt) + 2 * __popc(b1 & lt) + 4 * __popc(b2 & lt);
  total = __popc(b0) + 2 * __popc(b1) + 4 * __popc(b2);
}

struct EncSmem {
  uint32_t hist[256];   // exponent histogram
  uint32_t cnt[16];     // symbol counts
  uint32_t fc[16];      // f | cum << 16
  uint32_t rcp[16];     // x / f = umulhi(x, rcp) >> rsh for x < 2^31 (f >= 2)
  uint32_t rsh[16];
};

// One warp per group; the group's blob is built in its workspace slot of
// 4N + 192 bytes: header, sign+mantissa bytes, escape area (N), and a stream
// area (2N + 128 bytes, the most 2 bytes per symbol can take) written
// backwards from its end, then moved down behind the escapes.  Pass 1 also
// keeps each value's exponent byte at the front of the stream area, so the
// later passes read N bytes instead of the 2N of the page: after the chunks
// from c on are coded the stream holds at most 256 bytes per chunk, and its
// front (at or above offset 2N + 192 + 256c) never reaches the exponents of
// the chunks before c (which end at 2N + 64 + 128c).
__global__ void __launch_bounds__(kExWarps * 32) exans_encode_kernel(const uint16_t* __restrict__ src,
                                                                    const int32_t* __restrict__ page_ids,
                                                                    long long n_src, uint32_t* flags,
                                                                    int n, long long N, unsigned char* ws) {
  __shared__ EncSmem smem[kExWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long g = (long long)blockIdx.x * kExWarps + warp;
  if (g >= n) return;
  EncSmem& S = smem[warp];
  const unsigned lt = lanemask_lt();
  long long pid = page_ids ? (long long)__ldg(page_ids + g) : g;
  if (pid < 0 || pid >= n_src) {          // an id outside the source: code page 0, flag it
    if (flags && lane == 0) atomicOr(flags, 1u);
    pid = 0;
  }
  const uint16_t* x = src + pid * N;
  const long long cap = 4 * N + 192;
  unsigned char* slot = ws + g * cap;
  const int chunks = (int)(N / 128);
  for (int i = lane; i < 256; i += 32) S.hist[i] = 0u;
  if (lane < 16) S.cnt[lane] = 0u;
  __syncwarp();

  // pass 1: exponent histogram; sign+mantissa bytes; exponent bytes kept
  // for passes 2 and 3 (chunks is a multiple of 8; four chunks' loads are
  // issued together)
  uint32_t* xe = reinterpret_cast<uint32_t*>(slot + kExHeader + 2 * N);
  for (int c0 = 0; c0 < chunks; c0 += 4) {
    uint2 vq[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) vq[k] = *reinterpret_cast<const uint2*>(x + (long long)(c0 + k) * 128 + 4 * lane);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t smw = 0, ew = 0;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const uint32_t b = quad_elem(vq[k], r);
        atomicAdd(&S.hist[(b >> 7) & 0xFFu], 1u);
        smw |= (((b >> 8) & 0x80u) | (b & 0x7Fu)) << (8 * r);
        ew |= ((b >> 7) & 0xFFu) << (8 * r);
      }
      *reinterpret_cast<uint32_t*>(slot + kExHeader + (long long)(c0 + k) * 128 + 4 * lane) = smw;
      xe[(long long)(c0 + k) * 32 + lane] = ew;
    }
  }
  __syncwarp();
  // centre: the most frequent exponent, the smallest among ties
  uint32_t best = 0;
  for (int i = lane; i < 256; i += 32) best = max(best, (S.hist[i] << 8) | (255u - i));
  best = __reduce_max_sync(kFull, best);
  const int centre = 255 - (int)(best & 255u);

  // pass 2: symbol counts; escape bytes in element order
  unsigned char* esc_out = slot + kExHeader + N;
  long long esc_base = 0;
  for (int c0 = 0; c0 < chunks; c0 += 4) {
   uint32_t eq[4];
#pragma unroll
   for (int k = 0; k < 4; ++k) eq[k] = xe[(long long)(c0 + k) * 32 + lane];
#pragma unroll
   for (int k = 0; k < 4; ++k) {
    uint32_t e[4];
    int s[4], nesc = 0;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      e[r] = (eq[k] >> (8 * r)) & 0xFFu;
      s[r] = symbol_of(e[r], centre);
      atomicAdd(&S.cnt[s[r]], 1u);
      nesc += s[r] == kExEscape;
    }
    int prefix, total;
    count_scan(nesc, lt, prefix, total);
    if (nesc) {
      int j = 0;
#pragma unroll
      for (int r = 0; r < 4; ++r)
        if (s[r] == kExEscape) esc_out[esc_base + prefix + j++] = (unsigned char)e[r];
    }
    esc_base += total;
   }
  }
  __syncwarp();
  // frequencies: f = max(1, n*4096/N) for present symbols, the remainder to
  // the largest f (the first among ties)
  if (lane == 0) {
    int f[16], sum = 0, arg = 0;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      const unsigned long long c = S.cnt[t];
      f[t] = c ? (int)max(1ull, c * kExM / (unsigned long long)N) : 0;
      sum += f[t];
      if (f[t] > f[arg]) arg = t;
    }
    f[arg] += (int)kExM - sum;
    uint32_t cum = 0;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      S.fc[t] = (uint32_t)f[t] | (cum << 16);
      cum += (uint32_t)f[t];
      // division by the frequency as a multiply (Granlund and Montgomery's
      // round-up reciprocal): with l = ceil(log2 f) and m = ceil(2^(31+l) / f)
      // < 2^32, floor(x / f) = floor(x * m / 2^(31+l)) for every x < 2^31,
      // since the rounding adds less than x / 2^(31+l) < 1/f
      const uint32_t fu = (uint32_t)f[t];
      const int l = fu > 1u ? 32 - __clz(fu - 1u) : 0;
      S.rcp[t] = fu > 1u ? (uint32_t)(((1ull << (31 + l)) + fu - 1u) / fu) : 0u;
      S.rsh[t] = fu > 1u ? (uint32_t)(l - 1) : 0u;
    }
  }
  __syncwarp();

  // pass 3: rANS over the steps in reverse, each step's bytes placed in
  // front of the later steps' (round-0 bytes, then round-1 bytes, lane order)
  unsigned char* area_end = slot + cap;
  long long written = 0;                     // warp-uniform
  uint32_t st = kExL;
  for (int c0 = chunks - 4; c0 >= 0; c0 -= 4) {
   uint32_t eq[4];
#pragma unroll
   for (int k = 0; k < 4; ++k) eq[k] = xe[(long long)(c0 + k) * 32 + lane];
#pragma unroll
   for (int k = 3; k >= 0; --k) {
#pragma unroll
    for (int r = 3; r >= 0; --r) {
      const int s = symbol_of((eq[k] >> (8 * r)) & 0xFFu, centre);
      const uint32_t fc = S.fc[s];
      const uint32_t f = fc & 0xFFFFu, cum = fc >> 16;
      const uint32_t xmax = f << (23 - kExScaleBits + 8);
      uint32_t first = 0, second = 0;
      int nb = 0;
      const uint32_t low = st & 0xFFu;
      if (st >= xmax) {
        st >>= 8;
        first = low;
        nb = 1;
      }
      if (st >= xmax) {
        second = low;
        first = st & 0xFFu;
        st >>= 8;
        nb = 2;
      }
      // (st / f) << 12 + st % f + cum, with st < f * 2^19 <= 2^31 here
      const uint32_t q = f == 1u ? st : (__umulhi(st, S.rcp[s]) >> S.rsh[s]);
      st = st + cum + q * (kExM - f);
      const unsigned b1 = __ballot_sync(kFull, nb >= 1), b2 = __ballot_sync(kFull, nb == 2);
      const int n1 = __popc(b1), n2 = __popc(b2);
      written += n1 + n2;
      unsigned char* blk = area_end - written;
      if (nb >= 1) blk[__popc(b1 & lt)] = (unsigned char)first;
      if (nb == 2) blk[n1 + __popc(b2 & lt)] = (unsigned char)second;
    }
   }
  }
  written += 128;
  {
    unsigned char* p0 = area_end - written + 4 * lane;
#pragma unroll
    for (int k = 0; k < 4; ++k) p0[k] = (unsigned char)(st >> (8 * k));
  }
  const long long nesc = S.cnt[kExEscape];
  const long long esc_pad = round16(nesc);
  const long long total = kExHeader + N + esc_pad + round16(written);
  uint32_t hdr[6];
  if (total > kExHeader + 2 * N) {
    // raw: the 2N bytes as they are
    const uint4* s4 = reinterpret_cast<const uint4*>(x);
    uint4* d4 = reinterpret_cast<uint4*>(slot + kExHeader);
    for (long long i = lane; i < N / 8; i += 32) d4[i] = s4[i];
    hdr[0] = (uint32_t)(kExHeader + 2 * N);
    hdr[1] = 0u;
    hdr[2] = (uint32_t)N;
    hdr[3] = hdr[4] = hdr[5] = 0u;
  } else {
    if (lane < esc_pad - nesc) esc_out[nesc + lane] = 0;
    // move the stream down behind the escapes (destination below source:
    // each 32-byte piece is read by the warp before it is written)
    unsigned char* dsts = slot + kExHeader + N + esc_pad;
    const unsigned char* srcs = area_end - written;
    for (long long o = 0; o < written; o += 32) {
      const bool ok = o + lane < written;
      const unsigned char b = ok ? srcs[o + lane] : 0;
      __syncwarp();
      if (ok) dsts[o + lane] = b;
      __syncwarp();
    }
    if (lane < round16(written) - written) dsts[written + lane] = 0;
    hdr[0] = (uint32_t)total;
    hdr[1] = 1u;
    hdr[2] = (uint32_t)N;
    hdr[3] = (uint32_t)centre;
    hdr[4] = (uint32_t)nesc;
    hdr[5] = (uint32_t)written;
  }
  const bool coded = hdr[1] == 1u;
  if (lane < 16) {
    uint32_t v = 0;
    if (lane < 6) {
      v = hdr[lane];
    } else if (lane >= 8 && coded) {
      const int t = 2 * (lane - 8);
      v = (S.fc[t] & 0xFFFFu) | ((S.fc[t + 1] & 0xFFFFu) << 16);
    }
    reinterpret_cast<uint32_t*>(slot)[lane] = v;
  }
}

// Offsets of the compacted blobs: offsets[i] = sum of the totals before i.
// One CTA of 1024 threads, each over a contiguous range of groups.
__global__ void __launch_bounds__(1024) exans_scan_kernel(const unsigned char* ws, long long cap, int n,
                                                          long long* offsets) {
  __shared__ long long part[1024];
  const int t = threadIdx.x;
  const long long per = ((long long)n + 1023) / 1024;
  const long long lo = t * per, hi = min((long long)n, lo + per);
  long long s = 0;
  for (long long i = lo; i < hi; ++i) s += *reinterpret_cast<const uint32_t*>(ws + i * cap);
  part[t] = s;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    const long long v = t >= o ? part[t - o] : 0;
    __syncthreads();
    part[t] += v;
    __syncthreads();
  }
  long long base = t ? part[t - 1] : 0;
  for (long long i = lo; i < hi; ++i) {
    offsets[i] = base;
    base += *reinterpret_cast<const uint32_t*>(ws + i * cap);
  }
  if (t == 1023) offsets[n] = part[1023];
}

// Copy each slot's blob to its offset; one warp per group, 16-byte moves.
__global__ void __launch_bounds__(256) exans_compact_kernel(const unsigned char* ws, long long cap, int n,
                                                            const long long* offsets, unsigned char* dst) {
  const long long g = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (g >= n) return;
  const unsigned char* s = ws + g * cap;
  const long long total = *reinterpret_cast<const uint32_t*>(s);
  const uint4* s4 = reinterpret_cast<const uint4*>(s);
  uint4* d4 = reinterpret_cast<uint4*>(dst + offsets[g]);
  for (long long i = lane; i < total / 16; i += 32) d4[i] = s4[i];
}

// One warp per group.  The stream is read through a 256-byte ring in shared
// memory holding stream bytes [base, base + 256); once the read position
// passes base + 128 the consumed half is refilled with the next 128 bytes,
// which a register per lane has prefetched one refill ahead (the load has
// the ~10 steps until the next refill to arrive).
__global__ void __launch_bounds__(kExWarps * 32) exans_decode_kernel(const unsigned char* __restrict__ pool,
                                                                    const long long* __restrict__ offsets,
                                                                    int n_blobs, const int32_t* __restrict__ ids,
                                                                    long long src_bytes, int n, long long N,
                                                                    uint16_t* __restrict__ dst, uint32_t* flags) {
  __shared__ unsigned char tab[kExWarps][kExM];
  __shared__ uint32_t fcs[kExWarps][16];
  __shared__ __align__(16) unsigned char ring[kExWarps][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long g = (long long)blockIdx.x * kExWarps + warp;
  if (g >= n) return;
  const unsigned lt = lanemask_lt();
  const long long id = ids ? (long long)ids[g] : g;
  bool bad = id < 0 || id >= n_blobs;
  long long o0 = 0, o1 = 0;
  if (!bad) {
    o0 = offsets[id];
    o1 = offsets[id + 1];
    bad = o0 < 0 || o1 > src_bytes || o1 - o0 < kExHeader || (o0 & 15) != 0;
  }
  uint32_t h = 0;
  if (!bad && lane < 16) h = reinterpret_cast<const uint32_t*>(pool + o0)[lane];
  const uint32_t total = __shfl_sync(kFull, h, 0), mode = __shfl_sync(kFull, h, 1);
  const uint32_t nn = __shfl_sync(kFull, h, 2), centre = __shfl_sync(kFull, h, 3);
  const long long nesc = __shfl_sync(kFull, h, 4), nstream = __shfl_sync(kFull, h, 5);
  // frequencies of lanes 0..15 and their prefix
  const uint32_t pair = __shfl_sync(kFull, h, 8 + ((lane >> 1) & 7));
  const uint32_t f = lane < 16 ? ((lane & 1) ? pair >> 16 : pair & 0xFFFFu) : 0u;
  uint32_t cum = f;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(kFull, cum, o);
    if (lane >= o) cum += v;
  }
  const uint32_t fsum = __shfl_sync(kFull, cum, 31);
  cum -= f;
  if (!bad) {
    bad = (long long)total != o1 - o0 || nn != (uint32_t)N || mode > 1u;
    if (mode == 0u) bad = bad || total != kExHeader + 2 * N;
    else bad = bad || nstream < 128 || fsum != kExM || centre > 255u ||
               (long long)total != kExHeader + N + round16(nesc) + round16(nstream);
  }
  if (bad) {
    if (lane == 0 && flags) atomicOr(flags, 1u);
    return;
  }
  uint16_t* out = dst + g * N;
  if (mode == 0u) {
    const uint4* s4 = reinterpret_cast<const uint4*>(pool + o0 + kExHeader);
    uint4* d4 = reinterpret_cast<uint4*>(out);
    for (long long i = lane; i < N / 8; i += 32) d4[i] = s4[i];
    return;
  }
  if (lane < 16) fcs[warp][lane] = f | (cum << 16);
  __syncwarp();
  for (int s = 0; s < 16; ++s) {
    const uint32_t fc = fcs[warp][s];
    const uint32_t fs = fc & 0xFFFFu, cs = fc >> 16;
    for (uint32_t i = lane; i < fs; i += 32) tab[warp][cs + i] = (unsigned char)s;
  }
  __syncwarp();

  const unsigned char* smp = pool + o0 + kExHeader;
  const unsigned char* escp = smp + N;
  const unsigned char* strm = escp + round16(nesc);
  const int slen = (int)round16(nstream);
  const int nesc32 = (int)nesc;
  auto stream_word = [&](int b) -> uint32_t {
    const int a = b + 4 * lane;
    return a + 4 <= slen ? *reinterpret_cast<const uint32_t*>(strm + a) : 0u;
  };
  unsigned char* rg = ring[warp];
  uint32_t x = *reinterpret_cast<const uint32_t*>(strm + 4 * lane);
  int base = 128, pos = 128, esc_pos = 0;
  *reinterpret_cast<uint32_t*>(rg + ((base + 4 * lane) & 255)) = stream_word(base);
  *reinterpret_cast<uint32_t*>(rg + ((base + 128 + 4 * lane) & 255)) = stream_word(base + 128);
  uint32_t nxt = stream_word(base + 256);
  __syncwarp();
  bool corrupt = false;
  const int chunks = (int)(N / 128);
  for (int c = 0; c < chunks; ++c) {
    const uint32_t smw = *reinterpret_cast<const uint32_t*>(smp + (long long)c * 128 + 4 * lane);
    int sy[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const uint32_t slot = x & (kExM - 1);
      const int s = tab[warp][slot];
      const uint32_t fc = fcs[warp][s];
      x = (fc & 0xFFFFu) * (x >> kExScaleBits) + slot - (fc >> 16);
      sy[r] = s;
      // both renormalisation rounds decided from x: a lane reads a round-0
      // byte if x < 2^23 and a round-1 byte if x < 2^15 ((x << 8) | b < 2^23)
      const bool need1 = x < kExL, need2 = x < (kExL >> 8);
      const unsigned bal1 = __ballot_sync(kFull, need1);
      if (bal1) {
        const unsigned bal2 = __ballot_sync(kFull, need2);
        const int n1 = __popc(bal1);
        const uint32_t by1 = rg[(pos + __popc(bal1 & lt)) & 255];
        const uint32_t by2 = rg[(pos + n1 + __popc(bal2 & lt)) & 255];
        if (need2) x = (x << 16) | (by1 << 8) | by2;
        else if (need1) x = (x << 8) | by1;
        pos += n1 + __popc(bal2);
      }
      if (pos >= base + 128) {                 // refill the consumed half
        __syncwarp();
        *reinterpret_cast<uint32_t*>(rg + ((base + 4 * lane) & 255)) = nxt;
        base += 128;
        nxt = stream_word(base + 256);
        __syncwarp();
      }
    }
    uint32_t e[4];
    int nesc_l = 0;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      e[r] = (uint32_t)(sy[r] - kExBias + (int)centre) & 0xFFu;
      nesc_l += sy[r] == kExEscape;
    }
    if (__any_sync(kFull, nesc_l != 0)) {
      int prefix, tot;
      count_scan(nesc_l, lt, prefix, tot);
      int j = 0;
#pragma unroll
      for (int r = 0; r < 4; ++r)
        if (sy[r] == kExEscape) {
          const int k = esc_pos + prefix + j++;
          if (k < nesc32) e[r] = escp[k];
          else corrupt = true;
        }
      esc_pos += tot;
    }
    // sign+mantissa bytes spread to the low bytes of two 16-bit halves
    const uint32_t s01 = __byte_perm(smw, 0u, 0x4140), s23 = __byte_perm(smw, 0u, 0x4342);
    const uint32_t o01 = ((s01 & 0x00800080u) << 8) | (s01 & 0x007F007Fu) | (e[0] << 7) | (e[1] << 23);
    const uint32_t o23 = ((s23 & 0x00800080u) << 8) | (s23 & 0x007F007Fu) | (e[2] << 7) | (e[3] << 23);
    *reinterpret_cast<uint2*>(out + (long long)c * 128 + 4 * lane) = make_uint2(o01, o23);
  }
  corrupt = corrupt || pos != nstream || esc_pos != nesc;
  if (__any_sync(kFull, corrupt) && lane == 0 && flags) atomicOr(flags, 2u);
}

}  // namespace

long long exans_slot_bytes(long long group_elems) { return 4 * group_elems + 192; }

cudaError_t launch_exans_encode(const void* src, const int32_t* page_ids, long long n_src, uint32_t* flags, int n,
                                long long group_elems, void* ws, long long* offsets, void* dst, cudaStream_t s) {
  const int grid = (int)((n + kExWarps - 1) / kExWarps);
  auto* w = static_cast<unsigned char*>(ws);
  exans_encode_kernel<<<grid, kExWarps * 32, 0, s>>>(static_cast<const uint16_t*>(src), page_ids, n_src, flags, n,
                                                     group_elems, w);
  const long long cap = exans_slot_bytes(group_elems);
  exans_scan_kernel<<<1, 1024, 0, s>>>(w, cap, n, offsets);
  exans_compact_kernel<<<(n + 7) / 8, 256, 0, s>>>(w, cap, n, offsets, static_cast<unsigned char*>(dst));
  return cudaGetLastError();
}

cudaError_t launch_exans_decode(const void* src, long long src_bytes, const long long* offsets, int n_blobs,
                                const int32_t* ids, int n, long long group_elems, void* dst, uint32_t* flags,
                                cudaStream_t s) {
  const int grid = (int)((n + kExWarps - 1) / kExWarps);
  exans_decode_kernel<<<grid, kExWarps * 32, 0, s>>>(static_cast<const unsigned char*>(src), offsets, n_blobs,
                                                     ids, src_bytes, n, group_elems, static_cast<uint16_t*>(dst), flags);
  return cudaGetLastError();
}

}  // namespace kvc
