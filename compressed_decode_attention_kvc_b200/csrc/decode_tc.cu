// Mixed-format paged decode attention on the tensor cores (sm_100a).
//
// Method: "Minima-KV" (twodots.gr), section "How mixed-format attention
// works" - every page is read in its own format directly as it is loaded (no
// dense shadow copy), each split emits a partial state (max score, sum of
// exponentials, output) and a common online-softmax normalisation merges
// them.  Ternary pages follow "Show HN: Vantage-V-AI" (newshot.cc), section
// "Core architecture" (codes {-1, 0, +1}, gamma = mean|X|, 4 codes per byte).
//
// Design (B200):
// * Work: the (sequence, KV-head group, page) units of the whole batch are
//   split over the CTAs of a persistent grid ("stream-K"), weighted by the
//   time a page costs: CTA W owns the units whose weighted start lies in
//   [W*C/NW, (W+1)*C/NW), a range that may span several (sequence, head
//   group) pairs, so ragged lengths and format mixes balance by
//   construction.  A CTA has one warp per KV head of its group (4, 2 or 1);
//   all its warps walk the same pages, each for its own head.
// * Staging: each CTA keeps a 2-slot ring in shared memory (8 KB per head
//   and slot; 4 KB at head_dim 64, 7 KB for two-head CTAs at head_dim 128),
//   holding the K groups then the V groups of up to 8 ternary pages, FP8
//   pages or one BF16 page (half a page where a slot is smaller), filled by
//   1-D TMA bulk copies (cp.async.bulk, no multicast) that complete on an
//   mbarrier; the heads' groups of a page are contiguous, so one copy moves
//   a page for all of them.  Page metadata (format, block-table slot, scales)
//   for 32 units at a time is loaded lane-parallel one chunk ahead.  The last
//   warp to release a slot refills it.
// * Math, register-sourced mma.sync, page tokens on M and the GQA group on N:
//   Q.K^T of ternary pages on int8 MMAs (codes as +-64 bytes: one AND and
//   one shift per four codes; Q as 15-bit int8 hi/lo digits per query head),
//   of FP8 pages on f16 MMAs, of BF16 pages on bf16 MMAs.  P.V has V^T as A
//   and P^T as B: with at most 4 query heads, ternary pages take one int8
//   MMA per m-tile and page pair (P as two exact unsigned digits, int32 sums
//   folded into fp32 once per entry); otherwise f16 / bf16 MMAs with P as a
//   hi + lo pair (movmatrix transposes the score tile).  No unpacked copy of
//   a page touches shared memory.
// * Softmax: online, in log2 units.  Full entries of 8 ternary pages test
//   the running maximum once, take P's digits relative to the entry's own
//   maximum and run their P.V as one straight run of code; shorter ternary
//   entries at GQA <= 4 test it per page pair (the maximum moves in whole
//   log2 units, so the digit sums rescale exactly by shifts); the other
//   paths use a lazy maximum that moves only when a score exceeds it by 2^8.  Per-page V scales are folded into P
//   relative to a per-warp reference scale.
// * Merge: each warp writes one partial state per (sequence, KV head) it
//   touched; the last writer for a pair (an atomic ticket, no waiting)
//   merges the pair's partials and writes the output rows.
#include "decode_common.cuh"

#include <math.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <utility>

namespace kvc {
namespace {

using namespace dec;

constexpr int kTcMaxBatchTpl = 1024;   // largest batch of the tensor-core kernel

constexpr int kEntries = 2;          // ring entries per warp
constexpr float kTau = 8.0f;         // lazy-max threshold, log2 units
// Work weights of one page of one KV head, in quarters of a ternary page: the
// time a page costs a warp (measured on B200; unpacking, the tensor-core
// work per byte and the per-entry issue work make a page's time grow more
// slowly than its bytes).  kCostMax bounds every weight.
constexpr int kCostTern = 4, kCostMax = 24;
template <int D, bool NARROW>
__host__ __device__ constexpr int cost_hp(int fmt) {
  return fmt == KVC_FMT_BF16 ? (D == 256 ? 21 : (NARROW ? 16 : 22)) : (NARROW || D == 256 ? 9 : 16);
}


// HPC: KV heads per CTA (1, 2 or 4), one warp each.  The warps of a CTA walk
// the same pages; a ring slot holds those pages for all HPC heads.
// A ring entry holds 8 KB per head (4 KB at head_dim 64).  Two-head CTAs at
// head_dim 128 (CTAs of 64 threads, six per SM by registers) take 7 KB, so
// that six of them also fit the shared memory with the sequence tables of a
// few hundred sequences (a BF16 page then fills two half-page entries).
template <int D, int HPC>
struct Shape {
  static constexpr int kEntryBytes = D == 64 ? 4096 : (D == 128 && HPC == 2 ? 7168 : 8192);   // per head
  static constexpr int kHeadHalf = kEntryBytes / 2;         // K (or V) bytes of one head per slot
  static constexpr int kSlotBytes = HPC * kEntryBytes;      // one ring slot of the CTA
  static constexpr int kHalf = kSlotBytes / 2;              // K region | V region
  static constexpr int kSteps = D / 16;                    // k-steps of Q.K^T = m-tiles of P.V
  static constexpr int kWPT = D / 64;                      // K words (16 dims) per thread per token
  static constexpr int kQ8 = 4 * kWPT;                     // int8 Q fragments (hi or lo) per thread
  static constexpr int kUPT = D / 64;                      // V units (8 dims) per thread
  static constexpr int kVW = kUPT > 1 ? kUPT / 2 : 1;      // V code words per thread per token
  static constexpr int kTernCap = kHeadHalf / (4 * D) < kMaxPages ? kHeadHalf / (4 * D) : kMaxPages;
  static constexpr int kFp8Cap = kHeadHalf / (16 * D);
  static constexpr int kBf16Rows = kHeadHalf / (2 * D) >= 16 ? 16 : 8;   // token rows of a BF16 page per entry
  static constexpr int kQBytes = 2 * kSteps * 32 * 4;      // per-warp f16 Q fragments
  static_assert(kTernCap >= 1 && kFp8Cap >= 1 && kHeadHalf >= 8 * 2 * D, "an entry must hold one page of each format");
};




// ----------------------------------------------------------- the worker
// NARROW (GQA group of at most 4 query heads): MMA column 2h + part belongs
// to query head h.  In Q.K^T of ternary pages the two parts are Q's int8 hi
// and lo (one int8 MMA per k-step instead of two); in P.V they are P's f16
// hi and lo (one MMA per m-tile carries the split P); elsewhere part 1 is 0.
// Otherwise (WIDE, up to 8 query heads) column n is query head n.
template <int D, int HPC, bool NARROW>
struct Worker {
  using S = Shape<D, HPC>;
  const DecodeParams& p;
  const Prologue& pr;
  unsigned char* ring;     // the CTA's kEntries slots
  uint32_t* qsm;           // this warp's bf16 Q fragments: [kSteps / 2][32 lanes][4]
  Desc* desc;              // this warp's [kEntries] entry descriptions
  uint64_t* bars;          // the CTA's [kEntries] slot barriers
  int* cnt;                // the CTA's [kEntries] counts of warps done with a slot
  int lane, gid, tig;
  int wi;                  // warp in the CTA = KV head within the group
  int u1, cursor, cb;      // unit range end, next unit to issue, chunk base
  int bf16_half;           // next half of a BF16 page to issue (half-page entries)
  Meta cur, nxt;
  MetaA nxa;
  bool nxt_b_pending;       // nxt still needs phase B (its phase A loads are in nxa)
  bool nxa_pending;         // nxa still needs phase A (the chunk after nxt)
  int W;
  uint32_t wait_limit;      // tries of a bounded slot wait

  // per (sequence, KV head) state
  int cur_bg;
  // Q of the group as int8 hi/lo fragments for ternary pages:
  // q ~= sq * (128 * hi + lo), sq = max|q| / 16256 per query head
  // (NARROW: qh holds this thread's column, hi or lo of one head)
  uint32_t qh[S::kQ8], ql[NARROW ? 1 : S::kQ8];
  float kq0, kq1;          // score scale of the thread's score columns: sq * log2(e) * softmax_scale / 64
  float acc[S::kSteps][4];
  float m0, m1, l0, l1, uref, inv_uref;
  bool q_f16;              // Q of the group fits the f16 range (FP8 pages use f16 products)

  __device__ Worker(const DecodeParams& pp, const Prologue& prr, unsigned char* r, uint32_t* q, Desc* d,
                    uint64_t* b, int w)
      : p(pp), pr(prr), ring(r), qsm(q), desc(d), bars(b), wi(w) {}
  __device__ void set_counts(int* c) { cnt = c; }

  __device__ __forceinline__ int shfl(int v, int src) { return __shfl_sync(kFull, v, src); }
  __device__ __forceinline__ float shflf(float v, int src) { return __shfl_sync(kFull, v, src); }

  // Describe the next entry of the CTA's unit range in this warp's desc[slot]
  // (every warp of the CTA forms the same entries); with `copy`, also fill
  // ring slot `slot` for all HPC heads.  False when the range is exhausted.
  __device__ bool issue(int slot, bool copy) {
    if (cursor >= u1) return false;
    int li = cursor - cb;
    if (li >= 32) {
      if (nxt_b_pending) meta_phase_b(p, nxa, nxt);   // only when a chunk took one entry
      cur = nxt;
      cb += 32;
      li -= 32;
      nxt_b_pending = false;
      nxa_pending = true;
    }
    const int m0l = shfl(cur.m, li);
    const int f0 = meta_fmt(m0l), bg0 = meta_bg(m0l) * HPC + wi;   // this warp's (sequence, KV head)
    int np = 1, row0 = 0, nrows, advance = 1;
    int bytes_per_page = 0, src_off = 0;
    if (f0 == KVC_FMT_BF16 && S::kBf16Rows == 8) {
      // a BF16 page of this head size fills two entries of 8 token rows
      const int ntok = meta_ntok(m0l);
      row0 = 8 * bf16_half;
      nrows = min(8, ntok - row0);
      bytes_per_page = 8 * 2 * D;
      src_off = row0 * 2 * D;
      if (bf16_half == 0 && ntok > 8) {
        bf16_half = 1;
        advance = 0;
      } else {
        bf16_half = 0;
      }
    } else {
      if (f0 != kSkip) {
        const int cap = f0 == KVC_FMT_TERNARY2 ? S::kTernCap : (f0 == KVC_FMT_FP8_E4M3 ? S::kFp8Cap : 1);
        // same format and (sequence, KV head); only the last page of a
        // (sequence, KV head) can be partial, and it ends the run
        const bool ok = lane >= li && (cb + lane) < u1 && cur.m >= 0 && ((cur.m ^ m0l) & ~(31 << 2)) == 0;
        const uint32_t run = __ballot_sync(kFull, ok) >> li;
        const int len = (run == 0xffffffffu) ? 32 : __ffs(~run) - 1;
        np = min(len, cap);
        bytes_per_page = group_bytes(f0, D);
      }
      advance = np;
      nrows = meta_ntok(shfl(cur.m, min(li + np - 1, 31)));
    }
    Desc& d = desc[slot];
    if (lane == li) {
      d.fmt = f0;
      d.np = np;
      d.bg = bg0;
      d.nrows = nrows;
      d.row0 = row0;
    }
    const int k = lane - li;
    const bool mine = k >= 0 && k < np;
    if (mine) {
      d.ks[k] = cur.ks;
      d.vs[k] = cur.vs;
    }
    // largest V scale of the entry (scales are >= 0: their bits order as unsigned)
    const uint32_t vmax = __reduce_max_sync(kFull, mine ? __float_as_uint(cur.vs) : 0u);
    if (lane == li) d.gvmax = __uint_as_float(vmax);
    __syncwarp();
    if (copy) {
      // the HPC heads' groups of a page are contiguous: one copy per page
      // for K and one for V (BF16 half pages: one per head, 8 rows each)
      const bool half = f0 == KVC_FMT_BF16 && S::kBf16Rows == 8;
      const int per = half ? 8 * 2 * D : HPC * bytes_per_page;   // bytes per copy
      const int ncopy = f0 == kSkip ? 0 : (half ? HPC : np);
      fence_proxy_async();
      if (lane == 0) mbar_arrive_expect_tx(&bars[slot], (uint32_t)(2 * ncopy * per));
      __syncwarp();
      const int src_lane = half ? li : li + lane;
      const int grp = shfl(cur.grp, min(src_lane, 31)) - wi;       // group of head 0 of the CTA
      if (lane < ncopy) {
        const unsigned char* kb;
        const unsigned char* vb;
        if (f0 == KVC_FMT_TERNARY2) {
          kb = static_cast<const unsigned char*>(p.cache.k_tern);
          vb = static_cast<const unsigned char*>(p.cache.v_tern);
        } else if (f0 == KVC_FMT_FP8_E4M3) {
          kb = static_cast<const unsigned char*>(p.cache.k_fp8);
          vb = static_cast<const unsigned char*>(p.cache.v_fp8);
        } else {
          kb = static_cast<const unsigned char*>(p.cache.k_bf16);
          vb = static_cast<const unsigned char*>(p.cache.v_bf16);
        }
        const int gb = group_bytes(f0, D);
        const long long off = half ? (long long)(grp + lane) * gb + src_off : (long long)grp * gb;
        unsigned char* e = ring + slot * S::kSlotBytes + lane * per;
        bulk_g2s(e, kb + off, (uint32_t)per, &bars[slot]);
        bulk_g2s(e + S::kHalf, vb + off, (uint32_t)per, &bars[slot]);
      }
    }
    cursor += advance;
    // Metadata prefetch for the next chunk, issued only after this entry's
    // copies: the proxy fence above would otherwise wait for these global
    // loads.  Phase B (which reads phase A's block-table entries) waits until
    // three quarters of the current chunk are issued, so those loads have
    // landed; its scale loads are first used at the next chunk switch.
    if (nxa_pending) {
      meta_phase_a(p, pr, cb + 32, u1, lane, HPC, wi, nxa);
      nxa_pending = false;
      nxt_b_pending = true;
    } else if (nxt_b_pending && cursor - cb >= 24) {
      meta_phase_b(p, nxa, nxt);
      nxt_b_pending = false;
    }
    return true;
  }

  // Start a new (sequence, KV head): load Q as f16 B fragments, reset state.
  __device__ void begin(int bg) {
    cur_bg = bg;
    const int b = bg / p.Hkv, g = bg - (bg / p.Hkv) * p.Hkv;
    const int r = NARROW ? gid >> 1 : gid;   // query head within the group
    uint32_t raw[S::kWPT * 8];               // 16 * kWPT bf16 of row r
    if (r < p.G) {
      const uint4* src = reinterpret_cast<const uint4*>(
          reinterpret_cast<const uint16_t*>(p.q) + ((long long)b * p.Hq + g * p.G + r) * D + 16 * tig * S::kWPT);
#pragma unroll
      for (int i = 0; i < 2 * S::kWPT; ++i) {
        const uint4 v = __ldg(src + i);
        raw[4 * i] = v.x; raw[4 * i + 1] = v.y; raw[4 * i + 2] = v.z; raw[4 * i + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < S::kWPT * 8; ++i) raw[i] = 0u;
    }
    // bf16 B fragments for FP8 / BF16 pages (Q as given), kept in shared
    // memory: fragment ri = (Q[dlo], Q[dlo + 8]), dlo = 16 * (ri >> 3) +
    // (ri & 7) (thread-local dims), stored at [ri >> 2][lane][ri & 3]
#pragma unroll
    for (int ri = 0; ri < 2 * S::kSteps; ++ri) {
      const int wl = ri >> 3, j = ri & 7;
      const uint32_t wa = raw[8 * wl + (j >> 1)], wb = raw[8 * wl + 4 + (j >> 1)];
      const uint32_t v = (NARROW && (gid & 1)) ? 0u : prmt(wa, wb, (j & 1) ? 0x7632u : 0x5410u);
      qsm[((ri >> 2) * 32 + lane) * 4 + (ri & 3)] = v;
    }
    // int8 hi/lo B fragments for ternary pages.  Fragment j carries, in
    // byte i, the thread-local dim 16 * (j >> 2) + 4 * i + (j & 3): the dims
    // whose codes tern8(word j >> 2, j & 3) puts in the same byte slots.
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < S::kWPT * 8; ++i)
      amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(raw[i] << 16)), fabsf(__uint_as_float(raw[i] & 0xFFFF0000u))));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
    const float inv = amax > 0.f ? 16256.f / amax : 0.f;
    q_f16 = __all_sync(kFull, amax <= 65504.f);
#pragma unroll
    for (int j = 0; j < S::kQ8; ++j) {
      uint32_t h = 0u, l = 0u;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int ld = 16 * (j >> 2) + 4 * i + (j & 3);
        const uint32_t w = raw[ld >> 1];
        const float x = __uint_as_float((ld & 1) ? (w & 0xFFFF0000u) : (w << 16));
        const int qi = __float2int_rn(x * inv);      // |qi| <= 16256
        const int hi = (qi + 64) >> 7;               // -127..127
        const int lo = qi - (hi << 7);               // -64..63
        h |= (uint32_t)(hi & 0xFF) << (8 * i);
        l |= (uint32_t)(lo & 0xFF) << (8 * i);
      }
      if constexpr (NARROW) {
        qh[j] = (gid & 1) ? l : h;
      } else {
        qh[j] = h;
        ql[j] = l;
      }
    }
    const float sq = amax * (1.f / 16256.f);
    const float f = p.scale_log2 * (1.f / 64.f);
    if constexpr (NARROW) {
      kq0 = __shfl_sync(kFull, sq, 8 * tig) * f;        // head tig (lane group gid = 2 * tig)
      kq1 = 0.f;
    } else {
      kq0 = __shfl_sync(kFull, sq, 8 * tig) * f;        // head 2 * tig (lane group gid = 2 * tig)
      kq1 = __shfl_sync(kFull, sq, 8 * tig + 4) * f;    // head 2 * tig + 1
    }
#pragma unroll
    for (int mt = 0; mt < S::kSteps; ++mt)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[mt][c] = 0.f;
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
    uref = 0.f;
    inv_uref = 0.f;
  }

  // Write this warp's partial state for cur_bg; the last writer merges.
  __device__ void finish() {
    if (cur_bg < 0) return;
    const int bg = cur_bg;
    const int G = p.G;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l0 += __shfl_xor_sync(kFull, l0, o);
      l1 += __shfl_xor_sync(kFull, l1, o);
    }
    const int rs = G * (D + 2);
    // record of (CTA W, pair bq, head wi): records of consecutive CTAs of a
    // pair are HPC apart, and distinct pairs never collide
    const int bq = bg / HPC;
    float* rec = p.partials + (long long)((W + bq) * HPC + wi) * rs;
    if constexpr (NARROW) {
      // head tig: columns 2 * tig (P hi) and 2 * tig + 1 (P lo) add up
      if (tig < G) {
        float* r = rec + tig * (D + 2);
        if (gid == 0) { r[0] = m0; r[1] = l0; }
#pragma unroll
        for (int mt = 0; mt < S::kSteps; ++mt) {
          const int la = mt, lb = mt + S::kSteps;
          const int da = 8 * (gid * S::kUPT + (la >> 3)) + (la & 7);
          const int db = 8 * (gid * S::kUPT + (lb >> 3)) + (lb & 7);
          r[2 + da] = (acc[mt][0] + acc[mt][1]) * uref;
          r[2 + db] = (acc[mt][2] + acc[mt][3]) * uref;
        }
      }
    }
    const int c0 = 2 * tig, c1 = 2 * tig + 1;
    if (!NARROW && gid == 0) {
      if (c0 < G) { rec[c0 * (D + 2)] = m0; rec[c0 * (D + 2) + 1] = l0; }
      if (c1 < G) { rec[c1 * (D + 2)] = m1; rec[c1 * (D + 2) + 1] = l1; }
    }
#pragma unroll
    for (int mt = 0; mt < S::kSteps && !NARROW; ++mt) {
      const int la = mt, lb = mt + S::kSteps;
      const int da = 8 * (gid * S::kUPT + (la >> 3)) + (la & 7);
      const int db = 8 * (gid * S::kUPT + (lb >> 3)) + (lb & 7);
      if (c0 < G) {
        rec[c0 * (D + 2) + 2 + da] = acc[mt][0] * uref;
        rec[c0 * (D + 2) + 2 + db] = acc[mt][2] * uref;
      }
      if (c1 < G) {
        rec[c1 * (D + 2) + 2 + da] = acc[mt][1] * uref;
        rec[c1 * (D + 2) + 2 + db] = acc[mt][3] * uref;
      }
    }
    __threadfence();
    __syncwarp();
    const int b = bg / p.Hkv, q = (bg - b * p.Hkv) / HPC;
    const int np = (pr.seqL[b] + kPage - 1) / kPage;
    const int x0 = pr.seqP[b] + q * np;
    const int w_first = pr.worker_of(x0), w_last = pr.worker_of(x0 + np - 1);
    unsigned last = 0;
    if (lane == 0) last = atomicAdd(p.tickets + bg, 1u) == (unsigned)(w_last - w_first);
    last = __shfl_sync(kFull, last, 0);
    if (!last) return;
    __threadfence();
    merge_partials<D>(MergeArgs{p.partials, p.out, p.tickets, p.G, p.Hq, p.Hkv}, bg, (w_first + bq) * HPC + wi,
                      HPC, w_last - w_first + 1, lane);
  }

  // ---------------------------------------------------------- Q . K^T
  // Ternary page: int8 tensor-core products of the codes (64 * c) with the
  // hi and lo parts of Q; the two int32 chains combine exactly to
  // 64 * sum_d c_d * q_int_d.
  __device__ __forceinline__ void qk_ternary(const unsigned char* kg, float (&s)[4]) {
    uint32_t wa[S::kWPT], wb[S::kWPT];
    const unsigned char* ra = kg + gid * (D / 4) + 4 * tig * S::kWPT;
    const unsigned char* rb = kg + (gid + 8) * (D / 4) + 4 * tig * S::kWPT;
    if constexpr (S::kWPT == 1) {
      wa[0] = lds<uint32_t>(ra); wb[0] = lds<uint32_t>(rb);
    } else if constexpr (S::kWPT == 2) {
      const uint2 a = lds<uint2>(ra), b = lds<uint2>(rb);
      wa[0] = a.x; wa[1] = a.y; wb[0] = b.x; wb[1] = b.y;
    } else {
      const uint4 a = lds<uint4>(ra), b = lds<uint4>(rb);
      wa[0] = a.x; wa[1] = a.y; wa[2] = a.z; wa[3] = a.w;
      wb[0] = b.x; wb[1] = b.y; wb[2] = b.z; wb[3] = b.w;
    }
    int th[4] = {0, 0, 0, 0}, tl[4] = {0, 0, 0, 0};
#pragma unroll
    for (int st = 0; st < S::kQ8 / 2; ++st) {
      const int j0 = 2 * st, j1 = 2 * st + 1;
      const uint32_t a0 = tern8(wa[j0 >> 2], j0 & 3), a1 = tern8(wb[j0 >> 2], j0 & 3);
      const uint32_t a2 = tern8(wa[j1 >> 2], j1 & 3), a3 = tern8(wb[j1 >> 2], j1 & 3);
      if constexpr (NARROW) {
        imma16832((st & 1) ? tl : th, a0, a1, a2, a3, qh[j0], qh[j1]);   // two chains
      } else {
        imma16832(th, a0, a1, a2, a3, qh[j0], qh[j1]);
        imma16832(tl, a0, a1, a2, a3, ql[j0], ql[j1]);
      }
    }
    if constexpr (NARROW) {
      // columns (hi, lo) of head tig: s[0] token gid, s[2] token gid + 8
      s[0] = (float)((th[0] + tl[0]) * 128 + (th[1] + tl[1]));
      s[2] = (float)((th[2] + tl[2]) * 128 + (th[3] + tl[3]));
      s[1] = s[3] = 0.f;
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) s[c] = (float)(th[c] * 128 + tl[c]);
    }
  }

  // f16 Q fragments of k-steps 2k and 2k + 1
  __device__ __forceinline__ uint4 qfrag(int k) const {
    return *reinterpret_cast<const uint4*>(qsm + (k * 32 + lane) * 4);
  }

  __device__ __forceinline__ void qk_fp8(const unsigned char* kg, float (&s)[4]) {
    float t[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int wl = 0; wl < S::kWPT; ++wl) {
      const uint4 xa = lds<uint4>(kg + gid * D + 16 * (tig * S::kWPT + wl));
      const uint4 xb = lds<uint4>(kg + (gid + 8) * D + 16 * (tig * S::kWPT + wl));
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {         // k-step 4*wl + q4: dims j, j+1 (and +8), j = 2*q4
        const int j = 2 * q4;
        const uint32_t sel = sel_pair(j & 3);
        const uint32_t pa = prmt(j < 4 ? xa.x : xa.y, j < 4 ? xa.z : xa.w, sel);
        const uint32_t pb = prmt(j < 4 ? xb.x : xb.y, j < 4 ? xb.z : xb.w, sel);
        const int st = 4 * wl + q4;
        const uint4 qv = qfrag(st >> 1);
        mma16816(t[st & 1], e4m3x2_f16(pa), e4m3x2_f16(pb), e4m3x2_f16(pa >> 16), e4m3x2_f16(pb >> 16),
                 bf16x2_f16((st & 1) ? qv.z : qv.x), bf16x2_f16((st & 1) ? qv.w : qv.y));
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) s[c] = t[0][c] + t[1][c];
  }

  // ROWS = token rows of the page held by the entry (16, or 8 for half pages)
  template <int ROWS>
  __device__ __forceinline__ void qk_bf16(const unsigned char* kg, float (&s)[4]) {
    float t[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int wl = 0; wl < S::kWPT; ++wl) {
      const unsigned char* ra = kg + gid * 2 * D + 32 * (tig * S::kWPT + wl);
      const unsigned char* rb = kg + (gid + 8) * 2 * D + 32 * (tig * S::kWPT + wl);
      const uint4 a0 = lds<uint4>(ra), a1 = lds<uint4>(ra + 16);
      uint4 b0 = make_uint4(0, 0, 0, 0), b1 = b0;
      if constexpr (ROWS == 16) {
        b0 = lds<uint4>(rb);
        b1 = lds<uint4>(rb + 16);
      }
      const uint32_t ya[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const uint32_t yb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {         // dims j = 2*q4 (+8) and 2*q4+1 (+8)
        const int st = 4 * wl + q4;
        const uint4 qv = qfrag(st >> 1);
        mma16816_bf16(t[st & 1], prmt(ya[q4], ya[4 + q4], 0x5410u), prmt(yb[q4], yb[4 + q4], 0x5410u),
                      prmt(ya[q4], ya[4 + q4], 0x7632u), prmt(yb[q4], yb[4 + q4], 0x7632u),
                      (st & 1) ? qv.z : qv.x, (st & 1) ? qv.w : qv.y);
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) s[c] = t[0][c] + t[1][c];
  }

  // ------------------------------------------------------------ P . V
  // token-pair masks (tokens >= nt contribute nothing)
  __device__ __forceinline__ void pv_masks(int nt, uint32_t& m01, uint32_t& m23) {
    const int t0 = 2 * tig;
    m01 = (t0 < nt ? 0x0000FFFFu : 0u) | (t0 + 1 < nt ? 0xFFFF0000u : 0u);
    m23 = (t0 + 8 < nt ? 0x0000FFFFu : 0u) | (t0 + 9 < nt ? 0xFFFF0000u : 0u);
  }

  // Threads with tig >= 2 read their token pairs in the order (2tig + 1, 2tig)
  // so that no two lanes of a load share a bank, and swap the two halves of
  // their P^T fragments to match.
  __device__ __forceinline__ void pv_ternary(const unsigned char* vg, uint32_t b0, uint32_t b1, int nt) {
    const int sw = tig >> 1;
    const int ta = 2 * tig + sw, tb = 2 * tig + 1 - sw;   // tokens of the low and high f16 halves
    const uint32_t hsel = sw ? 0x1032u : 0x3210u;
    b0 = prmt(b0, b0, hsel);
    b1 = prmt(b1, b1, hsel);
    const int vw0 = (gid * S::kUPT) >> 1;
    uint32_t w0[S::kVW], w1[S::kVW], w2[S::kVW], w3[S::kVW];
#pragma unroll
    for (int i = 0; i < S::kVW; ++i) {
      w0[i] = lds<uint32_t>(vg + ta * (D / 4) + 4 * (vw0 + i));
      w1[i] = lds<uint32_t>(vg + tb * (D / 4) + 4 * (vw0 + i));
      w2[i] = lds<uint32_t>(vg + (ta + 8) * (D / 4) + 4 * (vw0 + i));
      w3[i] = lds<uint32_t>(vg + (tb + 8) * (D / 4) + 4 * (vw0 + i));
    }
    uint32_t r01[S::kUPT], r23[S::kUPT];
#pragma unroll
    for (int ul = 0; ul < S::kUPT; ++ul) {
      const int gu = gid * S::kUPT + ul;
      const int wi = (gu >> 1) - vw0;
      const uint32_t sel = (gu & 1) ? 0x7632u : 0x5410u;
      r01[ul] = prmt(w0[wi], w1[wi], sel);
      r23[ul] = prmt(w2[wi], w3[wi], sel);
    }
    if (nt < kPage) {
      const uint32_t m01 = (ta < nt ? 0x0000FFFFu : 0u) | (tb < nt ? 0xFFFF0000u : 0u);
      const uint32_t m23 = (ta + 8 < nt ? 0x0000FFFFu : 0u) | (tb + 8 < nt ? 0xFFFF0000u : 0u);
#pragma unroll
      for (int ul = 0; ul < S::kUPT; ++ul) { r01[ul] &= m01; r23[ul] &= m23; }
    }
#pragma unroll
    for (int mt = 0; mt < S::kSteps; ++mt) {
      const int la = mt, lb = mt + S::kSteps;
      const int ua = la >> 3, ja = la & 7, ub = lb >> 3, jb = lb & 7;
      mma16816(acc[mt], tern2(r01[ua], 2 * ja), tern2(r01[ub], 2 * jb), tern2(r23[ua], 2 * ja),
               tern2(r23[ub], 2 * jb), b0, b1);
    }
  }

  __device__ __forceinline__ void pv_fp8(const unsigned char* vg, uint32_t b0, uint32_t b1, uint32_t lo0,
                                         uint32_t lo1, int nt) {
    const int t0 = 2 * tig;
    constexpr int NWD = 2 * S::kUPT;          // u32 words of the thread's 8*kUPT bytes
    uint32_t x0[NWD], x1[NWD], x2[NWD], x3[NWD];
    const int off = 8 * gid * S::kUPT;
#pragma unroll
    for (int i = 0; i < NWD; i += 2) {
      const uint2 a = lds<uint2>(vg + t0 * D + off + 4 * i);
      const uint2 b = lds<uint2>(vg + (t0 + 1) * D + off + 4 * i);
      const uint2 c = lds<uint2>(vg + (t0 + 8) * D + off + 4 * i);
      const uint2 e = lds<uint2>(vg + (t0 + 9) * D + off + 4 * i);
      x0[i] = a.x; x0[i + 1] = a.y; x1[i] = b.x; x1[i + 1] = b.y;
      x2[i] = c.x; x2[i + 1] = c.y; x3[i] = e.x; x3[i + 1] = e.y;
    }
    uint32_t m01 = 0xffffffffu, m23 = 0xffffffffu;
    if (nt < kPage) pv_masks(nt, m01, m23);
#pragma unroll
    for (int mt = 0; mt < S::kSteps; ++mt) {
      const int la = mt, lb = mt + S::kSteps;
      const int ua = la >> 3, ja = la & 7, ub = lb >> 3, jb = lb & 7;
      const int ia = 2 * ua + (ja >> 2), ib = 2 * ub + (jb >> 2);
      const uint32_t sa = sel_pair(ja & 3) & 0xFFu, sb = sel_pair(jb & 3) & 0xFFu;
      const uint32_t a0 = e4m3x2_f16(prmt(x0[ia], x1[ia], sa)) & m01;
      const uint32_t a1 = e4m3x2_f16(prmt(x0[ib], x1[ib], sb)) & m01;
      const uint32_t a2 = e4m3x2_f16(prmt(x2[ia], x3[ia], sa)) & m23;
      const uint32_t a3 = e4m3x2_f16(prmt(x2[ib], x3[ib], sb)) & m23;
      mma16816(acc[mt], a0, a1, a2, a3, b0, b1);
      if constexpr (!NARROW) mma16816(acc[mt], a0, a1, a2, a3, lo0, lo1);
    }
  }

  template <int ROWS>
  __device__ __forceinline__ void pv_bf16(const unsigned char* vg, uint32_t b0, uint32_t b1, uint32_t lo0,
                                          uint32_t lo1, int nt) {
    const int t0 = 2 * tig;
    const int off = 16 * gid * S::kUPT;       // bytes of the thread's dims in a row
    uint32_t m01 = 0xffffffffu, m23 = 0xffffffffu;
    if (nt < kPage) pv_masks(nt, m01, m23);
#pragma unroll
    for (int mt = 0; mt < S::kSteps; ++mt) {
      const int la = mt, lb = mt + S::kSteps;
      const int ua = la >> 3, ja = la & 7, ub = lb >> 3, jb = lb & 7;
      const int ba = off + 16 * ua + 4 * (ja >> 1), bb = off + 16 * ub + 4 * (jb >> 1);
      const uint32_t sa = (ja & 1) ? 0x7632u : 0x5410u, sb = (jb & 1) ? 0x7632u : 0x5410u;
      const uint32_t a0 = prmt(lds<uint32_t>(vg + t0 * 2 * D + ba), lds<uint32_t>(vg + (t0 + 1) * 2 * D + ba), sa) & m01;
      const uint32_t a1 = prmt(lds<uint32_t>(vg + t0 * 2 * D + bb), lds<uint32_t>(vg + (t0 + 1) * 2 * D + bb), sb) & m01;
      uint32_t a2 = 0u, a3 = 0u;
      if constexpr (ROWS == 16) {
        a2 = prmt(lds<uint32_t>(vg + (t0 + 8) * 2 * D + ba), lds<uint32_t>(vg + (t0 + 9) * 2 * D + ba), sa) & m23;
        a3 = prmt(lds<uint32_t>(vg + (t0 + 8) * 2 * D + bb), lds<uint32_t>(vg + (t0 + 9) * 2 * D + bb), sb) & m23;
      }
      mma16816_bf16(acc[mt], a0, a1, a2, a3, b0, b1);
      if constexpr (!NARROW) mma16816_bf16(acc[mt], a0, a1, a2, a3, lo0, lo1);
    }
  }

  // ---------------------------------- ternary pages, P.V on int8 (NARROW)
  // With at most 4 query heads a page pair (32 tokens) is one int8 MMA of
  // k = 32: V^T codes as A (tern8: 64 * code), P as B in two exact unsigned
  // digits, P ~= (256 * hi + lo) / 2^15 with P = p * gamma_v / gmax <= 1, hi in
  // column 2h and lo in column 2h + 1.  The int32 sums are exact; they are
  // folded into the float accumulators once per entry.  Token order along k
  // (both pages): (2t, 2t + 8, 2t + 1, 2t + 9) for t = tig, the order one
  // movmatrix of the (token gid, token gid + 8) digit pairs produces.
  static constexpr int kBB = 2 * S::kUPT;          // bytes of a V row this thread reads

  // The thread's byte block of V rows 2tig, 2tig + 8, 2tig + 1, 2tig + 9 of a
  // page, transposed: T[b] holds byte b of the four rows in that order.
  // Threads with tig >= 2 read (and order) 2tig + 1, 2tig + 9, 2tig, 2tig + 8
  // instead, so that no two lanes of a load share a bank; their P digits are
  // swapped to match (pv_digits).
  static constexpr int kVW4 = kBB < 4 ? 1 : kBB / 4;   // words of a V row this thread reads
  __device__ __forceinline__ void v_rows_t(const unsigned char* vg, uint32_t (&T)[kBB < 4 ? 4 : kBB]) {
    uint32_t r[4][kVW4];
    v_rows_ld(vg, r);
    v_rows_tr(r, T);
  }
  __device__ __forceinline__ void v_rows_ld(const unsigned char* vg, uint32_t (&r)[4][kVW4]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int tok = 2 * tig + ((q & 1) ? 8 : 0) + ((q >> 1) ^ (tig >> 1));
      const unsigned char* src = vg + tok * (D / 4) + kBB * gid;
      if constexpr (kBB == 2) {
        r[q][0] = lds<uint16_t>(src);
      } else if constexpr (kBB == 4) {
        r[q][0] = lds<uint32_t>(src);
      } else {
        const uint2 v = lds<uint2>(src);
        r[q][0] = v.x;
        r[q][1] = v.y;
      }
    }
  }
  __device__ __forceinline__ void v_rows_tr(const uint32_t (&r)[4][kVW4], uint32_t (&T)[kBB < 4 ? 4 : kBB]) {
#pragma unroll
    for (int w = 0; w < kVW4; ++w) {
      const uint32_t x01 = prmt(r[0][w], r[1][w], 0x5140u), x23 = prmt(r[0][w], r[1][w], 0x7362u);
      const uint32_t y01 = prmt(r[2][w], r[3][w], 0x5140u), y23 = prmt(r[2][w], r[3][w], 0x7362u);
      T[4 * w + 0] = prmt(x01, y01, 0x5410u);
      T[4 * w + 1] = prmt(x01, y01, 0x7632u);
      T[4 * w + 2] = prmt(x23, y23, 0x5410u);
      T[4 * w + 3] = prmt(x23, y23, 0x7632u);
    }
  }

  // Rescale of the digit sums by 2^-k (k >= 1): v = 256 hi + lo, floor(v / 2^k).
  // Within one entry (at most 8 pages) |hi| < 2^20 and |lo| < 2^21, so v
  // fits 31 bits.
  __device__ __forceinline__ static void shift_digits(int& hi, int& lo, int k) {
    const int w = (hi * 256 + lo) >> (k < 31 ? k : 31);
    hi = w >> 8;
    lo = w & 255;
  }

  __device__ __forceinline__ void process_ternary_int(const unsigned char* e, const Desc& d) {
    constexpr int GB = HPC * group_bytes(KVC_FMT_TERNARY2, D);   // page stride
    constexpr int NT = kBB < 4 ? 4 : kBB;
    e += wi * group_bytes(KVC_FMT_TERNARY2, D);
    const int np = d.np;
    const float gmax = d.gvmax;
    if (uref == 0.f && gmax > 0.f) {
      uref = gmax;
      inv_uref = 1.f / gmax;
    }
    const float r15 = gmax > 0.f ? 32768.f / gmax : 0.f;
    constexpr float kMagic = 12582912.f;     // 1.5 * 2^23: the low bits of x + kMagic hold round(x)
    int ai[S::kSteps][4];
#pragma unroll
    for (int mt = 0; mt < S::kSteps; ++mt)
#pragma unroll
      for (int c = 0; c < 4; ++c) ai[mt][c] = 0;
    float sA[4], sB[4] = {0.f, 0.f, 0.f, 0.f};
    qk_ternary(e, sA);
    if (np > 1) qk_ternary(e + GB, sB);
    for (int i = 0; i < np; i += 2) {
      const bool hasB = i + 1 < np;
      // the next pair's scores, independent of this pair's softmax and P.V
      float nA[4] = {0.f, 0.f, 0.f, 0.f}, nB[4] = {0.f, 0.f, 0.f, 0.f};
      if (i + 2 < np) {
        qk_ternary(e + (i + 2) * GB, nA);
        if (i + 3 < np) qk_ternary(e + (i + 3) * GB, nB);
      }
      uint32_t TA[NT], TB[NT];
      v_rows_t(e + S::kHalf + i * GB, TA);
      if (hasB) {
        v_rows_t(e + S::kHalf + (i + 1) * GB, TB);
      } else {
#pragma unroll
        for (int b = 0; b < NT; ++b) TB[b] = TA[b];   // any finite operand: its P digits are 0
      }
      const float scA = d.ks[i] * kq0, scB = hasB ? d.ks[i + 1] * kq0 : 0.f;
      float x0 = sA[0] * scA, x1 = sA[2] * scA, x2 = sB[0] * scB, x3 = sB[2] * scB;
      if (i + 2 >= np) {                      // the entry's last pair: masks
        const int ntA = hasB ? kPage : d.nrows, ntB = hasB ? d.nrows : 0;
        if (gid >= ntA) x0 = -INFINITY;
        if (gid + 8 >= ntA) x1 = -INFINITY;
        if (gid >= ntB) x2 = -INFINITY;
        if (gid + 8 >= ntB) x3 = -INFINITY;
      }
      const float mx = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
      // P <= 1 needs every score at or below the running maximum; the
      // maximum moves by a whole number k of log2 units, so the digit sums
      // rescale exactly by a shift
      if (__any_sync(kFull, mx > m0)) {
        float r = mx;
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) r = fmaxf(r, __shfl_xor_sync(kFull, r, o));
        if (r > m0) {
          if (m0 == -INFINITY) {
            m0 = ceilf(r);
          } else {
            const int k = (int)ceilf(r - m0);
            const float a = k < 126 ? __int_as_float((127 - k) << 23) : 0.f;   // 2^-k
#pragma unroll
            for (int mt = 0; mt < S::kSteps; ++mt) {
              shift_digits(ai[mt][0], ai[mt][1], k);
              shift_digits(ai[mt][2], ai[mt][3], k);
#pragma unroll
              for (int c = 0; c < 4; ++c) acc[mt][c] *= a;
            }
            l0 *= a;
            m0 += (float)k;
          }
        }
      }
      const float mm = m0 == -INFINITY ? 0.f : m0;
      const float p0 = ex2(x0 - mm), p1 = ex2(x1 - mm), p2 = ex2(x2 - mm), p3 = ex2(x3 - mm);
      l0 += (p0 + p1) + (p2 + p3);
      const float rA = d.vs[i] * r15, rB = hasB ? d.vs[i + 1] * r15 : 0.f;
      const uint32_t f0 = __float_as_uint(fmaf(p0, rA, kMagic)), f1 = __float_as_uint(fmaf(p1, rA, kMagic));
      const uint32_t f2 = __float_as_uint(fmaf(p2, rB, kMagic)), f3 = __float_as_uint(fmaf(p3, rB, kMagic));
      // (hi of token gid, hi of token gid + 8 | lo, lo) -> column (head, digit);
      // threads with tig >= 2 swap their two token pairs (see v_rows_t)
      const uint32_t sw = tig >= 2 ? 0x1032u : 0x3210u;
      const uint32_t t0 = movtrans(prmt(f0, f1, 0x4051u)), t1 = movtrans(prmt(f2, f3, 0x4051u));
      const uint32_t b0 = prmt(t0, t0, sw), b1 = prmt(t1, t1, sw);
#pragma unroll
      for (int mt = 0; mt < S::kSteps; ++mt) {
        const int lb = mt + S::kSteps;
        const int blo = 2 * (mt >> 3) + ((mt & 7) >> 2), bhi = 2 * (lb >> 3) + ((lb & 7) >> 2);
        const int f = mt & 3;
        imma16832_su(ai[mt], tern8(TA[blo], f), tern8(TA[bhi], f), tern8(TB[blo], f), tern8(TB[bhi], f), b0, b1);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        sA[c] = nA[c];
        sB[c] = nB[c];
      }
    }
    // sum = gmax * 2^-15 * (256 hi + lo) / 64 (tern8 carries 64 * code)
    const float cf = gmax * (1.f / 2097152.f) * inv_uref;
#pragma unroll
    for (int mt = 0; mt < S::kSteps; ++mt) {
      acc[mt][0] += (float)(ai[mt][0] * 256 + ai[mt][1]) * cf;
      acc[mt][2] += (float)(ai[mt][2] * 256 + ai[mt][3]) * cf;
    }
  }

  // A full entry of 8 ternary pages (the ring's capacity at head_dim 64 and
  // 128): the scores of all 8 pages first, one test of the running maximum
  // for the whole entry, then the four page pairs' P.V as one straight run
  // of code, so the loads, transposes and MMAs of one pair overlap the
  // softmax of the next.  P's digits are taken relative to the entry's own
  // maximum (process_ternary_int: relative to the running maximum).
  __device__ __forceinline__ void process_ternary_int8(const unsigned char* e, const Desc& d) {
    constexpr int GB = HPC * group_bytes(KVC_FMT_TERNARY2, D);   // page stride
    constexpr int NT = kBB < 4 ? 4 : kBB;
    e += wi * group_bytes(KVC_FMT_TERNARY2, D);
    const float gmax = d.gvmax;
    if (uref == 0.f && gmax > 0.f) {
      uref = gmax;
      inv_uref = 1.f / gmax;
    }
    const float r15 = gmax > 0.f ? 32768.f / gmax : 0.f;
    constexpr float kMagic = 12582912.f;
    float x[8][2];
#pragma unroll
    for (int pg = 0; pg < 8; ++pg) {
      float s[4];
      qk_ternary(e + pg * GB, s);
      const float sc = d.ks[pg] * kq0;
      x[pg][0] = s[0] * sc;
      x[pg][1] = s[2] * sc;
    }
    // only the entry's last page can be partial
    if (gid >= d.nrows) x[7][0] = -INFINITY;
    if (gid + 8 >= d.nrows) x[7][1] = -INFINITY;
    // the first pair's V rows, loaded before the maximum test so that their
    // latency overlaps it
    uint32_t ra[4][kVW4], rb[4][kVW4];
    v_rows_ld(e + S::kHalf, ra);
    v_rows_ld(e + S::kHalf + GB, rb);
    float mx = x[0][0];
#pragma unroll
    for (int pg = 0; pg < 8; ++pg) mx = fmaxf(mx, fmaxf(x[pg][0], x[pg][1]));
    int ai[S::kSteps][4];
#pragma unroll
    for (int mt = 0; mt < S::kSteps; ++mt)
#pragma unroll
      for (int c = 0; c < 4; ++c) ai[mt][c] = 0;
    if (__any_sync(kFull, mx > m0)) {
      float r = mx;
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) r = fmaxf(r, __shfl_xor_sync(kFull, r, o));
      if (r > m0) {
        if (m0 == -INFINITY) {
          m0 = ceilf(r);
        } else {
          const int k = (int)ceilf(r - m0);
          const float a = k < 126 ? __int_as_float((127 - k) << 23) : 0.f;   // 2^-k
#pragma unroll
          for (int mt = 0; mt < S::kSteps; ++mt)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[mt][c] *= a;
          l0 *= a;
          m0 += (float)k;
        }
      }
    }
    // P's digits are taken relative to this entry's own maximum per head, so
    // every entry keeps 15 bits of its largest P whatever the running
    // maximum; sblk = 2^(entry maximum - m0) <= 1 scales the entry into the
    // running state (the normaliser and the fold)
    float rh = mx;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) rh = fmaxf(rh, __shfl_xor_sync(kFull, rh, o));
    const float mm = rh == -INFINITY ? 0.f : rh;
    const float sblk = (rh == -INFINITY || m0 == -INFINITY) ? 0.f : ex2(rh - m0);
    const uint32_t sw = tig >= 2 ? 0x1032u : 0x3210u;
#pragma unroll
    for (int pr2 = 0; pr2 < 4; ++pr2) {
      const int i = 2 * pr2;
      uint32_t TA[NT], TB[NT];
      if (pr2 == 0) {
        v_rows_tr(ra, TA);
        v_rows_tr(rb, TB);
      } else {
        v_rows_t(e + S::kHalf + i * GB, TA);
        v_rows_t(e + S::kHalf + (i + 1) * GB, TB);
      }
      const float p0 = ex2(x[i][0] - mm), p1 = ex2(x[i][1] - mm);
      const float p2 = ex2(x[i + 1][0] - mm), p3 = ex2(x[i + 1][1] - mm);
      l0 += ((p0 + p1) + (p2 + p3)) * sblk;
      const float rA = d.vs[i] * r15, rB = d.vs[i + 1] * r15;
      const uint32_t f0 = __float_as_uint(fmaf(p0, rA, kMagic)), f1 = __float_as_uint(fmaf(p1, rA, kMagic));
      const uint32_t f2 = __float_as_uint(fmaf(p2, rB, kMagic)), f3 = __float_as_uint(fmaf(p3, rB, kMagic));
      const uint32_t t0 = movtrans(prmt(f0, f1, 0x4051u)), t1 = movtrans(prmt(f2, f3, 0x4051u));
      const uint32_t b0 = prmt(t0, t0, sw), b1 = prmt(t1, t1, sw);
#pragma unroll
      for (int mt = 0; mt < S::kSteps; ++mt) {
        const int lb = mt + S::kSteps;
        const int blo = 2 * (mt >> 3) + ((mt & 7) >> 2), bhi = 2 * (lb >> 3) + ((lb & 7) >> 2);
        const int f = mt & 3;
        imma16832_su(ai[mt], tern8(TA[blo], f), tern8(TA[bhi], f), tern8(TB[blo], f), tern8(TB[bhi], f), b0, b1);
      }
    }
    const float cf = gmax * (1.f / 2097152.f) * inv_uref * sblk;
#pragma unroll
    for (int mt = 0; mt < S::kSteps; ++mt) {
      acc[mt][0] += (float)(ai[mt][0] * 256 + ai[mt][1]) * cf;
      acc[mt][2] += (float)(ai[mt][2] * 256 + ai[mt][3]) * cf;
    }
  }

  // --------------------------------------------------- softmax, per page
  // Scales the score tile, applies the row mask, moves the lazy maximum when
  // needed, accumulates the row sums and returns P^T fragments (P scaled by
  // the page's V scale relative to the warp's reference scale).
  // With SPLIT, P is passed as an f16 hi + lo pair (b0/b1 and lo0/lo1,
  // ~22 bits): pages whose values can be large (FP8, BF16) need it to keep
  // the absolute error of P.V small; ternary values are bounded by gamma.
  // NARROW: one query head (tig) per thread, scores s[0] (token gid) and
  // s[2] (token gid + 8) scaled by sc0; P always goes out as the hi + lo pair
  // in columns (2 * tig, 2 * tig + 1), so SPLIT does not apply.
  // BF: P goes out in bf16 (BF16 pages multiply V as stored) instead of f16.
  template <bool SPLIT, bool BF = false>
  // sc0 / sc1 scale the thread's two score columns (s[0], s[2] and s[1], s[3]).
  __device__ __forceinline__ void softmax_page(float (&s)[4], float sc0, float sc1, float ratio, int nt,
                                               uint32_t& b0, uint32_t& b1, uint32_t& lo0, uint32_t& lo1) {
    if constexpr (NARROW) {
      float mx = fmaxf(s[0], s[2]) * sc0;
      bool masked = false;
      if (nt < kPage) {
        masked = true;
        mx = gid + 8 < nt ? mx : s[0] * sc0;
        if (gid >= nt) mx = -INFINITY;
      }
      if (__any_sync(kFull, mx > m0 + kTau)) {
        float r = mx;
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) r = fmaxf(r, __shfl_xor_sync(kFull, r, o));
        const float n0 = fmaxf(m0, r);
        const float a0 = n0 == -INFINITY ? 1.f : ex2(m0 - n0);
#pragma unroll
        for (int mt = 0; mt < S::kSteps; ++mt)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[mt][c] *= a0;
        l0 *= a0;
        m0 = n0;
      }
      float e0 = fmaf(s[0], sc0, -m0), e1 = fmaf(s[2], sc0, -m0);
      if (masked) {
        if (gid >= nt) e0 = -INFINITY;
        if (gid + 8 >= nt) e1 = -INFINITY;
      }
      const float p0 = ex2(e0), p1 = ex2(e1);
      l0 += p0 + p1;
      if constexpr (BF) {
        b0 = movtrans(split_bf16x2(p0 * ratio));
        b1 = movtrans(split_bf16x2(p1 * ratio));
      } else {
        b0 = movtrans(split_f16x2(p0 * ratio));
        b1 = movtrans(split_f16x2(p1 * ratio));
      }
      return;
    }
    // exponent arguments s*sc - m; the scales are >= 0 (gamma, s or 1, times max|q|)
    float mx0 = fmaxf(s[0], s[2]) * sc0, mx1 = fmaxf(s[1], s[3]) * sc1;
    bool masked = false;
    if (nt < kPage) {
      masked = true;
      const bool r0 = gid < nt, r1 = gid + 8 < nt;
      mx0 = r1 ? mx0 : s[0] * sc0;
      mx1 = r1 ? mx1 : s[1] * sc1;
      if (!r0) mx0 = mx1 = -INFINITY;
    }
    if (__any_sync(kFull, mx0 > m0 + kTau || mx1 > m1 + kTau)) {
      float r0 = mx0, r1 = mx1;
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        r0 = fmaxf(r0, __shfl_xor_sync(kFull, r0, o));
        r1 = fmaxf(r1, __shfl_xor_sync(kFull, r1, o));
      }
      const float n0 = fmaxf(m0, r0), n1 = fmaxf(m1, r1);
      const float a0 = n0 == -INFINITY ? 1.f : ex2(m0 - n0);
      const float a1 = n1 == -INFINITY ? 1.f : ex2(m1 - n1);
#pragma unroll
      for (int mt = 0; mt < S::kSteps; ++mt) {
        acc[mt][0] *= a0; acc[mt][2] *= a0;
        acc[mt][1] *= a1; acc[mt][3] *= a1;
      }
      l0 *= a0;
      l1 *= a1;
      m0 = n0;
      m1 = n1;
    }
    float e00 = fmaf(s[0], sc0, -m0), e01 = fmaf(s[1], sc1, -m1);
    float e10 = fmaf(s[2], sc0, -m0), e11 = fmaf(s[3], sc1, -m1);
    if (masked) {
      if (gid >= nt) e00 = e01 = -INFINITY;
      if (gid + 8 >= nt) e10 = e11 = -INFINITY;
    }
    const float p00 = ex2(e00), p01 = ex2(e01), p10 = ex2(e10), p11 = ex2(e11);
    l0 += p00 + p10;
    l1 += p01 + p11;
    // P scaled by the page's V scale (relative to the reference)
    const float y00 = p00 * ratio, y01 = p01 * ratio, y10 = p10 * ratio, y11 = p11 * ratio;
    if constexpr (BF) {
      const uint32_t h0 = bf16x2(y00, y01), h1 = bf16x2(y10, y11);
      b0 = movtrans(h0);
      b1 = movtrans(h1);
      const float2 g0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h0));
      const float2 g1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h1));
      lo0 = movtrans(bf16x2(y00 - g0.x, y01 - g0.y));
      lo1 = movtrans(bf16x2(y10 - g1.x, y11 - g1.y));
    } else {
      const uint32_t h0 = f16x2(y00, y01), h1 = f16x2(y10, y11);
      b0 = movtrans(h0);
      b1 = movtrans(h1);
      if constexpr (SPLIT) {
        const float2 g0 = __half22float2(*reinterpret_cast<const __half2*>(&h0));
        const float2 g1 = __half22float2(*reinterpret_cast<const __half2*>(&h1));
        lo0 = movtrans(f16x2(y00 - g0.x, y01 - g0.y));
        lo1 = movtrans(f16x2(y10 - g1.x, y11 - g1.y));
      }
    }
  }

  // Re-base the warp's value-scale reference when the entry's V scales
  // (vf * vs[i]) leave [ref/16, 16*ref]: P = p * vs / ref stays well inside
  // the f16 normal range.  Warp-uniform (every lane reads the same desc).
  __device__ __forceinline__ void rebase_value_scale(const Desc& d, float vf) {
    float vmax = 0.f, vmin = INFINITY;
    for (int i = 0; i < d.np; ++i) {
      const float v = d.vs[i] * vf;
      vmax = fmaxf(vmax, v);
      vmin = fminf(vmin, v);
    }
    if (vmax > 0.f && (uref == 0.f || vmax > 16.f * uref || vmin < uref * 0.0625f)) {
      const float beta = uref / vmax;
#pragma unroll
      for (int mt = 0; mt < S::kSteps; ++mt)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[mt][c] *= beta;
      uref = vmax;
      inv_uref = 1.f / vmax;
    }
  }

  // --------------------------------------------------------- one entry
  // e: the ring slot.  Page i of this warp's head starts at
  // e + (i * HPC + wi) * GB (K) and kHalf further (V).  Columns of padded
  // GQA rows (query heads >= G, Q = 0) run along with finite values and are
  // never written out.
  __device__ __forceinline__ void process(const unsigned char* e, const Desc& d) {
    const int fmt = d.fmt, np = d.np;
    uint32_t b0, b1, lo0 = 0u, lo1 = 0u;
    if (NARROW && fmt == KVC_FMT_TERNARY2 && p.tern_int) {
      if (S::kTernCap == 8 && p.tern_int == 2 && d.np == 8) process_ternary_int8(e, d);
      else process_ternary_int(e, d);
    } else if (fmt == KVC_FMT_TERNARY2) {
      constexpr int GB = HPC * group_bytes(KVC_FMT_TERNARY2, D);   // page stride
      e += wi * group_bytes(KVC_FMT_TERNARY2, D);
      rebase_value_scale(d, 0.5f);
      const float vf = 0.5f * inv_uref;
      // software pipeline: the scores of page i+1 are computed while page i
      // goes through the softmax and P.V (independent instruction streams);
      // only the entry's last page can be partial
      float s[4];
      qk_ternary(e, s);
      int i = 0;
      for (; i + 1 < np; ++i) {
        float sn[4];
        qk_ternary(e + (i + 1) * GB, sn);
        softmax_page<false>(s, d.ks[i] * kq0, d.ks[i] * kq1, d.vs[i] * vf, kPage, b0, b1, lo0, lo1);
        pv_ternary(e + S::kHalf + i * GB, b0, b1, kPage);
#pragma unroll
        for (int c = 0; c < 4; ++c) s[c] = sn[c];
      }
      softmax_page<false>(s, d.ks[i] * kq0, d.ks[i] * kq1, d.vs[i] * vf, d.nrows, b0, b1, lo0, lo1);
      pv_ternary(e + S::kHalf + i * GB, b0, b1, d.nrows);
    } else if (fmt == KVC_FMT_FP8_E4M3) {
      constexpr int GB = HPC * group_bytes(KVC_FMT_FP8_E4M3, D);
      e += wi * group_bytes(KVC_FMT_FP8_E4M3, D);
      rebase_value_scale(d, 1.f);
      if (!q_f16 && lane == 0) atomicOr(p.err, kErrRange);
      for (int i = 0; i < np; ++i) {
        const int nt = i == np - 1 ? d.nrows : kPage;
        float s[4];
        qk_fp8(e + i * GB, s);
        const float sc = d.ks[i] * p.scale_log2;
        softmax_page<true>(s, sc, sc, d.vs[i] * inv_uref, nt, b0, b1, lo0, lo1);
        pv_fp8(e + S::kHalf + i * GB, b0, b1, lo0, lo1, nt);
      }
    } else if (fmt == KVC_FMT_BF16) {
      rebase_value_scale(d, 1.f);
      e += wi * S::kBf16Rows * 2 * D;        // full page, or the 8 rows of a half page
      float s[4];
      if constexpr (S::kBf16Rows == 16) {
        qk_bf16<16>(e, s);
        softmax_page<true, true>(s, p.scale_log2, p.scale_log2, inv_uref, d.nrows, b0, b1, lo0, lo1);
        pv_bf16<16>(e + S::kHalf, b0, b1, lo0, lo1, d.nrows);
      } else {
        qk_bf16<8>(e, s);
        softmax_page<true, true>(s, p.scale_log2, p.scale_log2, inv_uref, d.nrows, b0, b1, lo0, lo1);
        pv_bf16<8>(e + S::kHalf, b0, b1, lo0, lo1, d.nrows);
      }
    }
  }

  // ------------------------------------------------------------- main
  __device__ __forceinline__ bool consume(int slot, uint32_t parity) {
    if (!mbar_wait(&bars[slot], parity, wait_limit)) return false;
    const Desc& d = desc[slot];
    const int bg = d.bg;
    if (bg != cur_bg) {
      finish();
      begin(bg);
    }
    if (d.fmt != kSkip) process(ring + slot * S::kSlotBytes, d);
    __syncwarp();
    return true;
  }

  // This warp is done reading ring slot `slot`.  True for the last of the
  // CTA's warps to get here, which then refills the slot (no warp waits for
  // another: the refill happens after every warp's reads of the slot).
  __device__ __forceinline__ bool release(int slot) {
    if constexpr (HPC == 1) {
      return true;
    } else {
      unsigned last = 0;
      // the warp's reads of the slot have completed (their values are in
      // registers and __syncwarp ordered them before this point)
      if (lane == 0) {
        last = atomicAdd(&cnt[slot], 1) == HPC - 1;
        if (last) cnt[slot] = 0;
      }
      return __shfl_sync(kFull, last, 0) != 0u;
    }
  }

  __device__ void run(int w_index) {
    lane = threadIdx.x & 31;
    gid = lane >> 2;
    tig = lane & 3;
    W = w_index;
    const long long c0 = (long long)W * pr.C / pr.nwg, c1 = (long long)(W + 1) * pr.C / pr.nwg;
    cursor = pr.unit_of_cost(c0);
    u1 = pr.unit_of_cost(c1);
    cb = cursor;
    bf16_half = 0;
    cur_bg = -1;
    {
      MetaA a;
      meta_phase_a(p, pr, cb, u1, lane, HPC, wi, a);
      meta_phase_b(p, a, cur);
    }
    meta_phase_a(p, pr, cb + 32, u1, lane, HPC, wi, nxa);
    nxt_b_pending = true;
    nxa_pending = false;

    // Failure-detection test mode: slot 0's first phase waits for 16 bytes
    // that no copy delivers, so every wait on it runs out (after a few short
    // tries) and the launch ends with the timeout flag.
    wait_limit = p.test_timeout ? 4u : kSpinLimit;
    if (p.test_timeout && wi == 0 && lane == 0) mbar_expect_tx(&bars[0], 16u);
    // warp 0 fills both slots first; later refills come from release()
    bool v0 = issue(0, wi == 0), v1 = issue(1, wi == 0);
    bool ok = true;
    for (int it = 0;; ++it) {          // one call site: the hot loop stays compact
      const int slot = it & 1;
      if (!(slot ? v1 : v0)) break;
      if (!(ok = consume(slot, (uint32_t)(it >> 1) & 1u))) break;
      const bool nv = issue(slot, release(slot));
      if (slot) v1 = nv; else v0 = nv;
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.err, kErrTimeout);
      // let copies still in flight land before the CTA's memory is released
      mbar_wait(&bars[0], 0u, wait_limit), mbar_wait(&bars[0], 1u, wait_limit);
      mbar_wait(&bars[1], 0u, wait_limit), mbar_wait(&bars[1], 1u, wait_limit);
      return;
    }
    finish();
  }
};

template <int D, int HPC, bool NARROW>
__global__ void __launch_bounds__(HPC * 32) decode_tc_kernel(DecodeParams p) {
  using S = Shape<D, HPC>;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* ring = smem;
  uint32_t* qbuf = reinterpret_cast<uint32_t*>(smem + kEntries * S::kSlotBytes);
  Desc* descs = reinterpret_cast<Desc*>(smem + kEntries * S::kSlotBytes + HPC * S::kQBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(descs + HPC * kEntries);
  int* cnt = reinterpret_cast<int*>(bars + kEntries);
  int* seqP = cnt + kEntries;
  int* seqC = seqP + (p.B + 1);
  int* seqL = seqC + (p.B + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int whp = cost_hp<D, NARROW>(p.hp);
  const int nq = p.Hkv / HPC;          // head groups per sequence

  if (threadIdx.x < kEntries) {
    mbar_init(&bars[threadIdx.x], 1);
    cnt[threadIdx.x] = 0;
  }
  if (warp == 0) {
    int carry_u = 0, carry_c = 0;
    for (int base = 0; base < p.B; base += 32) {
      const int b = base + lane;
      int u = 0, c = 0;
      if (b < p.B) {
        const int gb = p.b_base + b;               // virtual sequence of the whole batch
        int L = p.ctx[gb < p.Bseq ? gb : gb % p.Bseq];
        if (L < 0 || L > p.max_pages * kPage) {
          if (blockIdx.x == 0) atomicOr(p.err, kErrContext);
          L = 0;
        }
        seqL[b] = L;
        const SeqShape s = seq_shape(L, p.sink, p.window, whp, kCostTern);
        u = s.np * nq;
        c = s.cost * nq;
      }
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int tu = __shfl_up_sync(kFull, u, o), tc = __shfl_up_sync(kFull, c, o);
        if (lane >= o) { u += tu; c += tc; }
      }
      if (b < p.B) {
        seqP[b + 1] = carry_u + u;
        seqC[b + 1] = carry_c + c;
      }
      carry_u += __shfl_sync(kFull, u, 31);
      carry_c += __shfl_sync(kFull, c, 31);
    }
    if (lane == 0) seqP[0] = seqC[0] = 0;
  }
  fence_mbar_init();
  __syncthreads();
  // sequences with nothing to attend to get a zero row
  for (int b = blockIdx.x; b < p.B; b += gridDim.x)
    if (seqL[b] == 0)
      for (int i = threadIdx.x; i < p.Hq * D; i += blockDim.x) p.out[(long long)b * p.Hq * D + i] = 0.f;

  Prologue pr;
  pr.seqP = seqP;
  pr.seqC = seqC;
  pr.seqL = seqL;
  pr.B = p.B;
  pr.Hkv = p.Hkv;
  pr.sink = p.sink;
  pr.window = p.window;
  pr.whp = whp;
  pr.wt = kCostTern;
  pr.C = seqC[p.B];
  pr.U = seqP[p.B];
  if (pr.U == 0) return;
  // every worker's weight range is at least twice the heaviest unit, so
  // each one owns at least one unit
  const long long most = pr.C / (2 * kCostMax);
  pr.nwg = (int)((long long)gridDim.x < most ? gridDim.x : (most > 0 ? most : 1));
  const int W = blockIdx.x;
  if (W >= pr.nwg) return;
  Worker<D, HPC, NARROW> wk(p, pr, ring, qbuf + warp * (S::kQBytes / 4), descs + warp * kEntries, bars, warp);
  wk.set_counts(cnt);
  wk.run(W);
}

template <int D, int HPC>
size_t tc_smem_bytes(int batch) {
  using S = Shape<D, HPC>;
  return (size_t)kEntries * S::kSlotBytes + (size_t)HPC * S::kQBytes + HPC * kEntries * sizeof(Desc) +
         kEntries * sizeof(uint64_t) + kEntries * sizeof(int) + (size_t)(3 * batch + 2) * sizeof(int);
}

// The kernel's shared memory depends on the batch (the sequence tables); the
// largest size is opted into once per device, and CTAs per SM are cached per
// (device, head_dim, heads per CTA, batch) so a call costs no runtime query
// after the first.
constexpr int kMaxDev = 64;
template <int D, int HPC, bool NARROW>
cudaError_t tc_occupancy(int batch, int* ctas_per_sm) {
  static std::mutex mu;
  static bool opted[kMaxDev] = {};
  static std::map<std::pair<int, int>, int> cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(dev, batch);
  const auto it = cache.find(key);
  if (it != cache.end()) {
    *ctas_per_sm = it->second;
    return cudaSuccess;
  }
  if (dev >= 0 && dev < kMaxDev && !opted[dev]) {
    e = cudaFuncSetAttribute(decode_tc_kernel<D, HPC, NARROW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tc_smem_bytes<D, HPC>(kTcMaxBatchTpl));
    if (e != cudaSuccess) return e;
    opted[dev] = true;
  }
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, decode_tc_kernel<D, HPC, NARROW>, HPC * 32,
                                                    tc_smem_bytes<D, HPC>(batch));
  if (e == cudaSuccess) cache[key] = *ctas_per_sm;
  return e;
}

template <int D, bool NARROW>
cudaError_t tc_occupancy_hpc(int hpc, int batch, int* ctas_per_sm) {
  switch (hpc) {
    case 1: return tc_occupancy<D, 1, NARROW>(batch, ctas_per_sm);
    case 2: return tc_occupancy<D, 2, NARROW>(batch, ctas_per_sm);
    case 4: return tc_occupancy<D, 4, NARROW>(batch, ctas_per_sm);
    default: return cudaErrorInvalidValue;
  }
}

template <int D, bool NARROW>
void launch_tc(const DecodeParams& p, int hpc, int grid, cudaStream_t s) {
  switch (hpc) {
    case 1: decode_tc_kernel<D, 1, NARROW><<<grid, 32, tc_smem_bytes<D, 1>(p.B), s>>>(p); break;
    case 2: decode_tc_kernel<D, 2, NARROW><<<grid, 64, tc_smem_bytes<D, 2>(p.B), s>>>(p); break;
    default: decode_tc_kernel<D, 4, NARROW><<<grid, 128, tc_smem_bytes<D, 4>(p.B), s>>>(p); break;
  }
}

}  // namespace

// Virtual sequences per launch: each CTA keeps the launch's sequence tables
// in shared memory, so a launch takes at most kTcMaxBatchTpl of them (and
// few enough that the launch's total page weight fits 31 bits); a larger
// batch is decoded in consecutive launches of that many.
int tc_chunk(int hkv, int max_pages) {
  const long long per = (long long)hkv * std::max(1, max_pages) * kCostMax;
  const long long fit = ((1ll << 31) - 1) / per;
  return (int)std::min<long long>(kTcMaxBatchTpl, fit);
}

// KV heads per CTA: the largest of 4, 2, 1 that divides Hkv.
int tc_heads_per_cta(int hkv) { return hkv % 4 == 0 ? 4 : (hkv % 2 == 0 ? 2 : 1); }

cudaError_t tc_grid(int batch, int d, int hq, int hkv, int* grid) {
  int dev = 0, sms = 0, per = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int hpc = tc_heads_per_cta(hkv);
  const bool narrow = hq / hkv <= 4;
  switch (d) {
    case 64: e = narrow ? tc_occupancy_hpc<64, true>(hpc, batch, &per) : tc_occupancy_hpc<64, false>(hpc, batch, &per); break;
    case 128: e = narrow ? tc_occupancy_hpc<128, true>(hpc, batch, &per) : tc_occupancy_hpc<128, false>(hpc, batch, &per); break;
    case 256: e = narrow ? tc_occupancy_hpc<256, true>(hpc, batch, &per) : tc_occupancy_hpc<256, false>(hpc, batch, &per); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  *grid = sms * (per > 0 ? per : 1);
  return cudaSuccess;
}

int tc_warps_per_cta(int hkv) { return tc_heads_per_cta(hkv); }

cudaError_t launch_decode_tc(const DecodeParams& p, int head_dim, int grid, int chunk, cudaStream_t s) {
  const int hpc = tc_heads_per_cta(p.Hkv);
  const bool narrow = p.G <= 4;
  if (chunk < 1) return cudaErrorInvalidValue;
  // consecutive launches of `chunk` virtual sequences; each launch owns its
  // rows of Q, the output and the tickets, and reuses the partial records
  // (the launches run one after another on the stream)
  for (int b0 = 0; b0 < p.B; b0 += chunk) {
    DecodeParams c = p;
    c.b_base = p.b_base + b0;
    c.B = std::min(chunk, p.B - b0);
    c.q = p.q + (long long)b0 * p.Hq * head_dim;
    c.out = p.out + (long long)b0 * p.Hq * head_dim;
    c.tickets = p.tickets + (long long)b0 * p.Hkv;
    switch (head_dim) {
      case 64: narrow ? launch_tc<64, true>(c, hpc, grid, s) : launch_tc<64, false>(c, hpc, grid, s); break;
      case 128: narrow ? launch_tc<128, true>(c, hpc, grid, s) : launch_tc<128, false>(c, hpc, grid, s); break;
      case 256: narrow ? launch_tc<256, true>(c, hpc, grid, s) : launch_tc<256, false>(c, hpc, grid, s); break;
      default: return cudaErrorInvalidValue;
    }
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace kvc
