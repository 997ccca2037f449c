// Mixed-format paged decode attention with the 5th-generation tensor cores
// (tcgen05, accumulators in tensor memory) for the ternary pages (sm_100a).
//
// Method: "Minima-KV" (twodots.gr), section "How mixed-format attention
// works" - every page is read directly in its own format as it is loaded,
// each split emits a partial state (max score, sum of exponentials, output)
// and one online-softmax normalisation merges them.  Ternary pages follow
// "Show HN: Vantage-V-AI" (newshot.cc), section "Core architecture" (codes
// {-1, 0, +1}, gamma = mean|X|, 4 codes per byte).
//
// Design (one CTA = one warpgroup of 128 threads, persistent, stream-K):
// * Work: the (sequence, KV-head group, page) units of the batch are split
//   over the CTAs of a persistent grid by weight; a CTA walks its range in
//   entries of up to 8 pages of one (sequence, head group), staged through a
//   2-slot shared-memory ring by 1-D bulk copies (cp.async.bulk, no
//   multicast).
// * Ternary entries, per KV head of the group (a "head block" of up to 128
//   tokens):
//   - Q.K^T on tcgen05 (kind::i8, M = 128 tokens): thread t unpacks the
//     codes of token t into int8 (+-64, one shift and one AND per four
//     codes) and stores its row into tensor memory (A operand); Q is held in
//     shared memory as three signed base-128 digits per element (~22 bits
//     of max|q|), one MMA column per (query head, digit).  Int32 results.
//   - softmax per token thread: the digit columns are recombined in fp32,
//     scaled by gamma_K, exponentiated against a lazy running maximum (it
//     moves only when a score exceeds it by 2^8), and P * gamma_V / ref is
//     written as a 31-bit unsigned integer: its four bytes are the B operand
//     columns of P.V (one column per (query head, byte)).
//   - P.V on tcgen05 (kind::i8, M = 128 output dims, A = V^T read
//     MN-major from shared memory where thread t stored token t's unpacked
//     codes, B = the P bytes): int32 accumulators stay in tensor memory
//     across head blocks and are folded into fp32 registers (thread = output
//     dim) only when the maximum or the value reference changes, before the
//     int32 range could be exceeded, and at the end.
//   Double-buffered operands let the unpack of head h+1 overlap the
//   Q.K^T of head h and the P.V of head h-1.
// * BF16 / FP8 entries (sink and window pages, anchors): warp h of the CTA
//   handles KV head h with register-sourced mma.sync tiles (the pages' bytes
//   per token are 8-16x those of ternary pages, so their math is cheap per
//   byte) and keeps its own partial state.
// * Each CTA writes two partial records per (sequence, KV head) it touched
//   (ternary and high precision); the last writer (atomic ticket, no
//   waiting) merges all records of the pair.
#include "decode_common.cuh"

#include <map>
#include <mutex>
#include <utility>

namespace kvc {
namespace {

using namespace dec;

constexpr int kUmmaMaxBatch = 512;   // largest batch (per-CTA sequence tables in shared memory)
// Three warpgroups: two of compute warps, one of service warps (the MMA warp
// of each compute warpgroup, two spare).  The register file is split in four
// 16K partitions, one per scheduler, so 12 warps launch at 168 registers per
// thread.  setmaxnreg then moves registers between warpgroups, but only
// within what the CTA was launched with (384 x 168): the service warpgroup
// drops to 40 and the compute warpgroups rise to 232, which adds up exactly
// (a larger sum would leave setmaxnreg.inc waiting forever).
constexpr int kUmmaThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr int kComputeRegs = 232, kServiceRegs = 40;
static_assert(2 * 128 * kComputeRegs + 128 * kServiceRegs <= kUmmaThreads * kLaunchRegs,
              "register split exceeds the CTA's launch allocation");
static_assert(kComputeRegs % 8 == 0 && kServiceRegs % 8 == 0 && kServiceRegs >= 24, "setmaxnreg counts");
constexpr int kEntries = 2;          // ring slots
constexpr float kTauHp = 8.0f;       // lazy-max threshold of the high-precision path, log2 units
constexpr float kTau = 8.0f;         // ... of the ternary path: P <= 2^8
constexpr float kRatioMax = 4.0f;    // gamma_V / reference <= 4 before a re-base
constexpr float kXScale = 2097152.0f;  // 2^21: P * ratio * 2^21 <= 2^(8 + 2 + 21) fits 31 bits
constexpr float kQMax = 2088000.0f;  // |q| in digit units: three base-128 digits, top digit in [-128, 127]
constexpr int kFlushTokens = 65536;  // int32 P.V accumulators are folded at least this often
// Partition weights in units of one ternary page of one KV head (measured
// relative cost; a high-precision page also moves 8-16x the bytes).
constexpr int kCostTern = 2, kCostMax = 24;
template <int D, bool NARROW>
__host__ __device__ constexpr int ucost_hp(int fmt) {
  return fmt == KVC_FMT_BF16 ? (NARROW ? 16 : 22) : (NARROW ? 9 : 16);
}

__host__ __device__ constexpr int pow2_cols(int c) { return c <= 32 ? 32 : (c <= 64 ? 64 : (c <= 128 ? 128 : (c <= 256 ? 256 : 512))); }

template <int D, int HPC, bool NARROW>
struct UShape {
  static_assert(D == 64 || D == 128, "tensor-memory path: head_dim 64 or 128");
  static constexpr int kHeadHalf = 32 * D;                 // K (or V) bytes of one head per slot
  static constexpr int kSlotBytes = 2 * HPC * kHeadHalf;   // one ring slot: K region | V region
  static constexpr int kHalf = HPC * kHeadHalf;
  static constexpr int kTernCap = kHeadHalf / (4 * D);     // 8 ternary pages (128 tokens)
  static constexpr int kFp8Cap = kHeadHalf / (16 * D);     // 2 FP8 pages
  // high-precision path (mma.sync)
  static constexpr int kSteps = D / 16;                    // k-steps of Q.K^T = m-tiles of P.V
  static constexpr int kWPT = D / 64;
  static constexpr int kUPT = D / 64;
  // tensor-memory path
  static constexpr int kWords = D / 16;                    // 32-bit code words per token row
  static constexpr int kKCols = D / 4;                     // tensor-memory columns of one A_K buffer
  static constexpr int kKSteps = D / 32;                   // Q.K^T MMAs (K = 32 dims each)
  static constexpr int NQ = NARROW ? 16 : 32;              // Q.K^T columns: (query head, digit)
  static constexpr int NP = NARROW ? 16 : 32;              // P.V columns: (query head, byte)
  static constexpr int kGmax = NARROW ? 4 : 8;
  static constexpr int kAV = 128 * 128;                    // A_V buffer: 128 dims (64 used at D = 64) x 128 tokens
  static constexpr int kBP = 128 * NP;                     // B_P buffer: 128 tokens x NP
  static constexpr int kBQ = D * NQ;                       // B_Q of one head
  static constexpr int kColAK = 0, kColDS = 2 * kKCols, kColDO = 2 * kKCols + 2 * NQ;
  static constexpr int kTmemCols = pow2_cols(kColDO + HPC * NP);
  static_assert(kColDO + HPC * NP <= 256, "two CTAs per SM share the 512 tensor-memory columns");
};

// ------------------------------------------------------------- tcgen05 PTX
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
      "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
      "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,"
      "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// Shared-memory matrix descriptor, no swizzle ("interleaved" canonical
// layout): 8 rows of 16 bytes form a core matrix; lbo = byte distance of the
// next core matrix along K, sbo = along M/N.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}
// Instruction descriptor of kind::i8 (int32 accumulators).
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N, bool a_signed, bool b_signed, bool a_mn, bool b_mn) {
  return (2u << 4) | ((a_signed ? 1u : 0u) << 7) | ((b_signed ? 1u : 0u) << 10) | ((a_mn ? 1u : 0u) << 15) |
         ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void umma_i8_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n}"
               ::"r"(d), "r"(a), "l"(bdesc), "r"(idesc), "r"(acc) : "memory");
}
__device__ __forceinline__ void umma_i8_ss(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}"
               ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc) : "memory");
}
// true in exactly one lane of the (converged) warp
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile("{\n .reg .pred p;\n elect.sync _|p, 0xffffffff;\n selp.u32 %0, 1, 0, p;\n}" : "=r"(pred));
  return pred != 0;
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Commands from the compute warps of a warpgroup to its MMA warp: a ring of
// kCmdSlots entries, each with an mbarrier that all 128 compute threads
// arrive on once their operand writes are complete and fenced.
constexpr int kCmdSlots = 4;
constexpr int kCmdQK = 1, kCmdPV = 2, kCmdStop = 3;
struct Cmd {
  int type, h, j, nks_acc;   // nks_acc: P.V k-steps | accumulate << 8
};
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Position of dim d inside the MMA's K (Q.K^T) or M (P.V) axis: tern8 on the
// code word of dims 16j..16j+15 with field f yields dims 16j + 4b + f in byte
// b, which lands at index 16j + 4f + b.  The map is its own inverse.
__host__ __device__ constexpr int dim_perm(int d) { return (d & ~15) | ((d & 3) << 2) | ((d >> 2) & 3); }

// 32-bit float from three int32 digit columns: c0 + 128 c1 + 16384 c2.
__device__ __forceinline__ float digits3(uint32_t c0, uint32_t c1, uint32_t c2) {
  return fmaf((float)(int)c2, 16384.f, fmaf((float)(int)c1, 128.f, (float)(int)c0));
}
// ... from four byte columns: c0 + 2^8 c1 + 2^16 c2 + 2^24 c3.
__device__ __forceinline__ float bytes4(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3) {
  return fmaf((float)(int)c3, 16777216.f, fmaf((float)(int)c2, 65536.f, fmaf((float)(int)c1, 256.f, (float)(int)c0)));
}

// ----------------------------------------------------------- the worker
// NARROW (GQA group of at most 4 query heads): in the high-precision path
// MMA column 2h + part belongs to query head h, part 0/1 = P's f16 hi/lo.
template <int D, int HPC, bool NARROW>
struct UWorker {
  using S = UShape<D, HPC, NARROW>;
  const DecodeParams& p;
  const Prologue& pr;
  // shared memory
  unsigned char* ring;     // [kEntries] slots
  unsigned char* av;       // [2] A_V buffers
  unsigned char* bp;       // [2] B_P buffers
  unsigned char* bq;       // [HPC] B_Q
  Desc* descs;             // [HPC][kEntries]
  uint64_t* bars;          // [kEntries] slot barriers, then [2] Q.K^T, then [2] P.V
  float* mq;               // [HPC][8] running maximum (log2 units) of the ternary path
  float* cq;               // [HPC][8] score scale: digit scale * softmax scale * log2(e) / 64
  float* red;              // [4 warps][8] reduction scratch
  int* flags;              // [2..3]: ring slot holds an entry
  Cmd* cmds;               // [kCmdSlots] commands to the MMA warp
  uint64_t* cbars;         // [kCmdSlots] their barriers (128 arrivals)
  int ncmd;                // commands posted
  uint32_t tmem;           // tensor-memory base
  int tid, warp, lane, gid, tig;   // tid / warp: within the warpgroup
  int bar_id;              // named barrier of the warpgroup
  int W;
  int cur_bq;
  int jc;                  // head blocks of finished entries (buffer and barrier phase counter)
  int nqk, npv;            // Q.K^T and P.V MMA groups issued
  uint32_t fail;           // a bounded wait gave up
  // ternary path state of each KV head of the group; the head loop is not
  // unrolled (the hot loop stays small), so the registers of head h are
  // reached through with_head(h, f), a switch over the constant indices
  struct HeadState {
    float o[S::kGmax];   // thread = output row (dim perm): folded P.V
    float l[S::kGmax];   // thread = token: partial sums of P
    float uref;          // value reference (0: unset)
    int tok;             // tokens accumulated since the last fold
  };
  HeadState hs[HPC];
  uint32_t empty_mask;          // bit h: the P.V accumulators of head h hold nothing
  // metadata walk (warps < HPC)
  int u1, cursor, cb;
  Meta cur, nxt;
  MetaA nxa;
  bool nxt_b_pending, nxa_pending;
  // high-precision path state (warp h = KV head h)
  uint32_t qf[2 * S::kSteps];   // bf16 Q B-fragments (Q as given)
  bool q_f16;                   // Q of the group fits the f16 range (FP8 pages use f16 products)
  float acc[S::kSteps][4];
  float m0, m1, l0, l1, huref, inv_huref;
  int hp_used;

  __device__ UWorker(const DecodeParams& pp, const Prologue& prr) : p(pp), pr(prr) {}

  template <typename F>
  __device__ __forceinline__ void with_head(int h, F&& f) {
    if constexpr (HPC == 1) {
      f(hs[0]);
    } else if constexpr (HPC == 2) {
      if (h == 0) f(hs[0]); else f(hs[1]);
    } else {
      switch (h) {
        case 0: f(hs[0]); break;
        case 1: f(hs[1]); break;
        case 2: f(hs[2]); break;
        default: f(hs[3]); break;
      }
    }
  }

  // barriers of this warpgroup only (the CTA holds two independent ones)
  __device__ __forceinline__ void wg_sync() { asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory"); }
  __device__ __forceinline__ int wg_sync_or(int pred) {
    int r;
    asm volatile("{\n .reg .pred p, q;\n setp.ne.b32 p, %1, 0;\n bar.red.or.pred q, %2, 128, p;\n selp.s32 %0, 1, 0, q;\n}"
                 : "=r"(r) : "r"(pred), "r"(bar_id) : "memory");
    return r;
  }

  __device__ __forceinline__ int shfl(int v, int src) { return __shfl_sync(kFull, v, src); }
  __device__ __forceinline__ Desc& desc_of(int h, int slot) { return descs[h * kEntries + slot]; }
  __device__ __forceinline__ uint32_t tmem_row(int col) const { return tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)col; }
  __device__ __forceinline__ bool wait_bar(uint64_t* b, uint32_t parity) {
    const bool ok = mbar_wait(b, parity);
    if (!ok) fail = 1u;
    return ok;
  }

  // ------------------------------------------------------ staging (warps < HPC)
  // Describe the next entry of the CTA's unit range in desc_of(warp, slot);
  // every warp < HPC forms the same entries; warp 0 also fills the slot.
  __device__ bool issue(int slot, bool copy) {
    const int wi = warp;
    if (cursor >= u1) return false;
    int li = cursor - cb;
    if (li >= 32) {
      if (nxt_b_pending) meta_phase_b(p, nxa, nxt);
      cur = nxt;
      cb += 32;
      li -= 32;
      nxt_b_pending = false;
      nxa_pending = true;
    }
    const int m0l = shfl(cur.m, li);
    const int f0 = meta_fmt(m0l), bq0 = meta_bg(m0l), bg0 = bq0 * HPC + wi;
    int np = 1, nrows, bytes_per_page = 0;
    if (f0 != kSkip) {
      const int cap = f0 == KVC_FMT_TERNARY2 ? S::kTernCap : (f0 == KVC_FMT_FP8_E4M3 ? S::kFp8Cap : 1);
      const bool ok = lane >= li && (cb + lane) < u1 && cur.m >= 0 && ((cur.m ^ m0l) & ~(31 << 2)) == 0;
      const uint32_t run = __ballot_sync(kFull, ok) >> li;
      const int len = (run == 0xffffffffu) ? 32 : __ffs(~run) - 1;
      np = min(len, cap);
      bytes_per_page = group_bytes(f0, D);
    }
    nrows = meta_ntok(shfl(cur.m, min(li + np - 1, 31)));
    Desc& d = desc_of(wi, slot);
    if (lane == li) {
      d.fmt = f0;
      d.np = np;
      d.bg = bg0;
      d.bq = bq0;
      d.nrows = nrows;
      d.row0 = 0;
    }
    const int k = lane - li;
    float vmax = 0.f;
    if (k >= 0 && k < np) {
      d.ks[k] = cur.ks;
      d.vs[k] = cur.vs;
      vmax = cur.vs;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(kFull, vmax, o));
    if (lane == li) d.gvmax = vmax;
    __syncwarp();
    if (copy) {
      // the HPC heads' groups of a page are contiguous: one copy per page
      // for K and one for V
      const int per = HPC * bytes_per_page;
      const int ncopy = f0 == kSkip ? 0 : np;
      if (lane == 0) mbar_arrive_expect_tx(&bars[slot], (uint32_t)(2 * ncopy * per));
      __syncwarp();
      const int grp = shfl(cur.grp, min(li + lane, 31)) - wi;       // group of head 0 of the CTA
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
        const long long off = (long long)grp * bytes_per_page;
        unsigned char* e = ring + slot * S::kSlotBytes + lane * per;
        bulk_g2s(e, kb + off, (uint32_t)per, &bars[slot]);
        bulk_g2s(e + S::kHalf, vb + off, (uint32_t)per, &bars[slot]);
      }
    }
    cursor += np;
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

  // ------------------------------------------- begin / finish of a head group
  __device__ void begin(int bqn) {
    cur_bq = bqn;
    const int b = bqn / (p.Hkv / HPC), q = bqn - b * (p.Hkv / HPC);
    // ternary path: Q digits of every head of the group in B_Q (warp h builds
    // head h), score scales, state
    if (warp < HPC) {
      const int g = q * HPC + warp;
      unsigned char* dst = bq + warp * S::kBQ;
      constexpr int DPL = D / 32;                 // dims per lane
      for (int r = 0; r < p.G; ++r) {
        const uint16_t* src = reinterpret_cast<const uint16_t*>(p.q) + ((long long)b * p.Hq + g * p.G + r) * D + lane * DPL;
        float x[DPL];
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) {
          x[i] = __uint_as_float((uint32_t)__ldg(src + i) << 16);
          amax = fmaxf(amax, fabsf(x[i]));
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
        const float inv = amax > 0.f ? kQMax / amax : 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) {
          const int d = lane * DPL + i;
          const int qi = __float2int_rn(x[i] * inv);
          const int d0 = ((qi + 64) & 127) - 64;
          const int q1 = (qi - d0) >> 7;
          const int d1 = ((q1 + 64) & 127) - 64;
          const int d2 = (q1 - d1) >> 7;
          const int kap = dim_perm(d);
          unsigned char* row = dst + 16 * kap;
          const int n0 = 3 * r;
#pragma unroll
          for (int k = 0; k < 3; ++k) {
            const int n = n0 + k;
            row[(n >> 4) * (16 * D) + (n & 15)] = (unsigned char)(k == 0 ? d0 : (k == 1 ? d1 : d2));
          }
        }
        if (lane == 0) {
          cq[warp * 8 + r] = (amax / kQMax) * p.scale_log2 * (1.f / 64.f);
          mq[warp * 8 + r] = -INFINITY;
        }
      }
    }
#pragma unroll
    for (int h = 0; h < HPC; ++h) {
#pragma unroll
      for (int r = 0; r < S::kGmax; ++r) { hs[h].o[r] = 0.f; hs[h].l[r] = 0.f; }
      hs[h].uref = 0.f;
      hs[h].tok = 0;
    }
    empty_mask = (1u << HPC) - 1u;
    // high-precision path (warp h, head h): f16 Q fragments
    if (warp < HPC) {
      const int g = q * HPC + warp;
      const int r = NARROW ? gid >> 1 : gid;   // query head within the group
      uint32_t raw[S::kWPT * 8];
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
      // fragment ri = (Q[dlo], Q[dlo + 8]), dlo = 16 * (ri >> 3) + (ri & 7)
#pragma unroll
      for (int ri = 0; ri < 2 * S::kSteps; ++ri) {
        const int wl = ri >> 3, j = ri & 7;
        const uint32_t wa = raw[8 * wl + (j >> 1)], wb = raw[8 * wl + 4 + (j >> 1)];
        qf[ri] = (NARROW && (gid & 1)) ? 0u : prmt(wa, wb, (j & 1) ? 0x7632u : 0x5410u);
      }
      float qmax = 0.f;
#pragma unroll
      for (int i = 0; i < S::kWPT * 8; ++i)
        qmax = fmaxf(qmax, fmaxf(fabsf(__uint_as_float(raw[i] << 16)), fabsf(__uint_as_float(raw[i] & 0xFFFF0000u))));
      q_f16 = __all_sync(kFull, qmax <= 65504.f);
#pragma unroll
      for (int mt = 0; mt < S::kSteps; ++mt)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[mt][c] = 0.f;
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
      huref = inv_huref = 0.f;
      hp_used = 0;
    }
    fence_proxy_async();      // B_Q is read by the tensor cores
    wg_sync();
  }

  // Fold head h's int32 P.V accumulators into s.o (thread = output row).
  // The caller has made sure every P.V MMA into them has completed.
  __device__ __forceinline__ void fold(int h, HeadState& s) {
    if (empty_mask & (1u << h)) return;
    const float coef = s.uref * (1.f / kXScale) * (1.f / 64.f);
    if constexpr (S::NP == 16) {
      uint32_t c[16];
      tmem_ld16(tmem_row(S::kColDO + h * S::NP), c);
      tc_wait_ld();
#pragma unroll
      for (int r = 0; r < 4; ++r) s.o[r] = fmaf(coef, bytes4(c[4 * r], c[4 * r + 1], c[4 * r + 2], c[4 * r + 3]), s.o[r]);
    } else {
      uint32_t c[32];
      tmem_ld32(tmem_row(S::kColDO + h * S::NP), c);
      tc_wait_ld();
#pragma unroll
      for (int r = 0; r < 8; ++r) s.o[r] = fmaf(coef, bytes4(c[4 * r], c[4 * r + 1], c[4 * r + 2], c[4 * r + 3]), s.o[r]);
    }
    empty_mask |= 1u << h;
    s.tok = 0;
  }

  // Wait until the first n P.V MMA groups have completed (they complete in
  // issue order, so the latest commit suffices).
  __device__ __forceinline__ void wait_pv(int n) {
    if (n > 0) wait_bar(&bars[kEntries + 2 + ((n - 1) & 1)], (uint32_t)((n - 1) >> 1) & 1u);
    tc_fence_after();
  }

  __device__ void finish() {
    if (cur_bq < 0) return;
    const int G = p.G;
    const int rs = G * (D + 2);
    // ternary path: fold, reduce the row sums, write record 0 of each head
    wait_pv(jc);
#pragma unroll
    for (int h = 0; h < HPC; ++h) fold(h, hs[h]);
#pragma unroll
    for (int h = 0; h < HPC; ++h) {
#pragma unroll
      for (int r = 0; r < S::kGmax; ++r) {
        float v = hs[h].l[r];
#pragma unroll
        for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
        if (lane == 0) red[warp * 8 + r] = v;
      }
      wg_sync();
      float* rec = p.partials + (long long)(((W + cur_bq) * 2 + 0) * HPC + h) * rs;
      if (tid < G) {
        const float m = mq[h * 8 + tid];
        rec[tid * (D + 2)] = m;
        rec[tid * (D + 2) + 1] = red[tid] + red[8 + tid] + red[16 + tid] + red[24 + tid];
      }
      if (tid < D) {
        const int d = dim_perm(tid);
#pragma unroll
        for (int r = 0; r < S::kGmax; ++r)
          if (r < G) rec[r * (D + 2) + 2 + d] = hs[h].o[r];
      }
      wg_sync();
    }
    // high-precision path: record 1 of head `warp`
    if (warp < HPC) {
      const int wi = warp;
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        l0 += __shfl_xor_sync(kFull, l0, o);
        l1 += __shfl_xor_sync(kFull, l1, o);
      }
      float* rec = p.partials + (long long)(((W + cur_bq) * 2 + 1) * HPC + wi) * rs;
      if constexpr (NARROW) {
        if (tig < G) {
          float* r = rec + tig * (D + 2);
          if (gid == 0) { r[0] = m0; r[1] = l0; }
#pragma unroll
          for (int mt = 0; mt < S::kSteps; ++mt) {
            const int la = mt, lb = mt + S::kSteps;
            const int da = 8 * (gid * S::kUPT + (la >> 3)) + (la & 7);
            const int db = 8 * (gid * S::kUPT + (lb >> 3)) + (lb & 7);
            r[2 + da] = (acc[mt][0] + acc[mt][1]) * huref;
            r[2 + db] = (acc[mt][2] + acc[mt][3]) * huref;
          }
        }
      } else {
        const int c0 = 2 * tig, c1 = 2 * tig + 1;
        if (gid == 0) {
          if (c0 < G) { rec[c0 * (D + 2)] = m0; rec[c0 * (D + 2) + 1] = l0; }
          if (c1 < G) { rec[c1 * (D + 2)] = m1; rec[c1 * (D + 2) + 1] = l1; }
        }
#pragma unroll
        for (int mt = 0; mt < S::kSteps; ++mt) {
          const int la = mt, lb = mt + S::kSteps;
          const int da = 8 * (gid * S::kUPT + (la >> 3)) + (la & 7);
          const int db = 8 * (gid * S::kUPT + (lb >> 3)) + (lb & 7);
          if (c0 < G) {
            rec[c0 * (D + 2) + 2 + da] = acc[mt][0] * huref;
            rec[c0 * (D + 2) + 2 + db] = acc[mt][2] * huref;
          }
          if (c1 < G) {
            rec[c1 * (D + 2) + 2 + da] = acc[mt][1] * huref;
            rec[c1 * (D + 2) + 2 + db] = acc[mt][3] * huref;
          }
        }
      }
    }
    __threadfence();
    wg_sync();
    // one ticket per (sequence, KV head); the last writer merges
    if (warp < HPC) {
      const int wi = warp;
      const int bg = cur_bq * HPC + wi;
      const int b = bg / p.Hkv, q = (bg - b * p.Hkv) / HPC;
      const int np = (pr.seqL[b] + kPage - 1) / kPage;
      const int x0 = pr.seqP[b] + q * np;
      const int w_first = pr.worker_of(x0), w_last = pr.worker_of(x0 + np - 1);
      unsigned last = 0;
      if (lane == 0) last = atomicAdd(p.tickets + bg, 1u) == (unsigned)(w_last - w_first);
      last = __shfl_sync(kFull, last, 0);
      if (last) {
        __threadfence();
        merge_partials<D>(MergeArgs{p.partials, p.out, p.tickets, p.G, p.Hq, p.Hkv}, bg,
                          (w_first + cur_bq) * 2 * HPC + wi, HPC, 2 * (w_last - w_first + 1), lane);
      }
    }
    if (tid < HPC * 8) mq[tid] = -INFINITY;
    cur_bq = -1;
    wg_sync();
  }

  // ------------------------------------------------------- ternary entries
  // All entry-wide barriers: stores to tensor memory finished, shared-memory
  // operands visible to the tensor cores, then every thread synchronised.
  // Returns whether `pred` held for any thread.
  __device__ __forceinline__ bool sync_for_mma(bool pred = false) {
    tc_wait_st();
    fence_proxy_async();
    tc_fence_before();
    const int any = wg_sync_or(pred);
    tc_fence_after();
    return any != 0;
  }

  // code words of token row `rw` of page `pg`, head h (K or V region)
  __device__ __forceinline__ void load_words(const unsigned char* e, int h, int pg, int rw, uint32_t (&w)[S::kWords]) {
    const unsigned char* src = e + (pg * HPC + h) * (4 * D) + rw * (D / 4);
    if constexpr (S::kWords == 8) {
      // two 16-byte halves, the order alternating every 4 rows: the eight
      // rows of a quarter-warp then hit eight distinct bank groups
      const int c0 = (rw >> 2) & 1;
      const uint4 a = lds<uint4>(src + 16 * c0), b = lds<uint4>(src + 16 * (c0 ^ 1));
      const uint4 lo = c0 ? b : a, hi = c0 ? a : b;
      w[0] = lo.x; w[1] = lo.y; w[2] = lo.z; w[3] = lo.w;
      w[4] = hi.x; w[5] = hi.y; w[6] = hi.z; w[7] = hi.w;
    } else {
      const uint4 a = lds<uint4>(src);
      w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    }
  }

  // K codes of head h's block -> A_K[buf] (thread = token row = TMEM lane)
  __device__ __forceinline__ void unpack_k(const unsigned char* e, int h, int j, bool has, int pg, int rw, bool warp_has) {
    if (!warp_has) return;
    uint32_t w[S::kWords];
    if (has) load_words(e, h, pg, rw, w);
    else {
#pragma unroll
      for (int i = 0; i < S::kWords; ++i) w[i] = 0u;
    }
    const uint32_t col = S::kColAK + (j & 1) * S::kKCols;
    if constexpr (S::kWords == 8) {
      uint32_t t[32];
#pragma unroll
      for (int jw = 0; jw < 8; ++jw)
#pragma unroll
        for (int f = 0; f < 4; ++f) t[4 * jw + f] = tern8(w[jw], f);
      tmem_st32(tmem_row(col), t);
    } else {
      uint32_t t[16];
#pragma unroll
      for (int jw = 0; jw < 4; ++jw)
#pragma unroll
        for (int f = 0; f < 4; ++f) t[4 * jw + f] = tern8(w[jw], f);
      tmem_st16(tmem_row(col), t);
    }
  }

  // V codes of head h's block -> A_V[buf] (MN-major: byte (row mu, token k)
  // at (mu / 16) * 2048 + 16 k + mu % 16)
  __device__ __forceinline__ void unpack_v(const unsigned char* e, int h, int j, bool has, int pg, int rw) {
    if (j >= 2) wait_bar(&bars[kEntries + 2 + (j & 1)], (uint32_t)((j - 2) >> 1) & 1u);   // P.V(j - 2) read A_V[buf]
    if (!has) return;
    uint32_t w[S::kWords];
    load_words(e + S::kHalf, h, pg, rw, w);
    unsigned char* dst = av + (j & 1) * S::kAV + 16 * tid;
#pragma unroll
    for (int jw = 0; jw < S::kWords; ++jw) {
      uint4 v;
      v.x = tern8(w[jw], 0); v.y = tern8(w[jw], 1); v.z = tern8(w[jw], 2); v.w = tern8(w[jw], 3);
      *reinterpret_cast<uint4*>(dst + jw * 2048) = v;
    }
  }

  // Post an MMA command: this thread's tensor-memory stores have completed,
  // its shared-memory writes are visible to the tensor cores (async proxy),
  // then it arrives on the command's barrier; thread 0 writes the command
  // first.  Never blocks.
  __device__ __forceinline__ void post(int type, int h, int j, int nks_acc) {
    tc_wait_st();
    fence_proxy_async();
    tc_fence_before();
    const int s = ncmd & (kCmdSlots - 1);
    if (tid == 0) cmds[s] = Cmd{type, h, j, nks_acc};
    mbar_arrive(&cbars[s]);
    ++ncmd;
  }

  // MMA issue (MMA warp: converged, warp-uniform operands; one elected lane
  // issues the MMAs and the commit).
  __device__ __forceinline__ void issue_qk(int h, int j) {
    constexpr uint32_t idesc = idesc_i8(128, S::NQ, true, true, false, true);
    const uint32_t d = tmem + S::kColDS + (j & 1) * S::NQ;
    const uint32_t a = tmem + S::kColAK + (j & 1) * S::kKCols;
    const uint32_t b0 = smem_u32(bq + h * S::kBQ);
    if (elect_one()) {
#pragma unroll
      for (int s = 0; s < S::kKSteps; ++s)
        umma_i8_ts(d, a + 8 * s, smem_desc(b0 + 512 * s, 128, 16 * D), idesc, s > 0 ? 1u : 0u);
      umma_commit(&bars[kEntries + (j & 1)]);
    }
    __syncwarp();
  }

  __device__ __forceinline__ void issue_pv(int h, int j, int nks, bool accumulate) {
    constexpr uint32_t idesc = idesc_i8(128, S::NP, true, false, true, true);
    const uint32_t d = tmem + S::kColDO + h * S::NP;
    const uint32_t a0 = smem_u32(av + (j & 1) * S::kAV), b0 = smem_u32(bp + (j & 1) * S::kBP);
    if (elect_one()) {
      for (int s = 0; s < nks; ++s)
        umma_i8_ss(d, smem_desc(a0 + 512 * s, 128, 2048), smem_desc(b0 + 512 * s, 128, 2048), idesc,
                   (s > 0 || accumulate) ? 1u : 0u);
      umma_commit(&bars[kEntries + 2 + (j & 1)]);
    }
    __syncwarp();
  }

  // Softmax of head h's block: scores from D_S, P bytes into B_P[buf].
  // Returns through *l_blk the block's partial row sums of this thread.
  __device__ __forceinline__ bool softmax_block(int slot, int h, int j, bool valid, int pg, float (&ts)[S::kGmax],
                                                float (&lb)[S::kGmax], float w) {
    const int G = p.G;
    wait_bar(&bars[kEntries + (j & 1)], (uint32_t)(j >> 1) & 1u);
    tc_fence_after();
    uint32_t c[S::NQ];
    if constexpr (S::NQ == 16) tmem_ld16(tmem_row(S::kColDS + (j & 1) * S::NQ), c);
    else tmem_ld32(tmem_row(S::kColDS + (j & 1) * S::NQ), c);
    tc_wait_ld();
    const float gk = valid ? desc_of(h, slot).ks[pg] : 0.f;
    bool trig = false;
#pragma unroll
    for (int r = 0; r < S::kGmax; ++r) {
      ts[r] = -INFINITY;
      lb[r] = 0.f;
      if (r < G && valid) {
        ts[r] = digits3(c[3 * r], c[3 * r + 1], c[3 * r + 2]) * (gk * cq[h * 8 + r]);
        trig |= ts[r] - mq[h * 8 + r] > kTau;
      }
    }
    write_p(h, j, ts, lb, w, valid);
    return trig;
  }

  __device__ __forceinline__ void write_p(int h, int j, const float (&ts)[S::kGmax], float (&lb)[S::kGmax], float w,
                                          bool valid) {
    uint32_t x[S::kGmax];
#pragma unroll
    for (int r = 0; r < S::kGmax; ++r) {
      float pr_ = 0.f;
      if (valid && r < p.G) pr_ = ex2(ts[r] - mq[h * 8 + r]);
      lb[r] = pr_;
      x[r] = __float2uint_rn(pr_ * w);
    }
    unsigned char* dst = bp + (j & 1) * S::kBP + 16 * tid;
    if constexpr (S::NP == 16) {
      *reinterpret_cast<uint4*>(dst) = make_uint4(x[0], x[1], x[2], x[3]);
    } else {
      *reinterpret_cast<uint4*>(dst) = make_uint4(x[0], x[1], x[2], x[3]);
      *reinterpret_cast<uint4*>(dst + 2048) = make_uint4(x[4], x[5], x[6], x[7]);
    }
  }

  // One ternary entry: every KV head of the group, software-pipelined.
  __device__ void tern_entry(int slot) {
    const unsigned char* e = ring + slot * S::kSlotBytes;
    const Desc& d0 = desc_of(0, slot);
    const int np = d0.np, ntok = (d0.np - 1) * kPage + d0.nrows;
    const int pg = tid >> 4, rw = tid & 15;
    const bool has = pg < np, valid = tid < ntok;
    const bool warp_has = 2 * warp < np;
    const int nks = (ntok + 31) >> 5;
    unpack_k(e, 0, jc, has, pg, rw, warp_has);
    unpack_v(e, 0, jc, has, pg, rw);
    post(kCmdQK, 0, jc, 0);
    nqk = jc + 1;
#pragma unroll 1
    for (int h = 0; h < HPC; ++h) {
      const int j = jc + h;
      if (h + 1 < HPC) {
        unpack_k(e, h + 1, j + 1, has, pg, rw, warp_has);
        post(kCmdQK, h + 1, j + 1, 0);
        nqk = j + 2;
      }
      // value reference of this head: set, or re-based when a page's gamma_V
      // would push P * ratio past 2^(8 + 2)
      float uref_h = 0.f;
      int tok_h = 0;
      with_head(h, [&](HeadState& s) { uref_h = s.uref; tok_h = s.tok; });
      const float gvmax = desc_of(h, slot).gvmax;
      const bool rebase = uref_h == 0.f || gvmax > kRatioMax * uref_h;
      const float nref = rebase ? fmaxf(uref_h, gvmax) : uref_h;
      const float gv = valid ? desc_of(h, slot).vs[pg] : 0.f;
      const float wref = nref;
      float ts[S::kGmax], lb[S::kGmax];
      const bool trig = softmax_block(slot, h, j, valid, pg, ts, lb, wref > 0.f ? gv / wref * kXScale : 0.f);
      if (h + 1 < HPC) unpack_v(e, h + 1, j + 1, has, pg, rw);
      const bool slow = wg_sync_or(trig) || rebase || tok_h + 128 > kFlushTokens;
      float alpha[S::kGmax];
#pragma unroll
      for (int r = 0; r < S::kGmax; ++r) alpha[r] = 1.f;
      if (slow) {
        // new maximum of each query head over this block
#pragma unroll
        for (int r = 0; r < S::kGmax; ++r) {
          float v = ts[r];
#pragma unroll
          for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
          if (lane == 0) red[warp * 8 + r] = v;
        }
        // fold what the accumulators hold (every earlier P.V has completed)
        wait_pv(j);
        float mn[S::kGmax];
        wg_sync();
#pragma unroll
        for (int r = 0; r < S::kGmax; ++r) {
          const float mo = mq[h * 8 + r];
          mn[r] = fmaxf(mo, fmaxf(fmaxf(red[r], red[8 + r]), fmaxf(red[16 + r], red[24 + r])));
          alpha[r] = (mo == -INFINITY || mn[r] == -INFINITY) ? 0.f : ex2(mo - mn[r]);
        }
        with_head(h, [&](HeadState& s) {
          fold(h, s);
#pragma unroll
          for (int r = 0; r < S::kGmax; ++r) s.o[r] *= alpha[r];
          s.uref = nref;
        });
        tok_h = 0;
        wg_sync();                 // every thread has read mq[h] and red
        if (tid == 0) {
#pragma unroll
          for (int r = 0; r < S::kGmax; ++r) mq[h * 8 + r] = mn[r];
        }
        wg_sync();
        write_p(h, j, ts, lb, nref > 0.f ? gv / nref * kXScale : 0.f, valid);
      }
      with_head(h, [&](HeadState& s) {
#pragma unroll
        for (int r = 0; r < S::kGmax; ++r) s.l[r] = fmaf(s.l[r], alpha[r], lb[r]);
        s.tok = tok_h + 128;
      });
      const bool accumulate = !(empty_mask & (1u << h));
      post(kCmdPV, h, j, nks | (accumulate ? 256 : 0));
      npv = j + 1;
      empty_mask &= ~(1u << h);
    }
    jc += HPC;
  }

  // ---------------------------------------------- high-precision entries
  __device__ __forceinline__ void pv_masks(int nt, uint32_t& m01, uint32_t& m23) {
    const int t0 = 2 * tig;
    m01 = (t0 < nt ? 0x0000FFFFu : 0u) | (t0 + 1 < nt ? 0xFFFF0000u : 0u);
    m23 = (t0 + 8 < nt ? 0x0000FFFFu : 0u) | (t0 + 9 < nt ? 0xFFFF0000u : 0u);
  }

  __device__ __forceinline__ void qk_fp8(const unsigned char* kg, float (&s)[4]) {
    float t[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int wl = 0; wl < S::kWPT; ++wl) {
      const uint4 xa = lds<uint4>(kg + gid * D + 16 * (tig * S::kWPT + wl));
      const uint4 xb = lds<uint4>(kg + (gid + 8) * D + 16 * (tig * S::kWPT + wl));
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int jj = 2 * q4;
        const uint32_t sel = sel_pair(jj & 3);
        const uint32_t pa = prmt(jj < 4 ? xa.x : xa.y, jj < 4 ? xa.z : xa.w, sel);
        const uint32_t pb = prmt(jj < 4 ? xb.x : xb.y, jj < 4 ? xb.z : xb.w, sel);
        const int st = 4 * wl + q4;
        mma16816(t[st & 1], e4m3x2_f16(pa), e4m3x2_f16(pb), e4m3x2_f16(pa >> 16), e4m3x2_f16(pb >> 16),
                 bf16x2_f16(qf[2 * st]), bf16x2_f16(qf[2 * st + 1]));
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) s[c] = t[0][c] + t[1][c];
  }

  __device__ __forceinline__ void qk_bf16(const unsigned char* kg, float (&s)[4]) {
    float t[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int wl = 0; wl < S::kWPT; ++wl) {
      const unsigned char* ra = kg + gid * 2 * D + 32 * (tig * S::kWPT + wl);
      const unsigned char* rb = kg + (gid + 8) * 2 * D + 32 * (tig * S::kWPT + wl);
      const uint4 a0 = lds<uint4>(ra), a1 = lds<uint4>(ra + 16);
      const uint4 b0 = lds<uint4>(rb), b1 = lds<uint4>(rb + 16);
      const uint32_t ya[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const uint32_t yb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int st = 4 * wl + q4;
        mma16816_bf16(t[st & 1], prmt(ya[q4], ya[4 + q4], 0x5410u), prmt(yb[q4], yb[4 + q4], 0x5410u),
                      prmt(ya[q4], ya[4 + q4], 0x7632u), prmt(yb[q4], yb[4 + q4], 0x7632u), qf[2 * st], qf[2 * st + 1]);
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) s[c] = t[0][c] + t[1][c];
  }

  __device__ __forceinline__ void pv_fp8(const unsigned char* vg, uint32_t b0, uint32_t b1, uint32_t lo0,
                                         uint32_t lo1, int nt) {
    const int t0 = 2 * tig;
    constexpr int NWD = 2 * S::kUPT;
    uint32_t x0[NWD], x1[NWD], x2[NWD], x3[NWD];
    const int off = 8 * gid * S::kUPT;
#pragma unroll
    for (int i = 0; i < NWD; i += 2) {
      const uint2 a = lds<uint2>(vg + t0 * D + off + 4 * i);
      const uint2 b = lds<uint2>(vg + (t0 + 1) * D + off + 4 * i);
      const uint2 c = lds<uint2>(vg + (t0 + 8) * D + off + 4 * i);
      const uint2 ee = lds<uint2>(vg + (t0 + 9) * D + off + 4 * i);
      x0[i] = a.x; x0[i + 1] = a.y; x1[i] = b.x; x1[i + 1] = b.y;
      x2[i] = c.x; x2[i + 1] = c.y; x3[i] = ee.x; x3[i + 1] = ee.y;
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

  __device__ __forceinline__ void pv_bf16(const unsigned char* vg, uint32_t b0, uint32_t b1, uint32_t lo0,
                                          uint32_t lo1, int nt) {
    const int t0 = 2 * tig;
    const int off = 16 * gid * S::kUPT;
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
      const uint32_t a2 = prmt(lds<uint32_t>(vg + (t0 + 8) * 2 * D + ba), lds<uint32_t>(vg + (t0 + 9) * 2 * D + ba), sa) & m23;
      const uint32_t a3 = prmt(lds<uint32_t>(vg + (t0 + 8) * 2 * D + bb), lds<uint32_t>(vg + (t0 + 9) * 2 * D + bb), sb) & m23;
      mma16816_bf16(acc[mt], a0, a1, a2, a3, b0, b1);
      if constexpr (!NARROW) mma16816_bf16(acc[mt], a0, a1, a2, a3, lo0, lo1);
    }
  }

  // Scales the score tile, applies the row mask, moves the lazy maximum when
  // needed, accumulates the row sums and returns P^T fragments (P scaled by
  // the page's V scale relative to the warp's reference), P as an f16 hi + lo
  // pair (~22 bits).  NARROW: one query head (tig) per thread, scores s[0]
  // (token gid) and s[2] (token gid + 8); hi and lo in columns 2 tig, 2 tig + 1.
  // BF: P goes out in bf16 (BF16 pages multiply V as stored) instead of f16.
  template <bool BF>
  __device__ __forceinline__ void softmax_page(float (&s)[4], float sc, float ratio, int nt, uint32_t& b0,
                                               uint32_t& b1, uint32_t& lo0, uint32_t& lo1) {
    if constexpr (NARROW) {
      float mx = fmaxf(s[0], s[2]) * sc;
      bool masked = false;
      if (nt < kPage) {
        masked = true;
        mx = gid + 8 < nt ? mx : s[0] * sc;
        if (gid >= nt) mx = -INFINITY;
      }
      if (__any_sync(kFull, mx > m0 + kTauHp)) {
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
      float e0 = fmaf(s[0], sc, -m0), e1 = fmaf(s[2], sc, -m0);
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
    float mx0 = fmaxf(s[0], s[2]) * sc, mx1 = fmaxf(s[1], s[3]) * sc;
    bool masked = false;
    if (nt < kPage) {
      masked = true;
      const bool r0 = gid < nt, r1 = gid + 8 < nt;
      mx0 = r1 ? mx0 : s[0] * sc;
      mx1 = r1 ? mx1 : s[1] * sc;
      if (!r0) mx0 = mx1 = -INFINITY;
    }
    if (__any_sync(kFull, mx0 > m0 + kTauHp || mx1 > m1 + kTauHp)) {
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
    float e00 = fmaf(s[0], sc, -m0), e01 = fmaf(s[1], sc, -m1);
    float e10 = fmaf(s[2], sc, -m0), e11 = fmaf(s[3], sc, -m1);
    if (masked) {
      if (gid >= nt) e00 = e01 = -INFINITY;
      if (gid + 8 >= nt) e10 = e11 = -INFINITY;
    }
    const float p00 = ex2(e00), p01 = ex2(e01), p10 = ex2(e10), p11 = ex2(e11);
    l0 += p00 + p10;
    l1 += p01 + p11;
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
      const float2 g0 = __half22float2(*reinterpret_cast<const __half2*>(&h0));
      const float2 g1 = __half22float2(*reinterpret_cast<const __half2*>(&h1));
      lo0 = movtrans(f16x2(y00 - g0.x, y01 - g0.y));
      lo1 = movtrans(f16x2(y10 - g1.x, y11 - g1.y));
    }
  }

  // Re-base the warp's value-scale reference when the entry's V scales leave
  // [ref/16, 16*ref].
  __device__ __forceinline__ void rebase_value_scale(const Desc& d) {
    float vmax = 0.f, vmin = INFINITY;
    for (int i = 0; i < d.np; ++i) {
      vmax = fmaxf(vmax, d.vs[i]);
      vmin = fminf(vmin, d.vs[i]);
    }
    if (vmax > 0.f && (huref == 0.f || vmax > 16.f * huref || vmin < huref * 0.0625f)) {
      const float beta = huref / vmax;
#pragma unroll
      for (int mt = 0; mt < S::kSteps; ++mt)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[mt][c] *= beta;
      huref = vmax;
      inv_huref = 1.f / vmax;
    }
  }

  // warp h: pages of KV head h in the slot
  __device__ void hp_entry(int slot) {
    const Desc& d = desc_of(warp, slot);
    const unsigned char* e = ring + slot * S::kSlotBytes;
    uint32_t b0, b1, lo0 = 0u, lo1 = 0u;
    rebase_value_scale(d);
    hp_used = 1;
    if (d.fmt == KVC_FMT_FP8_E4M3) {
      if (!q_f16 && lane == 0) atomicOr(p.err, kErrRange);
      constexpr int GB = HPC * group_bytes(KVC_FMT_FP8_E4M3, D);
      e += warp * group_bytes(KVC_FMT_FP8_E4M3, D);
      for (int i = 0; i < d.np; ++i) {
        const int nt = i == d.np - 1 ? d.nrows : kPage;
        float s[4];
        qk_fp8(e + i * GB, s);
        softmax_page<false>(s, d.ks[i] * p.scale_log2, d.vs[i] * inv_huref, nt, b0, b1, lo0, lo1);
        pv_fp8(e + S::kHalf + i * GB, b0, b1, lo0, lo1, nt);
      }
    } else {
      e += warp * group_bytes(KVC_FMT_BF16, D);
      float s[4];
      qk_bf16(e, s);
      softmax_page<true>(s, p.scale_log2, inv_huref, d.nrows, b0, b1, lo0, lo1);
      pv_bf16(e + S::kHalf, b0, b1, lo0, lo1, d.nrows);
    }
  }

  // ------------------------------------------------------------- main
  __device__ void attach_mma(unsigned char* smem_av, unsigned char* smem_bp, unsigned char* smem_bq, uint64_t* b,
                             Cmd* cm, uint32_t tmem_base) {
    av = smem_av; bp = smem_bp; bq = smem_bq; bars = b; cmds = cm;
    cbars = b + kEntries + 4;
    tmem = tmem_base;
  }

  __device__ void run(unsigned char* smem_ring, unsigned char* smem_av, unsigned char* smem_bp, unsigned char* smem_bq,
                      Desc* d, uint64_t* b, float* m, float* c, float* rd, int* fl, Cmd* cm, uint32_t tmem_base,
                      int wg, int w_index) {
    ring = smem_ring; av = smem_av; bp = smem_bp; bq = smem_bq; descs = d; bars = b; mq = m; cq = c; red = rd;
    flags = fl;
    cmds = cm;
    cbars = b + kEntries + 4;
    ncmd = 0;
    tid = threadIdx.x & 127;
    warp = tid >> 5;
    bar_id = 1 + wg;
    tmem = tmem_base;
    lane = tid & 31;
    gid = lane >> 2;
    tig = lane & 3;
    W = w_index;
    cur_bq = -1;
    jc = nqk = npv = 0;
    fail = 0u;
    // the unit range and the first metadata chunk (warps < HPC)
    if (warp < HPC) {
      const long long c0 = (long long)W * pr.C / pr.nwg, c1 = (long long)(W + 1) * pr.C / pr.nwg;
      cursor = pr.unit_of_cost(c0);
      u1 = pr.unit_of_cost(c1);
      cb = cursor;
      MetaA a;
      meta_phase_a(p, pr, cb, u1, lane, HPC, warp, a);
      meta_phase_b(p, a, cur);
      meta_phase_a(p, pr, cb + 32, u1, lane, HPC, warp, nxa);
      nxt_b_pending = true;
      nxa_pending = false;
      const bool v0 = issue(0, warp == 0), v1 = issue(1, warp == 0);
      if (warp == 0 && lane == 0) { flags[2] = v0; flags[3] = v1; }
    }
    wg_sync();
    bool ok = true;
    int it = 0;
#pragma unroll 1
    for (;; ++it) {
      const int slot = it & 1;
      if (!flags[2 + slot]) break;
      wait_bar(&bars[slot], (uint32_t)(it >> 1) & 1u);
      if (wg_sync_or(fail)) { ok = false; break; }
      const Desc& d0 = desc_of(0, slot);
      const int fmt = d0.fmt;
      if (d0.bq != cur_bq) {
        finish();
        begin(d0.bq);
      }
      if (fmt == KVC_FMT_TERNARY2) tern_entry(slot);
      else if (fmt != kSkip && warp < HPC) hp_entry(slot);
      // every read of the slot is done before the async proxy refills it
      fence_proxy_async();
      if (wg_sync_or(fail)) { ok = false; break; }
      if (warp < HPC) {
        const bool v = issue(slot, warp == 0);
        if (warp == 0 && lane == 0) flags[2 + slot] = v;
      }
      wg_sync();
    }
    if (ok) {
      finish();
      post(kCmdStop, 0, 0, 0);
    } else {
      post(kCmdStop, 0, 0, 0);
      if (tid == 0) atomicOr(p.err, kErrTimeout);
      // let copies and MMAs still in flight land (each wait bounded) before
      // the CTA's shared and tensor memory are released
      for (int k = it; k < it + 2; ++k)
        if (flags[2 + (k & 1)]) mbar_wait(&bars[k & 1], (uint32_t)(k >> 1) & 1u);
      if (nqk > 0) mbar_wait(&bars[kEntries + ((nqk - 1) & 1)], (uint32_t)((nqk - 1) >> 1) & 1u);
      if (npv > 0) mbar_wait(&bars[kEntries + 2 + ((npv - 1) & 1)], (uint32_t)((npv - 1) >> 1) & 1u);
    }
  }
};

// The MMA warp of a warpgroup: executes the posted commands in order until
// the stop command (or a bounded wait gives up).
template <int D, int HPC, bool NARROW>
__device__ void mma_loop(UWorker<D, HPC, NARROW>& wk) {
  for (int n = 0;; ++n) {
    const int s = n & (kCmdSlots - 1);
    if (!mbar_wait(&wk.cbars[s], (uint32_t)(n / kCmdSlots) & 1u)) {
      if ((threadIdx.x & 31) == 0) atomicOr(wk.p.err, kErrTimeout);
      return;
    }
    tc_fence_after();
    const Cmd c = wk.cmds[s];
    if (c.type == kCmdQK) wk.issue_qk(c.h, c.j);
    else if (c.type == kCmdPV) wk.issue_pv(c.h, c.j, c.nks_acc & 255, (c.nks_acc >> 8) != 0);
    else return;
  }
}

template <int D, int HPC, bool NARROW>
struct USmem {
  using S = UShape<D, HPC, NARROW>;
  static constexpr size_t kRing = 0;
  static constexpr size_t kAv = kRing + (size_t)kEntries * S::kSlotBytes;
  static constexpr size_t kBp = kAv + 2 * (size_t)S::kAV;
  static constexpr size_t kBq = kBp + 2 * (size_t)S::kBP;
  static constexpr size_t kDesc = kBq + (size_t)HPC * S::kBQ;
  static constexpr size_t kBars = (kDesc + (size_t)HPC * kEntries * sizeof(Desc) + 7) & ~(size_t)7;
  static constexpr size_t kCmd = kBars + (kEntries + 4 + kCmdSlots) * sizeof(uint64_t);
  static constexpr size_t kMq = kCmd + kCmdSlots * sizeof(Cmd);
  static constexpr size_t kCq = kMq + HPC * 8 * sizeof(float);
  static constexpr size_t kRed = kCq + HPC * 8 * sizeof(float);
  static constexpr size_t kFlags = kRed + 32 * sizeof(float);
  static constexpr size_t kWgBytes = (kFlags + 4 * sizeof(int) + 1023) & ~(size_t)1023;   // one warpgroup
  static constexpr size_t kTslot = 2 * kWgBytes;                 // tensor-memory address of the CTA
  static constexpr size_t kSeq = kTslot + 16;                    // sequence tables (both warpgroups)
  static size_t bytes(int batch) { return kSeq + (size_t)(3 * batch + 2) * sizeof(int); }
};

// One CTA per SM (a kernel that allocates tensor memory runs one CTA per
// SM) holding two warpgroups; each warpgroup is an independent worker of
// the stream-K partition with its own 256 tensor-memory columns, ring and
// operand buffers.
template <int D, int HPC, bool NARROW>
__global__ void __launch_bounds__(kUmmaThreads, 1) decode_umma_kernel(DecodeParams p) {
  // warps 0-3: compute warps of warpgroup 0, 4-7: of warpgroup 1; warp 8 /
  // 9: the MMA warp of warpgroup 0 / 1; warps 10, 11: spare
  using L = USmem<D, HPC, NARROW>;
  using S = UShape<D, HPC, NARROW>;
  extern __shared__ __align__(1024) unsigned char smem[];
  int* seqP = reinterpret_cast<int*>(smem + L::kSeq);
  int* seqC = seqP + (p.B + 1);
  int* seqL = seqC + (p.B + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int whp = ucost_hp<D, NARROW>(p.hp);
  const int nq = p.Hkv / HPC;          // head groups per sequence

  const bool service = warp >= 8;
  const bool mma_warp = warp == 8 || warp == 9;
  const int wg = service ? (warp - 8) & 1 : threadIdx.x >> 7;
  unsigned char* mine = smem + wg * L::kWgBytes;          // this warpgroup's block
  uint64_t* bars = reinterpret_cast<uint64_t*>(mine + L::kBars);
  const int ltid = threadIdx.x & 127;
  if (!service && ltid < kEntries + 4) mbar_init(&bars[ltid], 1);
  if (!service && ltid < kCmdSlots) mbar_init(&bars[kEntries + 4 + ltid], 128);
  if (!service && ltid < 4) reinterpret_cast<int*>(mine + L::kFlags)[ltid] = 0;
  if (!service && ltid < HPC * 8) reinterpret_cast<float*>(mine + L::kMq)[ltid] = -INFINITY;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + L::kTslot);
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"((uint32_t)(2 * S::kTmemCols)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (warp == 0) {
    int carry_u = 0, carry_c = 0;
    for (int base = 0; base < p.B; base += 32) {
      const int b = base + lane;
      int u = 0, c = 0;
      if (b < p.B) {
        const int gb = p.b_base + b;
        int Lb = p.ctx[gb < p.Bseq ? gb : gb % p.Bseq];
        if (Lb < 0 || Lb > p.max_pages * kPage) {
          if (blockIdx.x == 0) atomicOr(p.err, kErrContext);
          Lb = 0;
        }
        seqL[b] = Lb;
        const SeqShape s = seq_shape(Lb, p.sink, p.window, whp, kCostTern);
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
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
  const long long most = pr.C / (2 * kCostMax);
  const long long workers = 2ll * gridDim.x;
  pr.nwg = (int)(workers < most ? workers : (most > 0 ? most : 1));
  const int W = 2 * blockIdx.x + wg;                      // worker index
  const bool has_work = pr.U > 0 && W < pr.nwg;
  if (service) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kServiceRegs));
    if (mma_warp && has_work) {
      UWorker<D, HPC, NARROW> wk(p, pr);
      wk.attach_mma(mine + L::kAv, mine + L::kBp, mine + L::kBq, bars, reinterpret_cast<Cmd*>(mine + L::kCmd),
                    tmem + (uint32_t)(wg * S::kTmemCols));
      mma_loop(wk);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kComputeRegs));
    if (has_work) {
      UWorker<D, HPC, NARROW> wk(p, pr);
      wk.run(mine + L::kRing, mine + L::kAv, mine + L::kBp, mine + L::kBq, reinterpret_cast<Desc*>(mine + L::kDesc),
             bars, reinterpret_cast<float*>(mine + L::kMq), reinterpret_cast<float*>(mine + L::kCq),
             reinterpret_cast<float*>(mine + L::kRed), reinterpret_cast<int*>(mine + L::kFlags),
             reinterpret_cast<Cmd*>(mine + L::kCmd), tmem + (uint32_t)(wg * S::kTmemCols), wg, W);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)(2 * S::kTmemCols)));
}

// CTAs per SM are cached per (device, batch); the largest shared-memory size
// is opted into once per device.
constexpr int kMaxDev = 64;
template <int D, int HPC, bool NARROW>
cudaError_t umma_occupancy(int batch, int* ctas_per_sm) {
  using L = USmem<D, HPC, NARROW>;
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
    e = cudaFuncSetAttribute(decode_umma_kernel<D, HPC, NARROW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)L::bytes(kUmmaMaxBatch));
    if (e != cudaSuccess) return e;
    // all of the unified L1 as shared memory: two CTAs of ~110 KB per SM
    e = cudaFuncSetAttribute(decode_umma_kernel<D, HPC, NARROW>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    opted[dev] = true;
  }
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, decode_umma_kernel<D, HPC, NARROW>, kUmmaThreads,
                                                    L::bytes(batch));
  if (e == cudaSuccess) {
    if (*ctas_per_sm > 1) *ctas_per_sm = 1;               // the tensor memory serves one CTA
    cache[key] = *ctas_per_sm;
  }
  return e;
}

template <int D, bool NARROW>
cudaError_t umma_occupancy_hpc(int hpc, int batch, int* per) {
  switch (hpc) {
    case 1: return umma_occupancy<D, 1, NARROW>(batch, per);
    case 2: return umma_occupancy<D, 2, NARROW>(batch, per);
    case 4: return umma_occupancy<D, 4, NARROW>(batch, per);
    default: return cudaErrorInvalidValue;
  }
}

template <int D, bool NARROW>
void launch_umma(const DecodeParams& p, int hpc, int grid, cudaStream_t s) {
  switch (hpc) {
    case 1: decode_umma_kernel<D, 1, NARROW><<<grid, kUmmaThreads, USmem<D, 1, NARROW>::bytes(p.B), s>>>(p); break;
    case 2: decode_umma_kernel<D, 2, NARROW><<<grid, kUmmaThreads, USmem<D, 2, NARROW>::bytes(p.B), s>>>(p); break;
    default: decode_umma_kernel<D, 4, NARROW><<<grid, kUmmaThreads, USmem<D, 4, NARROW>::bytes(p.B), s>>>(p); break;
  }
}

}  // namespace

bool umma_supported(int batch, int d, int hkv, int max_pages) {
  return (d == 64 || d == 128) && batch <= kUmmaMaxBatch &&
         (long long)batch * hkv * max_pages * kCostMax < (1ll << 31);
}

int umma_heads_per_cta(int hkv) { return hkv % 4 == 0 ? 4 : (hkv % 2 == 0 ? 2 : 1); }

cudaError_t umma_grid(int batch, int d, int hq, int hkv, int* grid) {
  int dev = 0, sms = 0, per = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int hpc = umma_heads_per_cta(hkv);
  const bool narrow = hq / hkv <= 4;
  switch (d) {
    case 64: e = narrow ? umma_occupancy_hpc<64, true>(hpc, batch, &per) : umma_occupancy_hpc<64, false>(hpc, batch, &per); break;
    case 128: e = narrow ? umma_occupancy_hpc<128, true>(hpc, batch, &per) : umma_occupancy_hpc<128, false>(hpc, batch, &per); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  *grid = sms * (per > 0 ? per : 1);
  return cudaSuccess;
}

cudaError_t launch_decode_umma(const DecodeParams& p, int head_dim, int grid, cudaStream_t s) {
  const int hpc = umma_heads_per_cta(p.Hkv);
  const bool narrow = p.G <= 4;
  switch (head_dim) {
    case 64: narrow ? launch_umma<64, true>(p, hpc, grid, s) : launch_umma<64, false>(p, hpc, grid, s); break;
    case 128: narrow ? launch_umma<128, true>(p, hpc, grid, s) : launch_umma<128, false>(p, hpc, grid, s); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace kvc
