/*
 * kvc.h - C ABI of libkvc: a compressed, mixed-format paged KV cache and
 * single-token decode attention over it, for NVIDIA B200 (sm_100a).
 *
 * The cache layout follows two of the source pages:
 *   - "Show HN: Vantage-V-AI" (newshot.cc), section "Core architecture":
 *     keys and values quantised to ternary {-1, 0, +1} with an absmean scale
 *     gamma = mean(|X|), packed 4 codes per uint8 byte (2.0 bit/element);
 *     attention-sink tokens kept at full precision; section "Quick start":
 *     the knobs max_active_tokens (recent window), sink_tokens and
 *     quant_mode = "fp8" (dynamic FP8 streaming).
 *   - "Minima-KV" (twodots.gr), sections "Recent, Anchor and Stale" and
 *     "How mixed-format attention works": pages of one request held in
 *     different formats (recent pages high precision, older anchor pages kept
 *     at higher fidelity, stale pages compressed but still addressable), read
 *     directly by format-specific code paths whose partial states (max
 *     score, sum of exponentials, output) are merged by one online-softmax
 *     normalisation.  Section "Why the KV cache becomes a bottleneck":
 *     non-contiguous physical pages addressed through a block table.
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" must be CUDA device (or managed) memory on
 *     the current device; "host" pointers are ordinary host memory.  The
 *     caller owns every buffer; the library never allocates, frees or keeps
 *     a pointer after the call returns.
 *   - Calls that take a stream only enqueue work on it and never
 *     synchronise; inputs must stay valid until that work completes.
 *   - Argument errors are reported before anything is enqueued, as a
 *     kvc_status; nothing is written in that case.
 *   - Page size is fixed at 16 tokens; head_dim is 64, 128 or 256.
 *
 * Page layouts (HND: head-major inside each page; all little-endian):
 *   BF16       [page][Hkv][16][D]    bf16
 *   FP8_E4M3   [page][Hkv][16][D]    OCP e4m3 bytes; one float32 scale per
 *                                    page (over all KV heads), value = s * e
 *   TERNARY2   [page][Hkv][16][D/4]  2-bit codes, element i of a (page,
 *                                    head) group's row-major [token][dim]
 *                                    order in byte i/4 at bits 2*(i%4)..+1,
 *                                    00 = 0, 01 = +1, 11 = -1 (10 unused,
 *                                    read as 0); one float32 gamma per
 *                                    (page, KV head), value = gamma * c
 */
#ifndef KVC_H
#define KVC_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVC_API __attribute__((visibility("default")))
#else
#define KVC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, passed through untouched (0 = the legacy default stream). */
typedef struct CUstream_st* kvc_stream_t;

typedef enum {
  KVC_OK = 0,
  KVC_ERR_INVALID_ARG = 1,   /* null pointer, negative size, misaligned pointer, ... */
  KVC_ERR_UNSUPPORTED = 2,   /* a shape this build does not handle (head_dim, page size, GQA > 8) */
  KVC_ERR_WORKSPACE = 3,     /* workspace missing or smaller than kvc_decode_workspace_size() */
  KVC_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
  KVC_ERR_DEVICE_CHECK = 5,  /* a device-side check failed (see kvc_decode_read_error) */
  KVC_ERR_TIMEOUT = 6        /* a device-side wait gave up after its iteration limit */
} kvc_status;

typedef enum {
  KVC_FMT_BF16 = 0,
  KVC_FMT_FP8_E4M3 = 1,
  KVC_FMT_TERNARY2 = 2
} kvc_format;

#define KVC_PAGE_SIZE 16

/*
 * Version of the byte layouts the library writes and reads; compressed
 * pages are persistent data (saved, offloaded, reloaded), so a layout
 * change bumps it.  Version 1:
 *   ternary group  [Hkv][16][D/4] bytes per page, element i of a group's
 *                  row-major [token][dim] order at byte i/4, bits 2(i%4)..+1,
 *                  fields 00 = 0, 01 = +1, 11 = -1; gamma fp32 [Hkv] per page
 *   FP8 page       [Hkv][16][D] OCP e4m3 bytes + one fp32 scale per page
 *   BF16 page      [Hkv][16][D] bf16
 *   codec blob     as described above kvc_exans_encode
 */
#define KVC_LAYOUT_VERSION 1

/* Human-readable name of a status code (static string, never NULL). */
KVC_API const char* kvc_status_string(kvc_status status);

/* KVC_LAYOUT_VERSION of the library as built (compare with the header's). */
KVC_API int kvc_layout_version(void);

/*
 * kvc_quantize_pack_pages - compress whole pages into one page format.
 *
 * Ternary (Vantage, "Core architecture"; scale granularity per (page, KV
 * head)): for each (page, KV head) group of 16*D values,
 *   gamma = mean(|x|)  (float32, pairwise-tree sum),
 *   code  = +1 if x > gamma/2, -1 if x < -gamma/2, else 0
 *           (RoundClip(x / gamma, -1, +1), ties to 0),
 * packed 4 per byte as described above; dst_scale receives gamma [n][Hkv].
 * FP8 (Vantage "Quick start" quant_mode = "fp8"; Minima "Recent, Anchor and
 * Stale", recent pages in FP8): per page, amax = max |x| over all heads,
 *   s = amax / 448, e = round-to-nearest-even, saturating e4m3 of
 *   x * (448 / amax) (float32 arithmetic); amax = 0 gives s = 1;
 * dst_scale receives s [n].  BF16: dst[i] is a copy of the source page and
 * dst_scale is ignored (may be NULL).
 *
 *   src_bf16   device, bf16 [n_src][Hkv][16][D]; 16-byte aligned
 *   page_ids   device int32 [n]: dst page i is made from src page
 *              page_ids[i]; NULL means page_ids[i] = i
 *   n          number of pages to produce (0 is a no-op)
 *   page_size  must be 16
 *   dst        device, layout of `mode` [n][...]; 16-byte aligned
 *   dst_scale  device float32, [n][Hkv] (ternary) or [n] (FP8)
 *   n_src_pages  pages in src (>= 1; >= n when page_ids is NULL)
 *   device_flags device uint32 or NULL: an id outside [0, n_src_pages) is
 *              checked on the device, its dst page (and scale) left as it
 *              was, and bit 1 set in *device_flags (atomicOr; the caller
 *              zeroes and reads it)
 */
KVC_API kvc_status kvc_quantize_pack_pages(const void* src_bf16, const int32_t* page_ids, int n,
                                   int page_size, int n_kv_heads, int head_dim,
                                   kvc_format mode, void* dst, float* dst_scale,
                                   int64_t n_src_pages, uint32_t* device_flags,
                                   kvc_stream_t stream);

/*
 * kvc_dequantize_pages - expand compressed pages back to bf16 (the inverse
 * used to re-expand a stale page; Minima, "Recent, Anchor and Stale").
 * Ternary: bf16(gamma * c); FP8: bf16(s * e), the product in float32, both
 * rounded to nearest even.  BF16: a copy.
 *
 *   src        device, layout of `mode`, [n_src][...]
 *   src_scale  device float32: gamma [n_src][Hkv] (ternary) or s [n_src]
 *              (FP8); ignored for BF16
 *   page_ids   device int32 [n] or NULL: dst page i is made from src page
 *              page_ids[i] (NULL: i)
 *   dst_bf16   device bf16 [n][Hkv][16][D]; 16-byte aligned
 *   n_src_pages, device_flags   as for kvc_quantize_pack_pages (an id
 *              outside the source leaves its dst page as it was, bit 1)
 */
KVC_API kvc_status kvc_dequantize_pages(const void* src, const float* src_scale, const int32_t* page_ids,
                                int n, int page_size, int n_kv_heads, int head_dim,
                                kvc_format mode, void* dst_bf16, int64_t n_src_pages,
                                uint32_t* device_flags, kvc_stream_t stream);

/* Per-format page pools of one attention layer.  K and V are separate pools
 * that share the block table: logical page j of sequence b lives in slot
 * block_table[b][j] of the K and V pools of that page's format.  Pools of a
 * format that no page uses may be NULL. */
typedef struct kvc_paged_cache {
  const void* k_bf16;          /* bf16 [n_pages[0]][Hkv][16][D] */
  const void* v_bf16;
  const void* k_fp8;           /* e4m3 [n_pages[1]][Hkv][16][D] */
  const void* v_fp8;
  const float* k_fp8_scale;    /* [n_pages[1]] */
  const float* v_fp8_scale;
  const void* k_tern;          /* packed [n_pages[2]][Hkv][16][D/4] */
  const void* v_tern;
  const float* k_gamma;        /* [n_pages[2]][Hkv] */
  const float* v_gamma;
  int64_t n_pages[3];          /* pool sizes, indexed by kvc_format */
} kvc_paged_cache;

/*
 * kvc_append_retier - one decode step's cache update, for every sequence of
 * the batch: the sink tokens stay and the high-precision window slides
 * ("Show HN: Vantage-V-AI", section "Core architecture"), and the page that
 * ages out of the recent tier moves to the compressed stale tier (Minima-KV,
 * section "Recent, Anchor and Stale").  Per sequence b, with L the length
 * BEFORE the step (window_tokens >= 1, so the newest page is high
 * precision):
 *   1. retier: page j0 with (j0+1)*16 == L - window_tokens + 1, unless it
 *      holds sink tokens, leaves the window.  If its tag is TERNARY2
 *      (older_fmt NULL, or older_fmt[b][j0] == TERNARY2) its hp_mode content
 *      (the bf16 values, or bf16(s*e) of an FP8 page) is quantised to
 *      ternary -- the codec of kvc_quantize_pack_pages -- into ternary slot
 *      ternary_slot[b] of the K and V pools; block_table[b][j0] becomes that
 *      slot, older_fmt[b][j0] (if given) TERNARY2, and freed_hp_slot[b] the
 *      released high-precision slot.  A tag equal to hp_mode keeps the page
 *      in place (an anchor); freed_hp_slot[b] is -1 when nothing moved.
 *   2. append: token L (k_new[b], v_new[b]) goes to row L % 16 of page
 *      L / 16, whose hp_mode slot the caller has put in block_table[b][L/16]
 *      (a new slot when L % 16 == 0; that page is zeroed first).  BF16 pages
 *      take the row as it is; FP8 pages are re-quantised whole (decode to
 *      bf16(s*e), insert the row, new amax and scale, encode).
 * The caller then advances its lengths to L + 1.
 *
 *   k_new_bf16, v_new_bf16  device bf16 [batch][Hkv][D], 16-byte aligned
 *   cache          host pointer to the pools; the hp_mode pools and the
 *                  ternary pools are WRITTEN (the pointers are cast from
 *                  const); hp_mode BF16 or FP8_E4M3
 *   block_table    device int32 [batch][max_pages], read and updated
 *   older_fmt      device uint8 [batch][max_pages] or NULL, updated
 *   context_lens   device int32 [batch], each in [0, max_pages*16 - 1]
 *   ternary_slot   device int32 [batch]: ternary slot for a retiered page
 *   freed_hp_slot  device int32 [batch], out
 *   device_flags   device uint32 word or NULL: OR-ed with 1 (a block-table
 *                  or ternary slot outside its pool; that part is skipped),
 *                  2 (a leaving page tagged with the other high-precision
 *                  format; left in place), 4 (a length out of range; the
 *                  sequence is skipped)
 * Errors: INVALID_ARG for null or misaligned pointers, negative sizes,
 * window_tokens < 1 or a bad hp_mode; UNSUPPORTED for page_size != 16 or a
 * head_dim other than 64, 128, 256.  Asynchronous on `stream`; allocates
 * nothing.
 */
KVC_API kvc_status kvc_append_retier(const void* k_new_bf16, const void* v_new_bf16,
                                     const kvc_paged_cache* cache, int32_t* block_table,
                                     uint8_t* older_fmt, const int32_t* context_lens,
                                     const int32_t* ternary_slot, int32_t* freed_hp_slot,
                                     uint32_t* device_flags, int batch, int n_kv_heads,
                                     int head_dim, int page_size, int max_pages, int sink_tokens,
                                     int window_tokens, kvc_format hp_mode, kvc_stream_t stream);

/*
 * kvc_promote_pages - stale-to-anchor promotion: re-expand selected stale
 * (ternary) pages into anchors, the higher-fidelity tier that Minima-KV
 * keeps for critical older pages while stale pages stay addressable in
 * compressed form ("Minima-KV", section "Recent, Anchor and Stale").
 * Request i moves logical page req_page[i] of sequence req_seq[i] to slot
 * anchor_slot[i] of the anchor_fmt pools, K and V alike.  The page's
 * content is bf16(gamma * c) per KV head (what kvc_dequantize_pages gives);
 * a BF16 anchor stores it as it is, an FP8 anchor encodes the bf16 page
 * with the FP8 page codec of kvc_quantize_pack_pages (one scale over all KV
 * heads, K and V separately; heads whose codes are all 0 add nothing to
 * amax).  block_table[b][j] becomes the anchor slot, older_fmt[b][j]
 * becomes anchor_fmt and freed_ternary_slot[i] the released ternary slot
 * (the ternary bytes are left as they are).
 *
 *   cache          host pointer to the pools; the anchor_fmt pools (and
 *                  their FP8 scales) are WRITTEN (pointers cast from const)
 *   block_table    device int32 [batch][max_pages], read and updated
 *   older_fmt      device uint8 [batch][max_pages], read and updated
 *                  (required: the tag is what makes the page an anchor)
 *   context_lens   device int32 [batch]
 *   req_seq, req_page, anchor_slot  device int32 [n_requests]; requests
 *                  name distinct pages and distinct anchor slots
 *   freed_ternary_slot  device int32 [n_requests], out: the ternary slot,
 *                  or -1 for a skipped request
 *   device_flags   device uint32 word or NULL: OR-ed with 4 (sequence or
 *                  page outside the batch / the sequence's pages), 2 (the
 *                  page is not ternary: a sink, window or anchor page), 1
 *                  (a ternary or anchor slot outside its pool); such a
 *                  request is skipped and changes nothing
 *   hp_mode        format of sink and window pages (BF16 or FP8_E4M3), for
 *                  the page classification
 *   anchor_fmt     BF16 or FP8_E4M3
 * Errors: INVALID_ARG for null or misaligned pointers, negative sizes, a bad
 * hp_mode or anchor_fmt; UNSUPPORTED for page_size != 16, a head_dim other
 * than 64, 128, 256, or batch * max_pages >= 2^31.  Asynchronous on
 * `stream`; allocates nothing; one CTA per request.
 */
/*
 * Lossless exponent-split codec for high-precision pages ("ExANS komprimerer
 * KV-cache og goer AI-svar hurtigere paa H100 GPU", ainews.dk, on "ExANS -
 * Lossless KV cache compression at 622 GB/s on H100"): every BF16 value is
 * split into its exponent and its sign + mantissa; the exponents of a group
 * are coded with an asymmetric numeral system around the group's centre,
 * the sign + mantissa bytes are kept raw.  A group is one page of one pool
 * ([Hkv][16][D] bf16, N = Hkv*16*D values; N <= 2^22), coded on its own:
 *   - centre = the most frequent exponent (smallest among ties); symbol =
 *     exponent - centre + 8 when in 0..14, else 15 (escape, its exponent
 *     byte kept in an escape stream in element order);
 *   - byte-wise rANS, 32-bit state in [2^23, 2^31), 12-bit frequencies
 *     f = max(1, count*4096/N) per present symbol with the remainder on the
 *     largest; 32 interleaved states (state i codes elements 128c + 4i + r,
 *     r = 0..3) share one byte stream: after each symbol the states below
 *     2^23 take one byte each in state order, then a second round likewise;
 *   - a group whose coded blob would exceed 64 + 2N bytes is stored raw.
 * Blob (little-endian, a multiple of 16 bytes): u32 total, mode (0 raw,
 * 1 coded), N, centre, escapes, stream bytes; 8 zero bytes; u16 f[16]; then
 * the 2N raw bytes, or the N sign+mantissa bytes (sign << 7 | mantissa),
 * the escape bytes and the rANS stream (32 initial states as u32, then the
 * renormalisation bytes), each zero-padded to 16.
 */

/* Workspace bytes kvc_exans_encode needs for n pages: n * (4N + 192). */
KVC_API kvc_status kvc_exans_workspace_size(int n, int page_size, int n_kv_heads, int head_dim,
                                            size_t* bytes);

/*
 * kvc_exans_encode - code n pages into blobs stored back to back.
 *   src_bf16   device bf16 [n_src][Hkv][16][D], 16-byte aligned
 *   page_ids   device int32 [n] or NULL: blob i codes src page page_ids[i]
 *   workspace  device, >= kvc_exans_workspace_size bytes, 16-byte aligned
 *   dst        device, dst_bytes >= n * (64 + 2N) (no blob exceeds its raw
 *              size plus the header), 16-byte aligned
 *   offsets    device int64 [n + 1], out: blob i is dst[offsets[i],
 *              offsets[i+1]); offsets[n] = the coded size
 *   n_src_pages  pages in src (>= 1; >= n when page_ids is NULL)
 *   device_flags device uint32 or NULL: an id outside [0, n_src_pages) is
 *              checked on the device; its blob codes src page 0 instead (the
 *              blobs stay back to back) and bit 1 is set
 * Errors: INVALID_ARG (null or misaligned pointers, n outside 0..2^24,
 * dst_bytes too small, n_src_pages out of range), WORKSPACE, UNSUPPORTED
 * (page_size != 16, head_dim not 64/128/256, N > 2^22).  Asynchronous on `stream` (three launches:
 * code into per-page workspace slots, prefix sum of the sizes, compaction);
 * allocates nothing.
 */
KVC_API kvc_status kvc_exans_encode(const void* src_bf16, const int32_t* page_ids, int n, int page_size,
                                    int n_kv_heads, int head_dim, void* workspace, size_t workspace_bytes,
                                    void* dst, size_t dst_bytes, int64_t* offsets, int64_t n_src_pages,
                                    uint32_t* device_flags, kvc_stream_t stream);

/*
 * kvc_exans_decode - decode blobs back to bf16 pages (bit-exact inverse).
 *   src, src_bytes  device blobs as kvc_exans_encode wrote them
 *   offsets    device int64 [n_blobs + 1]
 *   blob_ids   device int32 [n] or NULL: page i decodes blob blob_ids[i]
 *   dst_bf16   device bf16 [n][Hkv][16][D], 16-byte aligned
 *   device_flags  device uint32 word or NULL: OR-ed with 1 (a blob id,
 *              offset or header that does not fit; that page is left as it
 *              is) or 2 (a coded stream or escape stream that does not end
 *              where its header says: corrupt data)
 * Errors: INVALID_ARG, UNSUPPORTED as above.  Asynchronous; one warp per
 * page.
 */
KVC_API kvc_status kvc_exans_decode(const void* src, size_t src_bytes, const int64_t* offsets, int n_blobs,
                                    const int32_t* blob_ids, int n, int page_size, int n_kv_heads,
                                    int head_dim, void* dst_bf16, uint32_t* device_flags,
                                    kvc_stream_t stream);

KVC_API kvc_status kvc_promote_pages(const kvc_paged_cache* cache, int32_t* block_table,
                                     uint8_t* older_fmt, const int32_t* context_lens,
                                     const int32_t* req_seq, const int32_t* req_page,
                                     const int32_t* anchor_slot, int n_requests,
                                     int32_t* freed_ternary_slot, uint32_t* device_flags, int batch,
                                     int n_kv_heads, int head_dim, int page_size, int max_pages,
                                     int sink_tokens, int window_tokens, kvc_format hp_mode,
                                     kvc_format anchor_fmt, kvc_stream_t stream);

/*
 * kvc_plan_paged_cache - host-side page placement (a small block manager).
 * Decides each logical page's format with the same rule the decode kernel
 * applies, and gives every page a slot in the pool of its format.
 *
 * Format of logical page j of sequence b (length L = context_lens[b]):
 *   hp_mode         if the page holds any of the first sink_tokens tokens
 *                   or any of the last window_tokens tokens,
 *   older_fmt[b][j] otherwise (TERNARY2 for stale pages, BF16 or FP8 for
 *                   anchors; older_fmt == NULL means TERNARY2).
 * Slots of each pool are handed out in increasing slot_key order (ties by
 * logical index b*max_pages + j); slot_key == NULL gives logical order.
 *
 *   context_lens  host int32 [batch], each in [0, max_pages*16]
 *   older_fmt     host uint8 [batch][max_pages] or NULL
 *   slot_key      host float32 [batch][max_pages] or NULL
 *   block_table   host int32 [batch][max_pages] out (unused entries 0)
 *   page_fmt      host uint8 [batch][max_pages] out (unused entries 255)
 *   pool_pages    host int32 [3] out: pages per format
 *   pool_src_ids  host int32 [batch*max_pages] out: the logical page id
 *                 b*max_pages + j held by each slot, format by format
 *                 (BF16 slots first, then FP8, then ternary) - the page_ids
 *                 to pass to kvc_quantize_pack_pages for each pool.
 */
KVC_API kvc_status kvc_plan_paged_cache(const int32_t* context_lens, int batch, int max_pages,
                                int page_size, int sink_tokens, int window_tokens,
                                kvc_format hp_mode, const uint8_t* older_fmt,
                                const float* slot_key, int32_t* block_table,
                                uint8_t* page_fmt, int32_t* pool_pages,
                                int32_t* pool_src_ids);

/*
 * kvc_decode_workspace_size - bytes of device workspace that
 * kvc_decode_attention_paged needs for these shapes on the current device
 * (split-K partial states, merge tickets and an error word).
 */
KVC_API kvc_status kvc_decode_workspace_size(int batch, int n_q_heads, int n_kv_heads, int head_dim,
                                     int max_pages, size_t* bytes);

/* Decode kernels (kvc_decode_plan_info's *kernel). */
#define KVC_DECODE_KERNEL_CUDA_CORE 0   /* CUDA-core fallback: shapes the others do not take */
#define KVC_DECODE_KERNEL_MMA 1         /* tensor-core kernel (register-sourced MMAs), the default */
#define KVC_DECODE_KERNEL_TCGEN05 2     /* tensor-memory kernel, opt-in (KVC_DECODE_KERNEL=tcgen05) */

/*
 * kvc_decode_plan_info - which kernel kvc_decode_attention_paged runs for
 * these shapes on the current device, and in how many launches (a batch
 * above the tensor-core kernel's per-launch limit of 1024 virtual sequences
 * is decoded in consecutive launches).  Host only; enqueues nothing.
 *
 *   batch     virtual sequences of the call (n_layers * batch for
 *             kvc_decode_attention_paged_layers)
 *   kernel    host int32 out: a KVC_DECODE_KERNEL_* value
 *   launches  host int32 out: kernel launches per call (0 for batch 0)
 *
 * Errors: as kvc_decode_workspace_size; KVC_ERR_INVALID_ARG for a NULL
 * output pointer.
 */
KVC_API kvc_status kvc_decode_plan_info(int batch, int n_q_heads, int n_kv_heads, int head_dim,
                                        int max_pages, int32_t* kernel, int32_t* launches);

/*
 * kvc_decode_attention_paged - one query token per sequence attends to its
 * whole mixed-format paged cache (Minima, "How mixed-format attention
 * works"; page formats as in kvc_plan_paged_cache).
 *
 * For query head h of sequence b (KV head g = h / (Hq/Hkv)):
 *   s_t   = softmax_scale * q_h . k_hat_t        for t < L_b
 *   out_h = sum_t softmax(s)_t * v_hat_t
 * where k_hat, v_hat are the decoded cache values (bf16 value, s*e, or
 * gamma*c, never re-rounded).  Each page is read in its own format; the
 * sequence is split over pages, each split emits (max score, sum of
 * exponentials, output) and the last split to finish merges them.  Tokens
 * at or beyond L_b are masked; L_b = 0 gives a zero output row.
 *
 *   q_bf16        device bf16 [batch][Hq][D]
 *   cache         host pointer to the pool descriptor (copied by value)
 *   block_table   device int32 [batch][max_pages]
 *   older_fmt     device uint8 [batch][max_pages] or NULL (all TERNARY2)
 *   context_lens  device int32 [batch], each in [0, max_pages*16]
 *   hp_mode       BF16 or FP8_E4M3: format of sink and window pages
 *   softmax_scale <= 0 selects 1/sqrt(head_dim)
 *   out           device float32 [batch][Hq][D]
 *   workspace     device, >= kvc_decode_workspace_size() bytes, 256-byte
 *                 aligned, any contents: each call clears its error word and
 *                 merge tickets first (one cudaMemsetAsync on `stream`,
 *                 captured with the kernel in a CUDA graph) and rewrites the
 *                 partial states, so one workspace serves repeated calls and
 *                 graph replay, but not two calls in flight at once.  The
 *                 flags of a call are therefore read before the next call.
 * Device-side checks (block-table entry outside its pool, unknown page
 * format, context length out of range) skip the offending page or
 * sequence and set a flag that kvc_decode_read_error() returns.
 * Arithmetic: products on tensor cores, sums in fp32 (ternary pages at
 * GQA <= 4: exact int32 sums of P's two 8-bit digits, P relative to the
 * running maximum, 2^-15 steps).  Environment, read once per process:
 * KVC_DECODE_KERNEL=tcgen05 selects the tensor-memory kernel;
 * KVC_DECODE_TERNARY_PV=f16 runs the ternary pages' P.V at GQA <= 4 on f16
 * MMAs (P as an f16 hi + lo pair) instead, =pair keeps the int8 products but
 * tests the running maximum per page pair rather than once per full entry
 * of 8 pages; KVC_TEST_DECODE_TIMEOUT=1 is a
 * failure-detection test mode of the tensor-core kernel: its first ring
 * slot waits for bytes no copy delivers, every bounded wait on it gives up
 * after a few short tries, and the call sets flag 8 (output rows not
 * written) without faulting or hanging.
 */
KVC_API kvc_status kvc_decode_attention_paged(const void* q_bf16, const kvc_paged_cache* cache,
                                      const int32_t* block_table, const uint8_t* older_fmt,
                                      const int32_t* context_lens, int batch, int n_q_heads,
                                      int n_kv_heads, int head_dim, int page_size, int max_pages,
                                      int sink_tokens, int window_tokens, kvc_format hp_mode,
                                      float softmax_scale, float* out, void* workspace,
                                      size_t workspace_bytes, kvc_stream_t stream);

/*
 * kvc_decode_attention_paged_layers - the same decode attention for all
 * attention layers of one decode step in a single launch (a step of a
 * multi-layer model replays one launch instead of one per layer; Minima-KV,
 * "What the memory measurements showed", runs its direct decode under CUDA
 * graphs).  Layers share the page placement: one block table, one set of
 * page tags and lengths; each layer has its own pools and queries.
 *
 *   q_bf16        device bf16 [n_layers][batch][Hq][D]
 *   cache         pools holding n_layers * n_pages[f] pages of each format:
 *                 slot s of layer l is page l * n_pages[f] + s (n_pages are
 *                 the per-layer pool sizes; gamma / FP8 scales likewise)
 *   block_table, older_fmt, context_lens   as for one layer, [batch][...]
 *   out           device float32 [n_layers][batch][Hq][D]
 *   workspace     >= kvc_decode_workspace_size(n_layers * batch, ...) bytes
 * n_layers * n_pages[f] * n_kv_heads must stay below 2^31 for every format
 * (KVC_ERR_UNSUPPORTED otherwise).
 * Everything else as kvc_decode_attention_paged, which is this call with
 * n_layers = 1.  INVALID_ARG also for n_layers < 1 or n_layers * batch
 * above 2^30.
 */
KVC_API kvc_status kvc_decode_attention_paged_layers(const void* q_bf16, const kvc_paged_cache* cache,
                                                     const int32_t* block_table, const uint8_t* older_fmt,
                                                     const int32_t* context_lens, int n_layers, int batch,
                                                     int n_q_heads, int n_kv_heads, int head_dim,
                                                     int page_size, int max_pages, int sink_tokens,
                                                     int window_tokens, kvc_format hp_mode,
                                                     float softmax_scale, float* out, void* workspace,
                                                     size_t workspace_bytes, kvc_stream_t stream);

/*
 * kvc_decode_read_error - synchronise `stream`, then read and clear the
 * device error flags in `workspace` (as sized for these shapes).  *flags
 * receives a bit mask: 1 = block-table entry out of range, 2 = unknown page
 * format, 4 = context length out of range, 8 = a bounded wait timed out,
 * 16 = a query value beyond the f16 range (|q| > 65504) met an FP8 page, whose
 * products are taken in f16 (its output rows are then not reliable; BF16
 * and ternary pages take any finite bf16 Q, K and V).
 * Returns KVC_OK, or KVC_ERR_CUDA if the copy failed.
 */
KVC_API kvc_status kvc_decode_read_error(void* workspace, int batch, int n_q_heads, int n_kv_heads,
                                 int head_dim, int max_pages, uint32_t* flags,
                                 kvc_stream_t stream);

/*
 * kvc_decode_attention_paged_noalloc - kvc_decode_attention_paged for
 * callers that cannot allocate device memory (code whose allocations all go
 * through a framework's own pool, plugins with a fixed memory budget, or
 * latency-critical paths that must not add a cudaMalloc).  The source
 * pages have no counterpart of this entry point; it exists for such
 * callers only.
 *
 * Same arguments and result as kvc_decode_attention_paged, without the
 * workspace: the split-K partial states, merge tickets and error word live
 * in a file-scope device array of KVC_NOALLOC_SCRATCH_BYTES bytes that
 * every GPU loading the library holds until the process exits.  The call
 * allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *   - The first call on a device looks up the array's device address on
 *     that device (cudaGetSymbolAddress, with the device current) and caches
 *     it; make that first call before any stream capture.  The cached
 *     address belongs to that device's primary context: after
 *     cudaDeviceReset the library must be reloaded (a new process) before
 *     this entry point is used again on that device.
 *   - Each call clears the error word and the merge tickets with
 *     cudaMemsetAsync on `stream` before the kernel; the partial states are
 *     fully rewritten.
 *   - Every call on a device shares the one array: calls whose work
 *     overlaps on the GPU (other streams, other host threads) race and give
 *     wrong results.  Serialise them.
 *   - Shapes whose workspace (kvc_decode_workspace_size) exceeds
 *     KVC_NOALLOC_SCRATCH_BYTES are rejected with KVC_ERR_WORKSPACE.
 *   - Device-side check flags are written into the shared array and are not
 *     reported by this entry point.
 */
#define KVC_NOALLOC_SCRATCH_BYTES (16u << 20)

KVC_API kvc_status kvc_decode_attention_paged_noalloc(
    const void* q_bf16, const kvc_paged_cache* cache, const int32_t* block_table,
    const uint8_t* older_fmt, const int32_t* context_lens, int batch, int n_q_heads,
    int n_kv_heads, int head_dim, int page_size, int max_pages, int sink_tokens,
    int window_tokens, kvc_format hp_mode, float softmax_scale, float* out, kvc_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KVC_H */
