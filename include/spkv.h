/*
 * spkv.h -- C ABI of libspkv.so: Spherical KV angle-domain attention (ADA)
 * paged decode for NVIDIA B200 (sm_100a).
 *
 * Source of the method ("the pages"): "SPHERICAL KV: Angle-Domain Attention
 * and Rate-Distortion Retention for Efficient Long-Context Inference",
 * technical summary, section 2.1 "Angle-Domain Attention (ADA)" (spherical
 * parametrisation r = ||k||, phi = Phi(k^); logit ~= ||q|| r~ f_b(c_q, c_k);
 * f_b a fused cosine from angle codes; no dense key ever written to HBM),
 * section 2.2 (tier-homogeneous pages read by header-guided streaming; the
 * retention decision z_i and tier b_i) and section 2.3 (dense keys are mapped
 * to spherical codes and stored in a paged, ragged KV substrate).
 *
 * Numerical definitions (readings of the pages, numbered as in the oracle):
 *   d = 128; angles phi_1..phi_126 in [0, pi], phi_127 in [0, 2 pi) (n-sphere
 *   chart); b-bit uniform codes c = floor(phi 2^b / range), midpoint
 *   reconstruction; the query is coded at each page's b; radius code
 *   c_r = clamp(floor((log2 ||k|| - L_h)/Delta_h + 1/2), 0, 255) with
 *   r~ = 2^(L_h + c_r Delta_h); logit = ||q|| r~ f_b / sqrt(d); softmax over
 *   retained slots (an empty set gives 0); out = sum p v over bf16 values.
 *
 * ---------------------------------------------------------------- layout
 * Page size 16 tokens.  All buffers are caller-owned DEVICE memory (except the
 * spkv_cache struct itself, which is read on the host) and must be 16-byte
 * aligned.  bf16 values are passed as uint16_t bit patterns.
 *
 *   code arena: for page p, hdr[p].code_off16 * 16 is the byte offset of the
 *   page's block of H_kv records, one per kv head, each
 *   REC(b) = 256*b + 16 bytes long:
 *     bytes [0, 256 b):   angle codes of the 16 slots, chunk-major: the 16-byte
 *                         chunk k (k < b) of slot s sits at (k*16 + s)*16.
 *                         Concatenating chunks 0..b-1 of a slot gives its
 *                         128*b-bit little-endian bitstream; angle i
 *                         (1-based, i <= 127) occupies bits [(i-1) b, i b);
 *                         the 128th field is padding and is written as 0.
 *     bytes [256 b, 256 b + 16): radius code of slot s at byte 256 b + s.
 *   values:  v_pages[p][h][s][0..127] bf16, i.e. [num_pages, H_kv, 16, 128].
 *   keep mask (optional): keep_mask[p * H_kv + h], bit s = slot s retained.
 *   block table: block_table[b * max_pages + j] = physical page of the j-th
 *   16-token page of sequence b; only j < ceil(ctx_len_b / 16) is read.
 *
 * ---------------------------------------------------------------- rules
 * Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 * default stream), never synchronises, and allocates no device memory.
 * Host-side argument checks run before any launch and return a status; no
 * C++ exception crosses the ABI.  Device-side problems found while running
 * (a page id outside [0, num_pages), a header with b not in {3,4,6,8}, a
 * record beyond the arena, a context length beyond max_ctx) set bits in
 * *err_flags (if err_flags != NULL) with atomicOr and the offending page or
 * token is skipped; kernels never trap.
 */
#ifndef SPKV_H_
#define SPKV_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SPKV_API __attribute__((visibility("default")))
#else
#define SPKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SPKV_OK = 0,
    SPKV_ERR_INVALID_ARG = 1, /* NULL pointer, negative size, misalignment     */
    SPKV_ERR_UNSUPPORTED = 2, /* head_dim != 128, page_size != 16, bad G, ...  */
    SPKV_ERR_WORKSPACE = 3,   /* ws_bytes smaller than the required size        */
    SPKV_ERR_CUDA = 4         /* a CUDA runtime call or launch failed           */
} spkv_status;

/* Device error bits written to *err_flags. */
#define SPKV_DEVERR_PAGE_ID 0x1u   /* block-table entry outside [0, num_pages) */
#define SPKV_DEVERR_BITS 0x2u      /* page header b not in {3,4,6,8}           */
#define SPKV_DEVERR_RECORD 0x4u    /* record would lie beyond the code arena   */
#define SPKV_DEVERR_CTX 0x8u       /* ctx_len < 0 or > max_ctx or > max_pages*16 */
#define SPKV_DEVERR_TIMEOUT 0x10u  /* a bounded pipeline wait gave up          */
#define SPKV_DEVERR_RADIUS 0x20u   /* Delta_h <= 0 or not finite               */

/* Per-page header (tier-homogeneous pages, section 2.2): every slot and every
 * kv head of a page shares one bit width. */
typedef struct {
    uint32_t code_off16; /* byte offset of the page's records / 16          */
    uint8_t bits;        /* b in {3, 4, 6, 8}                                */
    uint8_t pad[3];
} spkv_page_hdr;

/* Compressed paged key store plus bf16 value pages.  The struct lives in host
 * memory; every pointer in it is device memory. */
typedef struct {
    int32_t num_kv_heads;        /* H_kv >= 1                                    */
    int32_t head_dim;            /* must be 128                                  */
    int32_t page_size;           /* must be 16                                   */
    int32_t num_pages;           /* physical pages                               */
    uint8_t *code_arena;         /* records, see layout above                    */
    uint64_t code_arena_bytes;   /* arena size, for bounds checks                */
    const spkv_page_hdr *hdr;    /* [num_pages]                                  */
    const float *rad_lo_log2;    /* [H_kv] L_h                                   */
    const float *rad_step_log2;  /* [H_kv] Delta_h (> 0)                         */
    uint16_t *v_pages;           /* [num_pages, H_kv, 16, 128] bf16              */
    const uint16_t *keep_mask;   /* [num_pages, H_kv] or NULL (all retained)     */
    uint32_t *err_flags;         /* device word for SPKV_DEVERR_* bits, or NULL  */
    uint32_t tiers;              /* bit t set when some page uses b = {3,4,6,8}[t]; 0 = any.
                                    Decoding codes the query only for these tiers; a page
                                    of another tier sets SPKV_DEVERR_BITS and is skipped. */
} spkv_cache;

/* Human-readable name of a status. */
SPKV_API const char *spkv_status_string(spkv_status s);

/* Encode and append keys (and optionally values) into the paged store
 * (sections 2.1 and 2.3: dense keys -> radius code + packed angle codes).
 *   keys      [B, n_new, H_kv, 128] bf16, device
 *   values    [B, n_new, H_kv, 128] bf16, device, or NULL to leave V untouched
 *   start_pos [B] int32, device: token n of sequence b goes to position
 *             start_pos[b] + n, i.e. page block_table[b][pos/16], slot pos%16
 *   block_table [B, max_pages] int32, device
 * Each key's bit width is its page's hdr.bits.  Angle and radius codes are
 * decided in fp64 from the exact squares of the bf16 inputs.  Only the slots
 * written are touched (their code bits, radius byte and, with values, V row).
 * Positions at or beyond max_pages*16 set SPKV_DEVERR_CTX and are skipped. */
SPKV_API spkv_status spkv_encode_keys(const spkv_cache *cache, const uint16_t *keys, const uint16_t *values,
                             const int32_t *start_pos, int32_t B, int32_t n_new,
                             const int32_t *block_table, int32_t max_pages, void *stream);

/* Number of work partitions ("splits") the decode calls use when num_splits
 * is 0: a multiple of the device's SM count, at most one per 8 (page, kv
 * head) units of the largest possible batch.  -1 on a CUDA error. */
SPKV_API int32_t spkv_decode_default_splits(int32_t B, int32_t num_kv_heads, int32_t max_ctx);

/* Workspace bytes needed by spkv_decode_attention / spkv_dense_decode /
 * spkv_decompress_then_dot for these sizes and this split count (0 = default):
 * the split partials (rounded up to 16 bytes), then one 4-byte counter per
 * (sequence, kv head) row (rounded up to 16 bytes) that the call zeroes on
 * its stream before its kernels run.  The workspace needs no initialisation.
 * Returns 0 for invalid sizes. */
SPKV_API size_t spkv_decode_workspace_bytes(int32_t B, int32_t num_q_heads, int32_t num_kv_heads,
                                   int32_t max_ctx, int32_t num_splits);

/* ADA decode attention (section 2.1): for every sequence b and query head
 * hq (kv head h = hq / G, G = Hq / H_kv), over the slots t < ctx_lens[b] that
 * the keep mask retains:
 *   logit_t = ||q|| r~_t f_b(c_q, c_t) / sqrt(128),  out = softmax(logit) . V
 * computed straight from the codes (no dense key is ever written).
 *   q        [B, Hq, 128] bf16, device
 *   block_table [B, max_pages] int32, device; ctx_lens [B] int32, device
 *   max_ctx  host upper bound of ctx_lens (sizes the work); ctx_lens[b]
 *            larger than max_ctx or than max_pages*16 sets SPKV_DEVERR_CTX
 *            and that sequence's output is 0
 *   out      [B, Hq, 128], fp32 (out_is_bf16 = 0) or bf16 (out_is_bf16 = 1)
 *   ws       device workspace of ws_bytes >= spkv_decode_workspace_bytes(...)
 *   num_splits  0 = default; otherwise the number of balanced partitions of
 *            the (page, kv head) work (any value gives the same result up to
 *            fp32 rounding order)
 * Supported: G in {1, 2, 4, 8}, B <= 1024. */
SPKV_API spkv_status spkv_decode_attention(const spkv_cache *cache, const uint16_t *q, int32_t B, int32_t num_q_heads,
                                  const int32_t *block_table, int32_t max_pages, const int32_t *ctx_lens,
                                  int32_t max_ctx, void *out, int32_t out_is_bf16, void *ws, size_t ws_bytes,
                                  int32_t num_splits, void *stream);

/* Flag bits of spkv_decode_attention_ex and spkv_debug_logits_ex. */
#define SPKV_DECODE_EXACT_Q 1u

/* spkv_decode_attention with flag bits; flags = 0 is spkv_decode_attention.
 *   SPKV_DECODE_EXACT_Q  the exact-query variant of f_b.  Section 2.1 of the
 *       summary writes f_b(c_q, c_k), a cosine from the codes of both sides,
 *       and leaves f_b itself open; with this flag the query is NOT coded:
 *       f = <q / ||q||, u~(c_k)>, the unquantised unit query against the
 *       decoded key (a zero query gives f = 0).  Same bytes read per token.
 * Unknown flag bits: SPKV_ERR_INVALID_ARG (before any launch).  Every other
 * argument, layout and rule is that of spkv_decode_attention. */
SPKV_API spkv_status spkv_decode_attention_ex(const spkv_cache *cache, const uint16_t *q, int32_t B,
                                     int32_t num_q_heads, const int32_t *block_table, int32_t max_pages,
                                     const int32_t *ctx_lens, int32_t max_ctx, void *out, int32_t out_is_bf16,
                                     void *ws, size_t ws_bytes, int32_t num_splits, uint32_t flags, void *stream);

/* Decode step with the fused single-token append (the serving loop's per-step
 * path; section 2.3 of the summary maps each new key to its spherical codes
 * and stores it in the compressed format): for every sequence b with
 * ctx_lens[b] >= 1 whose pages the decode walks, token ctx_lens[b] - 1 takes
 *   new_keys[b, h, :]   -> its radius and angle codes, written into slot
 *                          (ctx - 1) mod 16 of page block_table[b][(ctx - 1) / 16]
 *                          exactly as spkv_encode_keys writes them, and
 *   new_values[b, h, :] -> the same slot of v_pages,
 * for every kv head h, and then the decode of spkv_decode_attention_ex runs
 * over ctx_lens[b] tokens including it -- all in the decode's own launches
 * (no separate encode launch).  The result equals spkv_encode_keys with
 * start_pos = ctx_lens - 1 and n_new = 1 followed by spkv_decode_attention_ex.
 *   new_keys, new_values  [B, H_kv, 128] bf16, device, 8-byte aligned
 * Everything else as spkv_decode_attention_ex (flags included).  The page's
 * header must already hold its bit width; a bad page id / header / record is
 * flagged by the decode and the token is not written.  Sequences the decode
 * skips (ctx 0, or ctx > max_ctx: SPKV_DEVERR_CTX) get no append. */
SPKV_API spkv_status spkv_decode_attention_append(const spkv_cache *cache, const uint16_t *new_keys,
                                         const uint16_t *new_values, const uint16_t *q, int32_t B,
                                         int32_t num_q_heads, const int32_t *block_table, int32_t max_pages,
                                         const int32_t *ctx_lens, int32_t max_ctx, void *out,
                                         int32_t out_is_bf16, void *ws, size_t ws_bytes, int32_t num_splits,
                                         uint32_t flags, void *stream);

/* Page-sharded decode, for one long sequence (the 128K regime of the
 * summary's section 4) whose pages are split across GPUs: each GPU decodes
 * the pages it holds with this call and the shards are combined with
 * spkv_merge_partials.  Same arguments and rules as spkv_decode_attention_ex
 * (block_table / ctx_lens describe this shard's pages), but instead of the
 * output it writes for every sequence b and query head hq the record
 *   partial_out[b, hq, 0..131] = { M, L, 0, 0, o[0..127] }
 *   M  max over the shard's retained tokens of logit * log2(e)  (-inf: none)
 *   L  sum over them of 2^(logit * log2(e) - M)
 *   o  the shard's own attention output (softmax over its tokens times V)
 * partial_out: [B, Hq, 132] fp32, device, 16-byte aligned. */
SPKV_API spkv_status spkv_decode_attention_partial(const spkv_cache *cache, const uint16_t *q, int32_t B,
                                          int32_t num_q_heads, const int32_t *block_table, int32_t max_pages,
                                          const int32_t *ctx_lens, int32_t max_ctx, float *partial_out, void *ws,
                                          size_t ws_bytes, int32_t num_splits, uint32_t flags, void *stream);

/* Combine R shard records of spkv_decode_attention_partial:
 *   out[b, hq, :] = sum_r w_r o_r / sum_r w_r,  w_r = 2^(M_r - max_r M_r) L_r
 * (shards with M_r = -inf carry no weight; 0 when no shard retained a token),
 * which is the attention over the union of the shards' tokens.
 *   partials [R, B, Hq, 132] fp32, device, 16-byte aligned (R >= 1)
 *   out      [B, Hq, 128] fp32 or bf16 (out_is_bf16), device, 16-byte aligned */
SPKV_API spkv_status spkv_merge_partials(const float *partials, int32_t R, int32_t B, int32_t num_q_heads,
                                void *out, int32_t out_is_bf16, void *stream);

/* Dense paged decode over bf16 keys, the uncompressed comparison path
 * (section 4 of the summary compares against dense KV):
 * logit = q . k / sqrt(128), same paging, mask, split and output rules as
 * spkv_decode_attention.
 *   k_pages, v_pages [num_pages, H_kv, 16, 128] bf16, device
 *   keep_mask [num_pages, H_kv] or NULL;  err_flags device word or NULL */
SPKV_API spkv_status spkv_dense_decode(const uint16_t *k_pages, const uint16_t *v_pages, int32_t num_pages,
                              int32_t num_kv_heads, const uint16_t *keep_mask, uint32_t *err_flags,
                              const uint16_t *q, int32_t B, int32_t num_q_heads, const int32_t *block_table,
                              int32_t max_pages, const int32_t *ctx_lens, int32_t max_ctx, void *out,
                              int32_t out_is_bf16, void *ws, size_t ws_bytes, int32_t num_splits,
                              void *stream);

/* The "decompress, then dot" strawman of the summary's problem statement:
 * first writes k~ = bf16(r~ u~(c)) for every page the block table references
 * below ctx_lens into k_scratch ([num_pages, H_kv, 16, 128] bf16, device;
 * other pages are left untouched), then runs spkv_dense_decode on k_scratch
 * and cache->v_pages with the UNQUANTISED query.  Same arguments and rules as
 * spkv_decode_attention otherwise. */
SPKV_API spkv_status spkv_decompress_then_dot(const spkv_cache *cache, uint16_t *k_scratch, const uint16_t *q, int32_t B,
                                     int32_t num_q_heads, const int32_t *block_table, int32_t max_pages,
                                     const int32_t *ctx_lens, int32_t max_ctx, void *out, int32_t out_is_bf16,
                                     void *ws, size_t ws_bytes, int32_t num_splits, void *stream);

/* Size of the library-owned workspace used by spkv_decode_attention_static_ws
 * (bytes, per device). */
#define SPKV_STATIC_WS_BYTES (16u * 1024u * 1024u)

/* ADA decode attention for callers that cannot allocate device memory while
 * they decode (a fixed memory budget checked at start-up, an allocator that
 * is not reachable from the decoding thread, a host program that must not
 * call the CUDA allocator after initialisation).  The summary pages have no
 * counterpart of this entry point: it is spkv_decode_attention with its
 * split-partials workspace taken from an array of SPKV_STATIC_WS_BYTES that
 * the library holds in device memory on every device that loads it, until
 * the process exits; it allocates nothing itself.
 *   Arguments and results: as spkv_decode_attention, without ws / ws_bytes;
 *   its argument checks run first, so an invalid argument gets the status it
 *   gets there.
 *   Limit: then returns SPKV_ERR_WORKSPACE when spkv_decode_workspace_bytes(B,
 *   num_q_heads, H_kv, max_ctx, num_splits) exceeds SPKV_STATIC_WS_BYTES
 *   (e.g. B = 8, 32 query / 8 kv heads and the default split count need
 *   about 4.6 MB).
 *   Set-up: the first call in a CUDA context, with the device current, looks
 *   up the array's device address (cudaGetSymbolAddress) and caches it with
 *   the context's id (cuCtxGetId); make that first call before any stream
 *   capture.  A call from another context of the device -- after
 *   cudaDeviceReset, or once the primary context was released and created
 *   again, when the module is loaded at a new address -- looks the address up
 *   again, so that first call in the new context must also come before any
 *   capture.
 *   Sharing: every call on a device uses the same array, and each call
 *   overwrites what the previous one left there (nothing in it needs to start
 *   at zero).  Calls whose kernels overlap on the GPU (different streams, no
 *   ordering between them) race on the array and give wrong results. */
SPKV_API spkv_status spkv_decode_attention_static_ws(const spkv_cache *cache, const uint16_t *q, int32_t B,
                                                     int32_t num_q_heads, const int32_t *block_table,
                                                     int32_t max_pages, const int32_t *ctx_lens,
                                                     int32_t max_ctx, void *out, int32_t out_is_bf16,
                                                     int32_t num_splits, void *stream);

/* Test hook: the ADA logits themselves (natural-log units, before softmax),
 * logits[b, hq, t] for t < ctx_lens[b]; evicted slots get -inf; entries at or
 * beyond ctx_lens[b] are not written.  logits: [B, Hq, max_ctx] fp32, device. */
SPKV_API spkv_status spkv_debug_logits(const spkv_cache *cache, const uint16_t *q, int32_t B, int32_t num_q_heads,
                              const int32_t *block_table, int32_t max_pages, const int32_t *ctx_lens,
                              int32_t max_ctx, float *logits, void *stream);

/* spkv_debug_logits with the flag bits of spkv_decode_attention_ex. */
SPKV_API spkv_status spkv_debug_logits_ex(const spkv_cache *cache, const uint16_t *q, int32_t B,
                                 int32_t num_q_heads, const int32_t *block_table, int32_t max_pages,
                                 const int32_t *ctx_lens, int32_t max_ctx, float *logits, uint32_t flags,
                                 void *stream);

/* Test hook for the bounded waits: one kernel waits, with the decode
 * kernels' own bounded-wait routine, on an mbarrier that nothing completes,
 * for at most limit_ns (1 .. 1e9 ns).  The wait gives up: it sets
 * SPKV_DEVERR_TIMEOUT in *err_flags and the kernel returns normally, writing
 *   status[0] = 1 (the wait gave up; 0 would mean it completed),
 *   status[1] = microseconds waited, status[2] = 1 (the abort flag it raised).
 * err_flags: one device word; status: 3 int32 on the device.  Invalid
 * arguments: SPKV_ERR_INVALID_ARG, nothing launched.  (The pages have no
 * counterpart: this checks the library's own failure handling.) */
SPKV_API spkv_status spkv_debug_wait_timeout(uint32_t *err_flags, int32_t *status, uint64_t limit_ns, void *stream);

/* ------------------------------------------------------------------ RDR
 * Rate-distortion retention controller (technical summary section 2.2: a
 * residency decision and a precision tier for every state under a hard
 * memory budget, from a distortion surrogate built on the codes' angular
 * error scaled by query and key magnitudes; protected states at the top
 * tier; tier-homogeneous pages).  Readings, for the parts the section leaves
 * open:
 *   - the unit is a token: its kv heads share a page and so a tier;
 *   - D_t(b) = w_t eps_b, w_t = sum_h qn_h ||k_{t,h}||_2, eps_b =
 *     pi / (2^b sqrt 12); an evicted token costs w_t (eps = 1);
 *   - rate R(b) = H_kv (16 b + 1 + 256) bytes for a resident token (angle
 *     codes, radius byte, bf16 value row), 0 when evicted;
 *   - protected tokens take b_max, the largest tier in tier_mask.
 * Each token minimises D_t(b) + lambda R(b) (ties: the larger b); lambda is
 * the smallest multiplier whose total rate fits the budget, found by doubling
 * from 1 and bisection on [0, hi] in fp64 (at most 100 halvings).  The plan
 * is then packed: resident tokens grouped by tier (b ascending), ascending t
 * within a tier, each group filling whole pages of 16 slots, its last page
 * partly (attention over the kept tokens does not depend on their order).
 *
 *   keys        [total_tokens, H_kv, 128] bf16, device, 16-byte aligned:
 *               sequence s owns rows seq_start[s] .. seq_start[s+1]-1
 *   seq_start   [B + 1] int32, device, nondecreasing, in [0, total_tokens]
 *   q_norms     [B, H_kv] fp32, device: qn_h per sequence (>= 0)
 *   protect     [total_tokens] uint8, device, or NULL: nonzero = protected
 *   budget_bytes [B] fp64, device: the rate budget of each sequence
 *   tier_mask   allowed tiers, bit i: b = {3,4,6,8}[i]; nonzero, < 16
 *   max_pages_out  capacity of page_bits / page_keep per sequence; a plan
 *               needs at most ceil(T_s / 16) + 3 pages
 * Outputs (device):
 *   tier        [total_tokens] uint8: b, or 0 = evicted
 *   dst_pos     [total_tokens] int32: page * 16 + slot of the token in its
 *               sequence's packed pages, -1 when evicted
 *   page_bits   [B, max_pages_out] uint8: b of packed page p (p < n_pages)
 *   page_keep   [B, max_pages_out] uint16: occupied slots of packed page p
 *   n_pages     [B] int32: packed pages of the sequence
 *   lambda, rate_bytes, distortion  [B] fp64: the multiplier (+inf when
 *               infeasible), the plan's rate and its surrogate distortion
 *   status      [B] int32: 0, or SPKV_RDR_* bits
 * ws: spkv_rdr_workspace_bytes(total_tokens) bytes of device memory, 16-byte
 * aligned, owned by the caller (the per-token weights).  Every pointer is
 * the caller's; the call only enqueues work on `stream`.  Argument errors
 * (NULL, misalignment, H_kv outside 1..32, a bad tier_mask, a short
 * workspace) return without launching. */
#define SPKV_RDR_INFEASIBLE 0x1 /* protected tokens alone exceed the budget:
                                   they are kept at b_max, all others evicted */
#define SPKV_RDR_PAGES 0x2      /* the packed plan needs more than max_pages_out
                                   pages: n_pages says how many; dst_pos = -1
                                   and no page entries written */
#define SPKV_RDR_BAD_RANGE 0x4  /* seq_start out of order or out of range: the
                                   sequence's n_pages, lambda, rate and
                                   distortion are 0; no tier, dst_pos or page
                                   entry is written for it */

SPKV_API size_t spkv_rdr_workspace_bytes(int64_t total_tokens);

SPKV_API spkv_status spkv_rdr_plan(const uint16_t *keys, const int32_t *seq_start, int32_t B, int64_t total_tokens,
                                   int32_t num_kv_heads, const float *q_norms, const uint8_t *protect,
                                   const double *budget_bytes, uint32_t tier_mask, int32_t max_pages_out,
                                   uint8_t *tier, int32_t *dst_pos, uint8_t *page_bits, uint16_t *page_keep,
                                   int32_t *n_pages, double *lambda, double *rate_bytes, double *distortion,
                                   int32_t *status, void *ws, size_t ws_bytes, void *stream);

/* Encode keys (and optionally values) to scattered positions: the packed
 * layout of an RDR plan (section 2.2) or any other placement.
 *   keys, values  [total_tokens, H_kv, 128] bf16, device (values may be NULL)
 *   seq_start     [B + 1] int32, device: sequence s owns rows
 *                 seq_start[s] .. seq_start[s+1]-1
 *   dst_pos       [total_tokens] int32, device: position of the token in its
 *                 sequence (page block_table[s][pos/16], slot pos%16); a
 *                 negative position skips the token
 *   block_table   [B, max_pages] int32, device
 * Codes and errors as spkv_encode_keys. */
SPKV_API spkv_status spkv_encode_keys_packed(const spkv_cache *cache, const uint16_t *keys, const uint16_t *values,
                                             const int32_t *seq_start, int32_t B, int64_t total_tokens,
                                             const int32_t *dst_pos, const int32_t *block_table, int32_t max_pages,
                                             void *stream);

/* Host tables of the non-uniform angle quantiser (an f_b variant; technical
 * summary section 2.1 leaves the quantiser open).  Reading: for a direction
 * drawn uniformly on the unit sphere of R^d, polar angle phi_i (i = 1..d-2)
 * has the density sin^(d-1-i)(phi)/Z on [0, pi]; each polar angle gets 2^b
 * cells of equal probability (edges at the j/2^b quantiles) reconstructed at
 * the cell median (the (j+1/2)/2^b quantile); the azimuth keeps the uniform
 * cells.  Computed on the host in fp64 (no GPU, no stream):
 *   edge_cos [(d-2) * (2^b - 1)]  cos of edge j = 1..2^b-1 of angle i, row i-1
 *   mid_cos, mid_sin [(d-2) * 2^b] cos / sin of the reconstruction angles
 * All three are caller-owned host arrays.  d in 3..4096, b in 1..12, else
 * SPKV_ERR_INVALID_ARG with nothing written. */
SPKV_API spkv_status spkv_nonuniform_tables(int32_t d, int32_t b, double *edge_cos, double *mid_cos,
                                            double *mid_sin);

/* Encode with the non-uniform angle quantiser (the tables above, d = 128):
 * as spkv_encode_keys, except that polar angle i (i = 1..126) takes the code
 * of the largest edge j of ITS OWN edges that it reaches (phi_i >= theta_ij
 * <=> x_i <= sqrt(S_i) cos theta_ij, decided exactly on x_i^2 vs S_i cos^2
 * and the signs, so an input on an edge goes to the upper cell up to the
 * tables' 1e-12); the azimuth and the radius byte are as spkv_encode_keys.
 *   bits      b in {3, 4, 6, 8}: every page written must have this width
 *             (others set SPKV_DEVERR_BITS and are skipped), else
 *             SPKV_ERR_UNSUPPORTED
 *   edge_cos  [126 * (2^b - 1)] fp64, device, 8-byte aligned: the edge_cos
 *             table of spkv_nonuniform_tables(128, b), row i-1 for angle i
 * Decode such a cache with spkv_decode_attention_nonuniform. */
SPKV_API spkv_status spkv_encode_keys_nonuniform(const spkv_cache *cache, const uint16_t *keys,
                                                 const uint16_t *values, const int32_t *start_pos, int32_t B,
                                                 int32_t n_new, const int32_t *block_table, int32_t max_pages,
                                                 int32_t bits, const double *edge_cos, void *stream);

/* Bytes of the workspace spkv_decode_attention_nonuniform needs (0: invalid
 * arguments): the per-split partial records and the decode's (cos, sin)
 * table.  num_splits 0: the default count, which queries the current
 * device's SM count. */
SPKV_API size_t spkv_decode_nonuniform_workspace_bytes(int32_t B, int32_t num_q_heads, int32_t num_kv_heads,
                                                       int32_t max_ctx, int32_t num_splits, int32_t bits);

/* ADA decode attention over a cache written by spkv_encode_keys_nonuniform
 * at b = bits (every page the block tables reference below ctx_lens must
 * have that width; others set SPKV_DEVERR_BITS and are dropped):
 *   out[b, hq, :] = softmax_t(||q|| r~_t f_b(q, k_t) / sqrt(128)) . V
 * with f_b the cosine of the decoded angles (cell medians: mid_cos / mid_sin
 * of spkv_nonuniform_tables(128, b) for the polar angles, the uniform medians
 * for the azimuth) and the query coded with the same quantiser at b.  Same
 * paging, keep-mask, context and error rules as spkv_decode_attention.
 *   edge_cos [126 * (2^b - 1)], mid_cos / mid_sin [126 * 2^b]: fp64, device
 *   out      [B, Hq, 128] fp32 or bf16 (out_is_bf16), device, 16-byte aligned
 *   logits   NULL, or [B, Hq, max_ctx] fp32 device: the logits (natural-log
 *            units) of t < ctx_lens[b], -inf for evicted slots
 *   ws       spkv_decode_nonuniform_workspace_bytes(...) bytes, device,
 *            256-byte aligned (else SPKV_ERR_WORKSPACE)
 *   num_splits  splits of each (sequence, kv head) row; 0: default
 * Bits of b outside {3, 4, 6, 8} or G = Hq / H_kv outside {1, 2, 4, 8}:
 * SPKV_ERR_UNSUPPORTED.  (A plain CUDA-core kernel: this variant is
 * checked against its oracle; the tuned path is the uniform quantiser's.) */
SPKV_API spkv_status spkv_decode_attention_nonuniform(const spkv_cache *cache, const uint16_t *q, int32_t B,
                                                      int32_t num_q_heads, const int32_t *block_table,
                                                      int32_t max_pages, const int32_t *ctx_lens, int32_t max_ctx,
                                                      int32_t bits, const double *edge_cos, const double *mid_cos,
                                                      const double *mid_sin, void *out, int32_t out_is_bf16,
                                                      float *logits, void *ws, size_t ws_bytes, int32_t num_splits,
                                                      void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SPKV_H_ */
