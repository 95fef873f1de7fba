/*
 * kvc.h -- C ABI of the compressed-KV single-token decode attention library
 * (libkvc.so, CUDA for NVIDIA B200 / sm_100a).
 *
 * What the library computes.  Single-token decode attention read directly
 * from a compressed KV cache.  Per KV head, keys and values are stored as a
 * token latent L (T x r) times a small factor B (r x d):
 *   - low-rank KV cache, optionally combined with quantization: "BELT Connects
 *     KV-Cache Compression to Faster Long-Context Decoding", sections 2-4;
 *   - INT4 latent with per-group fp16 scale and zero, min/max uniform rule:
 *     "BellowsKV Architecture: Block-Shared Cache Latents, Outlier-Free Low-Bit
 *     Storage, and Single-Decision Eviction ...", "Worked Example: Why the
 *     Latent Quantizes Flat";
 *   - keys stored before RoPE and rotated on reconstruction: "JoLT:
 *     Near-Lossless KV Cache Compression", "Key findings";
 *   - a rotated low-bit residual of the truncation error: "A JoLT for the KV
 *     cache: Near-Lossless KV Cache Compression via Joint Rank-bit
 *     Allocation", Abstract; attention evaluated over the stored factors
 *     without materializing dense K/V (same Abstract, FlashJoLT);
 *   - one latent shared by a block of layers, each layer with its own
 *     up-projection, symmetric per-group quantization without rotation:
 *     BellowsKV page, "Share the Input, Not the Cache" and "Three
 *     Measurements, Three Operators";
 *   - a per-token variable rank, never zero: "VarRate: Training-Free
 *     Variable-Rate KV Cache Compression for Long-Context LLMs", "Method".
 * The output equals (up to rounding) textbook softmax attention of each query
 * head over the dequantized, reconstructed keys and values.
 *
 * Conventions (all entry points):
 *   - The caller owns all device memory: cache buffers, factors, page table,
 *     offsets, queries, outputs and the workspace.  The library owns only the
 *     host-side layout handle.  No entry point allocates device memory.
 *   - Work is enqueued on the caller's stream (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream).  No entry point synchronizes the
 *     device.
 *   - Every entry point returns a kvc_status and never throws or aborts.  On
 *     error nothing is launched and kvc_last_error() describes the problem
 *     (thread-local string, valid until the next call on the same thread).
 *   - Device pointers must be 16-byte aligned (KVC_EALIGN otherwise).
 *   - A layout is immutable after creation and may be shared across threads.
 *   - Query head h reads KV head h / (n_q_heads / n_kv_heads).
 *   - fp16 = IEEE binary16, bf16 = bfloat16, both little-endian in memory.
 */
#ifndef KVC_H_
#define KVC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVC_OK = 0,
  KVC_EINVAL = 1,        /* bad argument: NULL pointer, bad shape, bad value   */
  KVC_EUNSUPPORTED = 2,  /* valid but unsupported combination of options       */
  KVC_ECAPACITY = 3,     /* token count or slot beyond the cache's capacity    */
  KVC_EALIGN = 4,        /* a device pointer is not 16-byte aligned            */
  KVC_EWORKSPACE = 5,    /* workspace smaller than kvc_workspace_bytes()       */
  KVC_ECUDA = 6          /* a kernel launch or CUDA call failed                */
} kvc_status;

typedef enum {
  KVC_DENSE_BF16 = 0,    /* plain bf16 K/V cache (baseline on the same library) */
  KVC_LOWRANK = 1,       /* per-head latent x factor, optional residual/pages   */
  KVC_BLOCK_SHARED = 2,  /* one latent per block of layers                      */
  KVC_VARRATE = 3        /* per-token rank, ragged records                      */
} kvc_kind;

/* Layout description.  Zero-initialise, then set the fields the kind uses.
 *
 * KVC_LOWRANK:  rank_k, rank_v (even, 2..128); latent_bits 16 (fp16 latent,
 *   no quantization) or 4 (INT4, asymmetric, group_size along the rank, one
 *   fp16 (scale, zero) pair per group, last group may be partial);
 *   rope = 1 stores keys pre-RoPE and rotates them on reconstruction with
 *   rope_theta ("rotate half": pairs (i, i + d/2), angle = t * theta^(-2i/d),
 *   t = the token's slot index); resid_bits = 2 adds a 2-bit residual per token
 *   in the basis Q = H_d diag(signs) / sqrt(d) (Sylvester Hadamard, d = 128);
 *   page_size = 16 stores tokens in 16-token pages of an n_pages pool.
 * KVC_VARRATE: rank_k = rank_v = max rank (64); per-token ranks from
 *   {4, 8, 16, 32, 64}; latent_bits = 4, group_size = 32.
 * KVC_BLOCK_SHARED: n_layers layers share one latent of latent_dim values per
 *   token, symmetric integer codes (x = (code - 2^(b-1)) * scale, codes from
 *   round(x / scale) with scale = max|x| / (2^(b-1) - 1) per group) with one
 *   fp16 scale per group_size values; latent_bits b in {4 (0 means 4), 8, 3};
 *   value_bits 0: the one latent feeds the keys and the values of every layer;
 *   value_bits in {2, 3, 4, 8}: a second latent at that width feeds the values
 *   (the key latent at latent_bits feeds the keys) -- the operating points of
 *   the BellowsKV page ("Reading the Retention Table": n = 2 with INT8, n = 4
 *   with INT4, INT3, a 3-bit key / 2-bit value variant); per-layer fp16
 *   up-projections W_k, W_v [n_layers, latent_dim, n_kv_heads * head_dim].
 * KVC_DENSE_BF16: bf16 K/V; n_layers >= 1 layers stored.
 */
typedef struct {
  int32_t kind;           /* kvc_kind                                         */
  int32_t batch;          /* B, 1..256                                        */
  int32_t n_q_heads;      /* Hq, multiple of n_kv_heads                       */
  int32_t n_kv_heads;     /* Hkv                                              */
  int32_t head_dim;       /* d: 64 or 128                                     */
  int32_t max_tokens;     /* capacity per batch row (multiple of page_size)   */
  int32_t n_layers;       /* BLOCK_SHARED / DENSE: layers (0 means 1)          */
  int32_t rank_k;         /* LOWRANK / VARRATE                                */
  int32_t rank_v;
  int32_t latent_bits;    /* 16 or 4                                          */
  int32_t group_size;     /* quantization group                               */
  int32_t latent_dim;     /* BLOCK_SHARED latent width (512; 16..512, a
                             multiple of 16)                                 */
  int32_t rope;           /* 0 or 1 (LOWRANK)                                 */
  int32_t resid_bits;     /* 0 or 2 (LOWRANK, head_dim 128)                   */
  int32_t page_size;      /* 0 (contiguous) or 16 (LOWRANK)                   */
  int32_t n_pages;        /* physical pages in the pool when paged            */
  int32_t out_bf16;       /* 0: fp32 output, 1: bf16 output                   */
  int32_t value_bits;     /* BLOCK_SHARED: 0 (shared) or a value latent's width */
  float softmax_scale;    /* 0 means 1/sqrt(head_dim)                         */
  double rope_theta;      /* RoPE base (500000 for Llama-3.1)                 */
} kvc_layout_desc;

typedef struct kvc_layout kvc_layout;  /* opaque, host-side */

/* Cache buffers (device pointers, caller-owned; unused fields NULL).
 *
 * Row index of token t of batch row b, KV head h:
 *   contiguous: row = (b * Hkv + h) * max_tokens + t
 *   paged:      row = (page_table[b * (max_tokens / P) + t / P] * Hkv + h) * P + t % P
 * KVC_LOWRANK, per row:
 *   lk_codes  INT4: rank_k/2 bytes, element 2i in the low nibble of byte i;
 *             fp16 latent: rank_k fp16 values
 *   lk_sz     INT4 only: ceil(rank_k/group_size) fp16 pairs (scale, zero)
 *   lv_codes, lv_sz   same for values with rank_v
 *   rk_codes, rv_codes  resid_bits = 2: d/4 bytes, element 4i+k in bits 2k..2k+1
 *                       of byte i; rk_scale, rv_scale: one fp16 per row
 *   bk, bv    fp16 [Hkv, rank, d] factors (k_t = l_t * Bk (+ Q^T y_t))
 *   signs_k, signs_v    int8 [d] of +-1 (the diagonal of the rotation)
 *   page_table          int32 [B, max_tokens / page_size], physical page ids
 * KVC_VARRATE: lk_codes / lv_codes are per-batch byte streams
 *   [B, kvc_buffer_sizes()/B]; token t of row b occupies
 *   stream[b][offset[b][t] .. offset[b][t+1]) and holds, for each KV head in
 *   order, r/2 INT4 code bytes then ceil(r/32) fp16 (scale, zero) pairs with
 *   r = rank[b][t]; offset_k/offset_v int32 [B, max_tokens + 1] (offset[b][0]
 *   must be 0), rank_k/rank_v uint8 [B, max_tokens]; bk, bv fp16 [Hkv, 64, d]
 *   of which a token uses its first r rows.
 * KVC_BLOCK_SHARED: lk_codes uint8 [B, max_tokens, latent_dim * latent_bits / 8]
 *   (element i in bits [b i, b i + b) of the row's little-endian bit stream),
 *   lk_sz fp16 [B, max_tokens, latent_dim/group_size]; with value_bits > 0 the
 *   value latent likewise in lv_codes / lv_sz; bk = W_k, bv = W_v.
 * KVC_DENSE_BF16: k_dense, v_dense bf16 [n_layers, B, Hkv, max_tokens, d].
 * n_tokens: tokens 0..n_tokens-1 of every row are attended.  seq_lens
 *   (optional, device int32 [B]) gives per-row lengths; values are clamped to
 *   [0, n_tokens].  A row of length 0 produces a zero output.
 * layer: BLOCK_SHARED and layered DENSE decode: 0 decodes all n_layers layers
 *   at once (q, out [n_layers, B, Hq, d]); l + 1 decodes layer l alone (q, out
 *   [B, Hq, d]) -- a layer of a block run on its own, reading the same shared
 *   latent.  Ignored by the other kinds and by kvc_append.
 * status: optional device uint32 word.  kvc_append ORs KVC_DEV_* bits into it
 *   for every token it had to skip because a device-side argument was invalid
 *   (see kvc_append); the library never clears it.  NULL: skips go unreported.
 * Page-table entries outside [0, n_pages) never make a kernel touch memory
 *   outside the cache: decode kernels clamp them (the row then reads some
 *   page's data), append skips the token and sets KVC_DEV_BAD_PAGE.
 */
typedef struct {
  void* lk_codes;
  void* lk_sz;
  void* lv_codes;
  void* lv_sz;
  void* rk_codes;
  void* rk_scale;
  void* rv_codes;
  void* rv_scale;
  void* k_dense;
  void* v_dense;
  const void* bk;
  const void* bv;
  const int8_t* signs_k;
  const int8_t* signs_v;
  const int32_t* page_table;
  int32_t* offset_k;
  int32_t* offset_v;
  uint8_t* rank_k;
  uint8_t* rank_v;
  const int32_t* seq_lens;
  int32_t n_tokens;
  int32_t layer;
  uint32_t* status;
} kvc_cache;

/* Bits of the device-side status words: kvc_cache.status (append) and the
 * workspace error word (decode, see kvc_decode_attn). */
enum {
  KVC_DEV_WAIT_TIMEOUT = 1u,   /* decode: a bounded wait gave up; output invalid  */
  KVC_DEV_BAD_POS = 2u,        /* append: pos[b] outside [0, max_tokens - n_new]  */
  KVC_DEV_BAD_RANK = 4u,       /* append: a VARRATE rank not in {4,8,16,32,64}    */
  KVC_DEV_BAD_PAGE = 8u,       /* append: a page-table entry outside [0, n_pages)  */
  KVC_DEV_BAD_OFFSET = 16u     /* append: a VARRATE record beyond its byte stream  */
};

/* Indices into the sizes[] array filled by kvc_buffer_sizes(). */
enum {
  KVC_BUF_LK_CODES = 0, KVC_BUF_LK_SZ, KVC_BUF_LV_CODES, KVC_BUF_LV_SZ,
  KVC_BUF_RK_CODES, KVC_BUF_RK_SCALE, KVC_BUF_RV_CODES, KVC_BUF_RV_SCALE,
  KVC_BUF_K_DENSE, KVC_BUF_V_DENSE, KVC_BUF_BK, KVC_BUF_BV,
  KVC_BUF_SIGNS_K, KVC_BUF_SIGNS_V, KVC_BUF_PAGE_TABLE,
  KVC_BUF_OFFSET_K, KVC_BUF_OFFSET_V, KVC_BUF_RANK_K, KVC_BUF_RANK_V,
  KVC_NBUF
};

/* Validate a description and create an immutable layout handle.  Host only.
 * Defines the stored format of the pages' compressed caches: a low-rank latent
 * times a factor ("BELT Connects KV-Cache Compression ...", section 3),
 * optionally quantized per group (BellowsKV page, "Worked Example: Why the
 * Latent Quantizes Flat"), with keys pre-RoPE ("JoLT: Near-Lossless KV Cache
 * Compression", "Key findings"), a rotated low-bit residual ("A JoLT for the KV
 * cache ...", "Abstract (arXiv)"), a block-shared latent (BellowsKV page,
 * "Share the Input, Not the Cache") or a per-token rank ("VarRate ...",
 * "Summary").  desc is read, not kept; *out receives a handle the caller
 * releases with kvc_destroy_layout.
 * Errors: KVC_EINVAL (NULL, non-positive or inconsistent sizes),
 * KVC_EUNSUPPORTED (e.g. resid_bits > 0 with head_dim != 128, rope with a
 * kind other than LOWRANK, a VARRATE max rank other than 64). */
kvc_status kvc_create_layout(const kvc_layout_desc* desc, kvc_layout** out);

/* Release a handle (NULL is ignored).  No counterpart on the pages. */
void kvc_destroy_layout(kvc_layout* layout);

/* Bytes each cache buffer must have (0 = buffer unused by this layout), in the
 * KVC_BUF_* order; sizes[] is caller-owned host memory of KVC_NBUF entries.
 * These are the closed forms of the stored format -- an INT4 low-rank row costs
 * rank/2 + 4*ceil(rank/group) bytes per component -- the byte arithmetic the
 * BellowsKV page does in "The Cache That Outgrew the Weights" for the dense
 * cache.  Errors: KVC_EINVAL on NULL. */
kvc_status kvc_buffer_sizes(const kvc_layout* layout, size_t sizes[KVC_NBUF]);

/* Compressed bytes a decode step reads for n_tokens tokens (cache rows only;
 * VARRATE: the exact record bytes are data dependent, so the expected size at
 * the average record is returned).  Used for achieved-bandwidth figures: decode
 * re-reads the whole cache every step (BellowsKV page, "The Cache That Outgrew
 * the Weights").  Returns 0 for a NULL layout or n_tokens <= 0. */
size_t kvc_step_bytes(const kvc_layout* layout, int32_t n_tokens);

/* Device workspace bytes kvc_decode_attn needs for contexts up to n_tokens
 * (error word, projected queries, split partials).  No counterpart on the
 * pages (split-T partials are this library's design).  0 for NULL. */
size_t kvc_workspace_bytes(const kvc_layout* layout, int32_t n_tokens);

/* Number of kernel launches one kvc_decode_attn call makes for n_tokens with
 * uniform lengths (per-row lengths may add the query projection). */
int32_t kvc_decode_launches(const kvc_layout* layout, int32_t n_tokens);

/* Append n_new tokens to every batch row: project each new pre-RoPE key and
 * value onto the latent and quantize it into its slot.  Passages: the latent
 * times factor representation ("BELT ...", section 3), the per-group min/max
 * INT4 rule with fp16 scale and zero (BellowsKV page, "Worked Example: Why the
 * Latent Quantizes Flat"), keys compressed before RoPE ("JoLT: Near-Lossless
 * KV Cache Compression", "Key findings"), the rotated low-bit residual of the
 * truncation error ("A JoLT for the KV cache ...", "Abstract (arXiv)"), ragged
 * per-token ranks ("VarRate ...", "Summary").
 *   k_new, v_new: device bf16 [B, Hkv, n_new, d] pre-RoPE keys / values
 *     (DENSE with n_layers > 1: [n_layers, B, Hkv, n_new, d]);
 *     BLOCK_SHARED: k_new = the (key) latent, bf16 [B, n_new, latent_dim]; v_new
 *     the value latent of the same shape when value_bits > 0, else unused.
 *   pos: DEVICE int32 [B], slot of each row's first new token; the tokens go to
 *     slots pos[b] .. pos[b] + n_new - 1.
 *   new_ranks: VARRATE only, DEVICE uint8 [2, B, n_new] (K ranks, then V
 *     ranks), each in {4, 8, 16, 32, 64}; the kernel stores them in rank_k /
 *     rank_v.  The records of row b are written from offset[b][pos[b]], which
 *     must already be valid, and offset[b][pos[b] + 1 ..] are set.
 * All pointers are caller-owned device memory read or written on the stream.
 * Host-detectable errors (NULL, misalignment, n_new < 1 or > max_tokens, a
 * VARRATE call without new_ranks) return before anything is launched.  pos and
 * the ranks live on the device, so the kernels check them: a row whose pos is
 * outside [0, max_tokens - n_new] is skipped (KVC_DEV_BAD_POS), a token with a
 * rank outside the set skips its row from that token on (KVC_DEV_BAD_RANK,
 * offsets stay consistent), a token whose page-table entry is outside
 * [0, n_pages) is skipped (KVC_DEV_BAD_PAGE), and a VARRATE record that would
 * run past its stream is not written (KVC_DEV_BAD_OFFSET); the bits are ORed
 * into cache->status when it is not NULL.  Nothing is written outside the
 * cache buffers.
 * Arithmetic: LOWRANK projects x onto the factor rows (l = x Bk^T, fp32),
 * then per group z = fp16(min), s = fp16((max - min)/15) and each element is
 * coded as the nearest step of s above z (IEEE fp32 division, ties to even,
 * clamped to 0..15; code 0 when s = 0); with a residual, y = Q (x - l_hat Bk)
 * is stored as 2-bit codes clamp(floor(y/s) + 2, 0, 3) with
 * s = fp16(max|y| / 1.5).  BLOCK_SHARED: s = fp16(max|x|/7) per group, code =
 * clamp(round(x/s), -7, 7) + 8.  fp16 latent layouts store l rounded to fp16. */
kvc_status kvc_append(const kvc_layout* layout, const kvc_cache* cache,
                      const void* k_new, const void* v_new, const int32_t* pos,
                      int32_t n_new, const uint8_t* new_ranks, void* stream);

/* Single-token decode attention over tokens [0, len_b) of every row,
 * evaluated directly over the stored factors without materializing dense K/V
 * ("A JoLT for the KV cache ...", "Abstract (arXiv)", FlashJoLT; "BELT ...",
 * section 4 on kernels over the compressed cache): latent-space scores
 * q Bk^T . l_t, or keys reconstructed and rotated per tile when stored
 * pre-RoPE ("JoLT: Near-Lossless KV Cache Compression", "Key findings"); one
 * latent read by all layers of its block (BellowsKV page, "Share the Input,
 * Not the Cache"); per-token ranks ("VarRate ...", "Summary").  The result is
 * softmax(scale * q . k_t) . v_t over the dequantized, reconstructed k, v.
 *   q: device bf16 [B, Hq, d] (already rotated by the caller when rope = 1);
 *      BLOCK_SHARED / layered DENSE: [n_layers, B, Hq, d].
 *   out: device fp32 (or bf16 if out_bf16) with q's shape.
 *   workspace: device, >= kvc_workspace_bytes(layout, cache->n_tokens) bytes,
 *      16-byte aligned, caller-owned; its contents on entry do not matter.
 *      Bytes 0..3 hold the error word afterwards: the call zeroes it (on the
 *      stream) before any kernel that can set it, and a kernel whose bounded
 *      wait gave up ORs KVC_DEV_WAIT_TIMEOUT into it -- the output of such a
 *      call is invalid.  Read it after the stream has completed.
 * Host-detectable errors (NULL, misalignment, n_tokens beyond max_tokens, a
 * small workspace, missing cache buffers) return before anything is enqueued.
 * Launches kvc_decode_launches() kernels: a query projection (where the
 * layout needs one and the split kernel does not form it itself), the split-T
 * fused decode over the compressed tiles, and the split combine with the
 * up-projection (on some paths a zeroing of the error word precedes them). */
kvc_status kvc_decode_attn(const kvc_layout* layout, const kvc_cache* cache,
                           const void* q, void* out, void* workspace,
                           size_t ws_bytes, void* stream);

/* Same as kvc_decode_attn, and records the CUDA events ev_begin / ev_end
 * (cudaEvent_t as void*, may be NULL) on the stream immediately before and
 * after the split-T decode kernel, so that its duration can be measured. */
kvc_status kvc_decode_attn_timed(const kvc_layout* layout, const kvc_cache* cache,
                                 const void* q, void* out, void* workspace,
                                 size_t ws_bytes, void* stream,
                                 void* ev_begin, void* ev_end);

/* Bytes of the library's built-in decode scratch area (see below). */
#define KVC_STATIC_SCRATCH_BYTES (4u << 20)

/* Decode without a caller-provided workspace.  This entry point has no
 * counterpart on the pages; it exists for callers that cannot allocate device
 * memory themselves -- code embedded in a host framework that owns every
 * device allocation and does not expose an allocator, or a latency-critical
 * serving loop that must not call cudaMalloc (which can synchronize the
 * device).  It allocates nothing: its scratch is a file-scope device array of
 * KVC_STATIC_SCRATCH_BYTES bytes that every GPU loading the library keeps
 * until the process exits.  The caller still passes the cache, q and out, as
 * for kvc_decode_attn, which this call runs with that array as the workspace.
 *   - Layouts whose kvc_workspace_bytes(layout, cache->n_tokens) exceeds
 *     KVC_STATIC_SCRATCH_BYTES are rejected with KVC_EWORKSPACE (nothing runs).
 *     Every other host-detectable error is reported as by kvc_decode_attn,
 *     also before anything is enqueued.
 *   - The first call on a device looks up the array's device address on the
 *     current device (once per device, with that device current); make that
 *     first call before any stream capture.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind; what must start at zero (the error word) is cleared on the
 *     stream before the kernels that can set it.  Calls that overlap on the
 *     GPU (other streams, other threads) race on the array: serialize them. */
kvc_status kvc_decode_attn_static(const kvc_layout* layout, const kvc_cache* cache,
                                  const void* q, void* out, void* stream);

/* Error word of the built-in scratch area on the current device (the
 * workspace error word of the last kvc_decode_attn_static call, see
 * kvc_decode_attn): enqueues a 4-byte copy of it to dst (device memory or
 * pinned host memory, caller-owned) on the stream; read dst after the stream
 * has completed.  No counterpart on the pages.  Errors: KVC_EINVAL on NULL dst,
 * KVC_ECUDA if the copy cannot be enqueued. */
kvc_status kvc_static_error_word(uint32_t* dst, void* stream);

/* ---- Bulk prefill compression: per-head factors by randomized SVD -------
 * "A JoLT for the KV cache ...", "Abstract (arXiv)": FlashJoLT replaces the
 * exact token-mode SVD with a randomized approximation; "JoLT: Near-Lossless
 * KV Cache Compression", "How JoLT works" and "Key findings": only the token
 * and feature axes are truncated (a factor per KV head), keys before RoPE.
 * The factor of KV head h (rank x 128) spans the top right singular subspace
 * of the head's token-major prefill matrix (the n_rows first tokens of every
 * batch row); kvc_append with n_new = the prefill length then projects and
 * quantizes every token onto it.  Method: the randomized range finder with
 * the caller's Gaussian test matrix omega and power_iters power iterations,
 * then the exact SVD of the small projection -- computed through the Gram
 * matrix X^T X (one tensor-core pass over x, fp32 accumulation) and fp64 dense
 * algebra on it (orthonormalisation, Cholesky, Jacobi eigensolver).  Factor
 * rows come largest singular value first, each scaled by +-1 so that its entry
 * of largest magnitude is positive, and are stored as fp16.  No call
 * synchronizes; nothing is allocated. */

/* Device workspace bytes kvc_fit_factors needs for n_kv_heads heads. */
size_t kvc_fit_workspace_bytes(int32_t n_kv_heads);

/* x: device bf16 [batch, n_kv_heads, capacity, head_dim] prefill keys (pre-RoPE)
 *   or values (the layout kvc_append reads with n_new = capacity);
 * omega: device fp32 [n_kv_heads, head_dim, k] test matrices (N(0,1) draws);
 * k: sketch width, even, 2..96 (rank + oversampling); rank <= k;
 * factor: device fp16 [n_kv_heads, rank, head_dim] (the layout's bk / bv);
 * sigma2: device fp32 [n_kv_heads, k] or NULL: the squared singular values of
 *   the projection, largest first (the spectrum kvc_rank_bit_tables takes);
 * workspace: device, >= kvc_fit_workspace_bytes(n_kv_heads), caller-owned.
 * All pointers 16-byte aligned.  Errors (before anything is enqueued):
 * KVC_EINVAL (NULL, sizes), KVC_EUNSUPPORTED (head_dim != 128), KVC_EALIGN,
 * KVC_EWORKSPACE; KVC_ECUDA if a launch fails. */
kvc_status kvc_fit_factors(const void* x, int32_t batch, int32_t n_kv_heads, int32_t capacity,
                           int32_t n_rows, int32_t head_dim, const float* omega, int32_t k,
                           int32_t rank, int32_t power_iters, void* factor, float* sigma2,
                           void* workspace, size_t ws_bytes, void* stream);

/* ---- Token importance: query salience, ranks by salience, block eviction --
 * "VarRate: Training-Free Variable-Rate KV Cache Compression for Long-Context
 * LLMs", "Summary" / "Method": every token gets a low-rank budget chosen by its
 * query salience and keeps a nonzero rank.  "BellowsKV Architecture ...",
 * "Three Measurements, Three Operators": the layers of a block agree on which
 * tokens matter, so one importance decision per block, from all n layers'
 * scores, is applied once to the shared latent.  Readings (the pages give no
 * formulas): the salience of token t is the attention probability it receives
 * from a window of queries, summed over the window and over all query heads;
 * ranks go by salience quantiles; a block's importance is the sum of its
 * layers' saliences and the decision keeps the `keep` most important tokens.
 * Ties in the ordering go to the lower position. */

/* Device workspace bytes kvc_window_salience needs. */
size_t kvc_salience_workspace_bytes(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                    int32_t window, int32_t n_tokens);

/* salience[b][t] = sum over query heads h and window queries w of
 * softmax_t(scale * q[b][h][w] . keys[b][h / G][t]) over t < n_tokens.
 *   q_window: device bf16 [batch, n_q_heads, window, 128] (as the attention
 *     sees them, i.e. rotated when the model uses RoPE);
 *   keys: device bf16 [batch, n_kv_heads, capacity, 128] prefill keys (rotated);
 *   salience: device fp32 [batch, n_tokens] (written); softmax_scale 0 means
 *     1/sqrt(128).  (n_q_heads / n_kv_heads) * window <= 128.
 * Two tensor-core passes over the keys (bf16 in, fp32 accumulate).  Errors
 * before anything is enqueued: KVC_EINVAL, KVC_EUNSUPPORTED (head_dim, too
 * many window rows), KVC_EALIGN, KVC_EWORKSPACE. */
kvc_status kvc_window_salience(const void* q_window, const void* keys, int32_t batch,
                               int32_t n_q_heads, int32_t n_kv_heads, int32_t window,
                               int32_t capacity, int32_t n_tokens, int32_t head_dim,
                               float softmax_scale, float* salience, void* workspace,
                               size_t ws_bytes, void* stream);

/* Ranks by salience: in each batch row, tokens in descending salience (ties:
 * lower position first) take rung_ranks[0] for the first rung_counts[0]
 * tokens, rung_ranks[1] for the next rung_counts[1], ...; the last rung takes
 * every remaining token, so no token is left without a rank.  Exact ordering
 * (a radix select on 64-bit keys), so the counts are exact.
 *   salience: device fp32 [batch, n_tokens];
 *   rung_ranks: host int32 [n_rungs] in {4, 8, 16, 32, 64} (1..8 rungs);
 *   rung_counts: host int32 [n_rungs - 1];
 *   ranks: device uint8 [2, batch, n_tokens] (written): K ranks then V ranks
 *     (equal), the new_ranks layout of kvc_append. */
kvc_status kvc_ranks_by_salience(const float* salience, int32_t batch, int32_t n_tokens,
                                 int32_t n_rungs, const int32_t* rung_ranks,
                                 const int32_t* rung_counts, uint8_t* ranks, void* stream);

/* One keep decision per block: importance[b][t] = sum over the block's layers
 * of salience_layers[l][b][t]; kept[b] (device int32 [batch, keep], written)
 * lists the positions of the `keep` most important tokens of row b in
 * ascending order.  salience_layers: device fp32 [n_layers, batch, n_tokens];
 * importance: device fp32 [batch, n_tokens] (written).  keep <= n_tokens. */
kvc_status kvc_block_keep(const float* salience_layers, int32_t n_layers, int32_t batch,
                          int32_t n_tokens, int32_t keep, float* importance, int32_t* kept,
                          void* stream);

/* Apply a keep decision once to a block-shared latent: row i of batch row b of
 * dst receives row kept[b][i] of src (codes and scales), i < keep.  Both
 * layouts are KVC_BLOCK_SHARED with the same batch and latent format; dst's
 * capacity holds keep tokens.  The caller sets dst->n_tokens = keep afterwards. */
kvc_status kvc_block_compact(const kvc_layout* src_layout, const kvc_cache* src,
                             const kvc_layout* dst_layout, const kvc_cache* dst,
                             const int32_t* kept, int32_t keep, void* stream);

/* ---- Joint rank / residual-bit allocation (host only) -------------------
 * "JoLT: Near-Lossless KV Cache Compression", section "How JoLT works": the
 * layers are grouped, the keys and the values of each group are separate
 * cells, and one Lagrangian multiplier picks every cell's ranks and residual
 * bit-width under a shared byte budget; "A JoLT for the KV cache ...",
 * "Abstract (arXiv)": a single Lagrangian dual under a global byte
 * constraint.  The chosen (rank, bits) of a cell become the rank_k / rank_v and
 * resid_bits of the layout that stores it. */
#define KVC_MAX_RESID_BITS 8

typedef struct {
  int32_t rank;   /* latent rank of the option (1..spec_len)                  */
  int32_t bits;   /* residual bits per coordinate, 0 = no residual (0..8)     */
} kvc_rank_bits;

/* Byte and distortion tables of every (cell, option), host arrays
 * [n_cells, n_options] written by the call.  Per cell: spectra
 * [n_cells, spec_len] squared singular values of its (rows x head_dim) data,
 * descending; rows[c] stored token rows, heads[c] factors (one per KV head).
 *   bytes(r, b) = rows * (ceil(r * latent_bits / 8) + 4 * ceil(r / group)
 *                 [+ head_dim * b / 8 + 2 when b > 0])
 *                 + heads * r * head_dim * 2 [+ heads * head_dim when b > 0]
 *   distortion(r, b) = eta_latent * (sum of the first r squared singular
 *                 values) + eta_resid[b] * (sum of the rest)
 * (latent_bits 16: no scale/zero bytes).  eta_resid is indexed by the bit
 * width (entries 0..KVC_MAX_RESID_BITS; eta_resid[0] = 1 means the truncated
 * tail is lost).  The distortion model is this library's reading: the pages
 * state the allocation, not the error model.  Errors: KVC_EINVAL (NULL,
 * empty sizes, an option outside the spectrum or the bit range). */
kvc_status kvc_rank_bit_tables(int32_t n_cells, int32_t spec_len, const double* spectra,
                               const int64_t* rows, const int32_t* heads, int32_t n_options,
                               const kvc_rank_bits* options, int32_t head_dim,
                               int32_t latent_bits, int32_t group, double eta_latent,
                               const double* eta_resid, double* bytes, double* distortion);

/* One Lagrangian multiplier for all cells: each cell takes the option that
 * minimises distortion + lambda * bytes (ties: fewer bytes, then the earlier
 * option), and lambda is the smallest of the pairwise break points
 * (D_a - D_b) / (B_b - B_a) (or 0) at which the total bytes fit the budget --
 * found exactly, by a binary search over the sorted break points.  choice
 * [n_cells] (host) receives the option index of every cell, *lambda (may be
 * NULL) the multiplier.  Among all allocations that use no more bytes, the
 * result has the least total distortion.  Errors: KVC_EINVAL (NULL, empty or
 * non-finite tables), KVC_ECAPACITY (even the cheapest options exceed the
 * budget). */
kvc_status kvc_allocate_rank_bits(int32_t n_cells, int32_t n_options, const double* bytes,
                                  const double* distortion, double budget, int32_t* choice,
                                  double* lambda);

/* Test switch (per calling thread, off by default): while on, decode calls
 * whose split kernel has bounded waits (the tcgen05 pre-RoPE kernel, the
 * block-shared tcgen05 kernel) enqueue that kernel without its tile copies or
 * dequantisation, so its waits run out after their limit
 * (0.5 s), it sets KVC_DEV_WAIT_TIMEOUT in the workspace error word and exits
 * cleanly; the output of such a call is invalid.  Used to test that a wait
 * that gives up is reported and leaves the context usable.  No counterpart on
 * the pages. */
void kvc_test_skip_tile_copies(int32_t on);

/* Kernel choice for pre-RoPE INT4 layouts (per calling thread): 0 (default)
 * and 1 run the warp-level kernel (reconstruction on mma.sync, fp32
 * accumulate; the faster of the two on the benchmark layout as measured), 2
 * the warpgroup kernel with the reconstruction on tcgen05 (fp32 accumulator in
 * TMEM) where the layout allows it.  Both compute the same decode; the switch
 * exists so that either can be tested and timed.  No counterpart on the
 * pages. */
void kvc_select_rope_kernel(int32_t which);

/* Kernel choice for the variable-rate layout with 8 KV heads x 4 query heads
 * and uniform lengths (per calling thread): 0 (default) runs the
 * lane-per-(KV head, query head) kernel on CUDA cores (the faster of the two
 * as measured), 1 the tensor-core kernel (scores and values on mma.sync at the
 * full rank, codes beyond a token's rank masked).  Both compute the same
 * decode (VarRate "Method"); the switch exists so that either can be tested
 * and timed.  No counterpart on the pages. */
void kvc_select_varrate_kernel(int32_t which);

/* Thread-local description of the last error on this thread ("" if none). */
const char* kvc_last_error(void);

/* Library version string. */
const char* kvc_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVC_H_ */
