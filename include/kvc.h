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
 *     Latent Quantizes Flat" (function qerr);
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
 *     device, except that kvc_append copies host-side VARRATE ranks with
 *     cudaMemcpyAsync from pageable memory (see kvc_append).
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
 *   token, INT4 symmetric (x = (code - 8) * scale) with one fp16 scale per
 *   group_size values; per-layer fp16 up-projections W_k, W_v
 *   [n_layers, latent_dim, n_kv_heads * head_dim].
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
  int32_t latent_dim;     /* BLOCK_SHARED latent width (512)                  */
  int32_t rope;           /* 0 or 1 (LOWRANK)                                 */
  int32_t resid_bits;     /* 0 or 2 (LOWRANK, head_dim 128)                   */
  int32_t page_size;      /* 0 (contiguous) or 16 (LOWRANK)                   */
  int32_t n_pages;        /* physical pages in the pool when paged            */
  int32_t out_bf16;       /* 0: fp32 output, 1: bf16 output                   */
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
 * KVC_BLOCK_SHARED: lk_codes uint8 [B, max_tokens, latent_dim/2],
 *   lk_sz fp16 [B, max_tokens, latent_dim/group_size]; bk = W_k, bv = W_v.
 * KVC_DENSE_BF16: k_dense, v_dense bf16 [n_layers, B, Hkv, max_tokens, d].
 * n_tokens: tokens 0..n_tokens-1 of every row are attended.  seq_lens
 *   (optional, device int32 [B]) gives per-row lengths; values are clamped to
 *   [0, n_tokens].  A row of length 0 produces a zero output.
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
  int32_t _reserved;
} kvc_cache;

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
 * Errors: KVC_EINVAL (NULL, non-positive or inconsistent sizes),
 * KVC_EUNSUPPORTED (e.g. resid_bits > 0 with head_dim != 128, rope with a
 * kind other than LOWRANK, a VARRATE max rank other than 64). */
kvc_status kvc_create_layout(const kvc_layout_desc* desc, kvc_layout** out);

/* Release a handle (NULL is ignored). */
void kvc_destroy_layout(kvc_layout* layout);

/* Bytes each cache buffer must have (0 = buffer unused by this layout), in the
 * KVC_BUF_* order.  These are the closed forms of the stored format: e.g. an
 * INT4 low-rank row costs rank/2 + 4*ceil(rank/group) bytes per component. */
kvc_status kvc_buffer_sizes(const kvc_layout* layout, size_t sizes[KVC_NBUF]);

/* Compressed bytes a decode step reads for n_tokens tokens (cache rows only,
 * VARRATE: the exact record bytes are data dependent, so the expected size at
 * the average record is returned).  Used for achieved-bandwidth figures. */
size_t kvc_step_bytes(const kvc_layout* layout, int32_t n_tokens);

/* Device workspace bytes kvc_decode_attn needs for contexts up to n_tokens. */
size_t kvc_workspace_bytes(const kvc_layout* layout, int32_t n_tokens);

/* Number of kernel launches one kvc_decode_attn call makes for n_tokens. */
int32_t kvc_decode_launches(const kvc_layout* layout, int32_t n_tokens);

/* Append n_new tokens to every batch row.
 *   k_new, v_new: device bf16 [B, Hkv, n_new, d] pre-RoPE keys / values
 *     (DENSE with n_layers > 1: [n_layers, B, Hkv, n_new, d]);
 *     BLOCK_SHARED: k_new = the latent, bf16 [B, n_new, latent_dim]; v_new unused.
 *   pos: HOST int32 [B], slot of each row's first new token; the tokens go to
 *     slots pos[b] .. pos[b] + n_new - 1 (KVC_ECAPACITY beyond max_tokens).
 *   new_ranks: VARRATE only, HOST uint8 [2, B, n_new] (K ranks, then V ranks),
 *     each in {4, 8, 16, 32, 64}; they are copied into rank_k / rank_v with
 *     cudaMemcpyAsync (pageable source: the call returns once they are
 *     staged).  The records of row b are written from offset[b][pos[b]], which
 *     must already be valid, and offset[b][pos[b] + 1 ..] are set.
 * LOWRANK append projects x onto the factor rows (l = x Bk^T), quantizes l per
 * group (codes = clamp(round_half_even((l - z) / s), 0, 15), s = fp16((max -
 * min)/15), z = fp16(min)); with a residual, y = Q (x - l_hat Bk) is stored as
 * 2-bit codes clamp(floor(y/s) + 2, 0, 3) with s = fp16(max|y| / 1.5).
 * BLOCK_SHARED: s = fp16(max|x|/7) per group, code = clamp(round(x/s),-7,7)+8.
 * fp16 latent layouts store l rounded to fp16. */
kvc_status kvc_append(const kvc_layout* layout, const kvc_cache* cache,
                      const void* k_new, const void* v_new, const int32_t* pos,
                      int32_t n_new, const uint8_t* new_ranks, void* stream);

/* Single-token decode attention over tokens [0, len_b) of every row.
 *   q: device bf16 [B, Hq, d] (already rotated by the caller when rope = 1);
 *      BLOCK_SHARED / layered DENSE: [n_layers, B, Hq, d].
 *   out: device fp32 (or bf16 if out_bf16) with q's shape.
 *   workspace: device, >= kvc_workspace_bytes(layout, cache->n_tokens) bytes;
 *      its contents on entry do not matter.
 * Launches kvc_decode_launches() kernels: a query projection, the split-T
 * fused decode over the compressed tiles, and the split combine with the
 * up-projection. */
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
 *   - The first call on a device looks up the array's device address on the
 *     current device (once per device, with that device current); make that
 *     first call before any stream capture.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind; the call clears what must start at zero (the error word) on the
 *     stream before the kernels run.  Calls that overlap on the GPU (other
 *     streams, other threads) race on the array: serialize them. */
kvc_status kvc_decode_attn_static(const kvc_layout* layout, const kvc_cache* cache,
                                  const void* q, void* out, void* stream);

/* Thread-local description of the last error on this thread ("" if none). */
const char* kvc_last_error(void);

/* Library version string. */
const char* kvc_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVC_H_ */
