// Internal declarations shared by the host layer and the kernels of libkvc.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kvc.h"

namespace kvc {

constexpr int kMaxBatch = 256;
constexpr int kNumSMs = 148;          // B200
constexpr int kResidDim = 128;        // rotated-residual width (Hadamard size)

// Everything a kernel needs about the layout, the cache and the call, passed
// by value (kernel parameter space).  Pointers are device pointers.
struct Params {
  // shape
  int kind, B, Hq, Hkv, G, d, L;
  int rk, rv, bits, g, ngk, ngv;
  int vbits;             // block-shared: width of the separate value latent (0 = shared)
  int resid, rope, page, tmax, n_pages;
  int D;                 // block-shared latent width
  int n_tokens;
  const int* seq_lens;
  // compressed rows (bytes per row of each component)
  int lk_row, lv_row, lksz_row, lvsz_row;
  // buffers
  const uint8_t* lk;     // codes (INT4) / fp16 latent / varrate K stream / block latent
  const __half* lksz;    // (scale, zero) pairs / block scales
  const uint8_t* lv;
  const __half* lvsz;
  const uint8_t* rkc;
  const __half* rks;
  const uint8_t* rvc;
  const __half* rvs;
  const __nv_bfloat16* kd;
  const __nv_bfloat16* vd;
  const __half* bk;
  const __half* bv;
  const int8_t* signs_k;
  const int8_t* signs_v;
  const int* page_table;
  const int* off_k;
  const int* off_v;
  const uint8_t* rank_k;
  const uint8_t* rank_v;
  size_t stream_bytes;   // varrate stream bytes per batch row
  // call
  const __nv_bfloat16* q;
  void* out;
  int out_bf16;
  float scale;           // softmax scale
  float scale_log2;      // softmax scale * log2(e)
  // workspace
  float* qt;             // projected queries [L*B*Hq, qdim]
  float* part;           // split partials [S, L*B*Hq, vdim + 2]
  int qdim, vdim;
  int S, split_len;      // splits per unit, tokens per split (multiple of the tile)
  // persistent tensor-core path: contiguous ranges of seg_W tiles per CTA over
  // units of seg_tpu tiles (0 = split partials indexed by split)
  int seg_W, seg_tpu;
  int seg_parts;         // partials written per CTA and unit on that path
  int path;              // split kernel: 0 generic, 1 rope_tc, 2 dense_tc, 3 latent_tc, 4 rope_mma,
                         // 5 varrate_warp, 6 block_mma, 7 rope_wg, 8 block_tc,
                         // 9 varrate_mma
  uint32_t* err;         // error word of the workspace (bounded waits that gave up)
  int test_no_copies;    // test switch: the tcgen05 producer issues no tile copies
  // RoPE: turns per position of frequency pair i, theta^(-2i/d) / (2 pi)
  double rope_f[64];
};

// Tokens per tile of the split kernel, per layout kind (a split is a whole
// number of tiles).
__host__ __device__ inline int split_tile(int kind, int rope) {
  if (kind == KVC_BLOCK_SHARED) return 16;
  return 64;
}

// Queries handled by one CTA of the block-shared split kernel.
constexpr int kBlockQueries = 32;

// Append-specific parameters.
struct AppendParams {
  Params p;
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  int n_new;
  const int* pos;              // device [B]: slot of each row's first new token
  const uint8_t* new_ranks;    // device [2, B, n_new] (VARRATE)
  uint32_t* status;            // optional device word for skipped tokens (KVC_DEV_*)
  uint8_t* lk_w;
  __half* lksz_w;
  uint8_t* lv_w;
  __half* lvsz_w;
  uint8_t* rkc_w;
  __half* rks_w;
  uint8_t* rvc_w;
  __half* rvs_w;
  __nv_bfloat16* kd_w;
  __nv_bfloat16* vd_w;
  int* off_k_w;
  int* off_v_w;
  uint8_t* rank_k_w;
  uint8_t* rank_v_w;
};

// tensor-core decode of pre-RoPE INT4 low-rank caches; every CTA writes one
// partial per epilogue warp and unit it touches
constexpr int kRopeTcParts = 8;
bool rope_tc_supported(const Params& p);
void rope_tc_plan(const Params& p, int* grid, int* W, int* tpu, int* slots);
cudaError_t launch_rope_tc(const Params& p, uint32_t* err, cudaStream_t s);

// warp-level tensor-core decode of dense bf16 caches (the baseline layout)
bool dense_tc_supported(const Params& p);
void dense_tc_plan(const Params& p, int* grid, int* W, int* tpu, int* slots);
int dense_tc_slots(int batch, int n_kv_heads, int n_tokens);
cudaError_t launch_dense_tc(const Params& p, cudaStream_t s);

// warp-level tensor-core decode of INT4 low-rank caches without RoPE (latent-
// space scores), with or without the rotated 2-bit residual, contiguous or paged
bool latent_tc_supported(const Params& p);
void latent_tc_plan(const Params& p, int* grid, int* W, int* tpu, int* slots);
int latent_tc_slots(int batch, int n_kv_heads, int n_tokens);
cudaError_t launch_latent_tc(const Params& p, cudaStream_t s);

// warp-level tensor-core decode of pre-RoPE INT4 low-rank caches (reconstruction,
// rotation and scores on mma.sync)
bool rope_mma_supported(const Params& p);
void rope_mma_plan(const Params& p, int* grid, int* W, int* tpu, int* slots);
int rope_mma_slots(int batch, int n_kv_heads, int n_tokens);
cudaError_t launch_rope_mma(const Params& p, cudaStream_t s);

// pre-RoPE INT4 low-rank caches, warpgroup-autonomous, reconstruction on
// tcgen05 (fp32 TMEM accumulator); four partials per warpgroup and unit
constexpr int kRopeWgParts = 4;
bool rope_wg_supported(const Params& p);
void rope_wg_plan(const Params& p, int* grid, int* W, int* tpu, int* slots);
int rope_wg_slots(int batch, int n_kv_heads, int n_tokens);
cudaError_t launch_rope_wg(const Params& p, cudaStream_t s);

// variable-rate layout, one lane per (KV head, query head)
bool varrate_warp_supported(const Params& p);
void varrate_warp_plan(const Params& p, int* splits, int* split_len);
int varrate_warp_slots(int batch, int n_tokens);
cudaError_t launch_varrate_warp(const Params& p, cudaStream_t s);

// variable-rate layout on warp-level tensor cores, one warp per (KV head, half
// of each 32-token chunk); projects its own queries (selectable)
bool varrate_mma_supported(const Params& p);
void varrate_mma_plan(const Params& p, int* splits, int* split_len);
cudaError_t launch_varrate_mma(const Params& p, cudaStream_t s);

// block-shared latent, 32 absorbed queries per CTA on mma.sync
bool block_mma_supported(const Params& p);
void block_mma_plan(const Params& p, int* splits, int* split_len);
int block_mma_slots(int batch, int n_layers, int n_q_heads, int n_tokens);
cudaError_t launch_block_mma(const Params& p, cudaStream_t s);

// block-shared latent on tcgen05: all 128 absorbed queries of a batch row per
// CTA, one CTA per half of the latent columns
bool block_tc_supported(const Params& p);
void block_tc_plan(const Params& p, int* splits, int* split_len);
int block_tc_slots(int batch, int n_tokens);
cudaError_t launch_block_tc(const Params& p, cudaStream_t s);

// factor fit by randomized SVD (bulk prefill compression)
constexpr int kFitChunks = 64;        // Gram partials (CTAs) per KV head
constexpr int kFitMaxK = 96;          // largest sketch width (rank + oversampling)
constexpr int kFitSweeps = 10;        // Jacobi sweeps of the small eigenproblem
struct FitParams {
  const __nv_bfloat16* x;             // [B, Hkv, cap, 128] prefill keys or values
  int B, Hkv, cap, n_rows;
  const float* omega;                 // [Hkv, 128, k]
  int k, rank, power_iters;
  __half* factor;                     // [Hkv, rank, 128]
  float* sigma2;                      // [Hkv, k] or null
  void* workspace;
};
size_t fit_workspace_bytes(int n_kv_heads);
cudaError_t launch_fit(const FitParams& f, cudaStream_t s);

// token-importance producers (salience, ranks by salience, block keep decision)
constexpr int kSalMaxRows = 128;      // query heads per KV head x window queries
struct SalienceCall {
  const __nv_bfloat16* q;             // [B, Hq, W, 128]
  const __nv_bfloat16* k;             // [B, Hkv, cap, 128]
  int B, Hq, Hkv, W, cap, T;
  float scale;
  float* sal;                         // [B, T]
  void* workspace;
};
struct RankLadder {
  int n;                              // rungs (<= 8)
  int rank[8];                        // rank of each rung, most salient first
  int count[8];                       // tokens of each rung but the last (the last takes the rest)
};
size_t salience_workspace_bytes(int B, int Hq, int Hkv, int W, int T);
cudaError_t launch_salience(const SalienceCall& c, cudaStream_t s);
cudaError_t launch_ranks(const float* part_sal, int Hkv, float* sal, int B, int T,
                         const RankLadder& lad, uint8_t* ranks, cudaStream_t s);
cudaError_t launch_keep(const float* sal_layers, int n_layers, float* importance, int B, int T,
                        int keep, int* kept, cudaStream_t s);
cudaError_t launch_compact(const uint8_t* src_codes, const __half* src_scales, uint8_t* dst_codes,
                           __half* dst_scales, const int* kept, int B, int cap_src, int cap_dst,
                           int keep, int code_bytes, int n_scales, cudaStream_t s);

// Record a status and message for kvc_last_error(); returns st.
kvc_status report_error(kvc_status st, const char* fmt, ...);

// kernel launchers (return the cudaGetLastError of the launch)
cudaError_t launch_qproj(const Params& p, cudaStream_t s);
cudaError_t launch_split(const Params& p, cudaStream_t s);
cudaError_t launch_combine(const Params& p, cudaStream_t s);
cudaError_t launch_append(const AppendParams& a, cudaStream_t s);

// Whether the decode of this layout runs a query projection first.
// (The variable-rate kernels, paths 5 and 9, project their queries themselves.)
__host__ __device__ inline bool needs_qproj(const Params& p) {
  return (p.kind == KVC_VARRATE && p.path != 5 && p.path != 9) || p.kind == KVC_BLOCK_SHARED ||
         (p.kind == KVC_LOWRANK && !p.rope);
}

// Whether the chosen split kernel has bounded waits that can set the
// workspace error word (the call zeroes the word first only then).
__host__ __device__ inline bool path_sets_error_word(const Params& p) {
  // tcgen05 split kernels, and the block-shared combine (bounded mbarrier waits)
  return p.path == 1 || p.path == 7 || p.path == 8 || p.kind == KVC_BLOCK_SHARED;
}

}  // namespace kvc
