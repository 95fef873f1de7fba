// Split-T fused decode for low-rank INT4 caches with keys stored before RoPE,
// on the 5th-generation tensor cores (tcgen05, accumulators in TMEM).
//
// Per KV head the cache holds INT4 latents L_k (T x rk) and L_v (T x rv) with
// per-group fp16 (scale, zero); keys are k_t = l_t Bk rotated by RoPE at slot
// t ("JoLT: Near-Lossless KV Cache Compression", Key findings: the method works
// pre-RoPE; the FlashJoLT decode "attends directly on the stored core,
// factors and residual").  For a tile of 128 tokens starting at t0 the kernel
//   1. stages the compressed rows with 1-D bulk copies (no multicast),
//   2. dequantizes L_k into TMEM (the A operand) and L_v into shared memory,
//   3. reconstructs K_hat = L_k Bk on the tensor cores (M = 128 tokens,
//      N = 128 dims, K = rk) into TMEM (fp32),
//   4. applies RoPE as R_t = R_t0 R_delta (delta = row in the tile), writing
//      K'' as packed fp16 back to TMEM (the A operand of the score MMA):
//      each epilogue thread owns one row, so R_delta is a per-thread constant
//      rotation, and R_t0 is folded into the queries (q_rot = R_t0^T q, so
//      q . R_t k = q_rot . R_delta k) -- no per-token sin/cos,
//   5. scores S = K'' q_rot^T on the tensor cores with K'' read from TMEM,
//   6. runs an online softmax with a lazily raised reference maximum,
//   7. accumulates acc^T += L_v^T P in latent space on the tensor cores, with
//      a constant-one row so that the same MMA also sums P (the softmax
//      denominator),
// and writes per-(segment, query head) partials (acc, m, l) that the split
// combine merges and up-projects by Bv once per head.
//
// The grid is persistent: the tiles of all (batch row, KV head) units are cut
// into equal contiguous ranges, one per CTA, so every SM streams the same
// number of bytes; a range may cross a unit boundary (two partials).
//
// Warp roles (448 threads, one CTA per SM):
//   warp 0      bulk-copy producer (6-stage ring of compressed tiles)
//   warp 1      TMEM allocation + MMA issue (one lane, non-blocking scheduler)
//   warps 2-9   epilogue: two groups of four warps work on the same tile;
//               group h rotates RoPE pairs 32h..32h+31 and owns query heads
//               2h, 2h+1 (their scores, softmax state, P columns, partials).
//               Software-pipelined: RoPE of tile t, then softmax of tile t-1.
//   warps 10-13 dequantization (thread = row)
// Buffer rings: compressed stages (6), dequantized operands (4), reconstructed
// keys and rotated keys in TMEM (2 each), scores (2), P and q_rot (2).  Every wait is bounded; on a
// timeout the CTA sets an error bit in the workspace, drains its own bulk
// copies and MMAs, frees TMEM and exits.
#include <math.h>

#include "kvc_device.cuh"
#include "tc_util.cuh"

namespace kvc {
namespace {

using namespace tc;

constexpr int kTile = 128;
constexpr int kStages = 6;
constexpr int kThreads = 448;
constexpr int kWarpProd = 0, kWarpMma = 1, kWarpEpi = 2, kWarpDeq = 10;
constexpr int kD = 128;            // head dim
constexpr int kHalf = 64;          // RoPE pairs
constexpr int kG = 4;              // query heads per KV head
constexpr int kVM = 64;            // M of the value MMA (rank_v + 1 <= 64)
constexpr int kN = 16;             // N of score / value MMAs (4 heads padded)
constexpr int kNB = 4;             // dequantized operand buffers (tile jj uses jj % kNB)

// TMEM columns (512 allocated); a 16-bit accumulator would still take one
// column per value, while a TMEM A operand packs two fp16 per column, so the
// reconstruction stays fp32 and the rotated keys get their own packed buffer
constexpr uint32_t kColALk = 0;    // kNB x 16   recon A (128 x rk fp16, rk <= 32)
constexpr uint32_t kColS = 64;     // 2 x 16     scores (fp32)
constexpr uint32_t kColAcc = 96;   // 16         value accumulator (M = 64 layout)
constexpr uint32_t kColDr = 128;   // 2 x 128    reconstructed keys K_hat (fp32)
constexpr uint32_t kColAK = 384;   // 2 x 64     rotated keys K'' (packed fp16)
constexpr uint32_t kTmemCols = 512;

// Shared memory carve-up (bytes, from a 1024-aligned base)
constexpr int kSmStage = 0;                            // kStages x stage bytes
constexpr int kStageMax = 8192;
constexpr int kSmBk = kSmStage + kStages * kStageMax;   // 8 KB   B of recon (128 x 32)
constexpr int kSmQ = kSmBk + 8192;                     // 2 x 4 KB   B of score (16 x 128)
constexpr int kSmLV = kSmQ + 2 * 4096;                 // kNB x 16 KB A of value (64 x 128)
constexpr int kSmP = kSmLV + kNB * 16384;              // 2 x 4 KB   B of value (128 x 16)
constexpr int kSmBar = kSmP + 2 * 4096;                // barriers + scratch
constexpr int kSmTotal = kSmBar + 1024;
constexpr int kSmAlloc = kSmTotal + 2048;              // > half the SM: one CTA per SM

struct Bars {
  uint64_t full[kStages], empty[kStages];
  uint64_t tile_in[kNB], v_done[kNB];       // per dequantized operand buffer
  uint64_t alk_free[kNB];                   // recon of the buffer's last tile completed
  uint64_t recon_done[2], kq_full[2];       // per reconstructed / rotated key buffer
  uint64_t score_done[2], p_full[2];        // per score / P buffer
  uint64_t acc_free;                        // the accumulator was read at a unit end
  uint64_t epi_sync[2];                     // bounded barrier among a group's 128 threads
  uint64_t mma_drain;                       // last MMAs of the CTA completed
  uint32_t tmem_base;
  int abort;
  int flag[2][3];
  float wmax[2][4][2];
};

struct Work {
  int W, tpu, total;     // tiles per CTA, tiles per unit, all tiles
};

// rank permutation of the nibble extraction: logical k = 8j + 2a + h holds
// physical rank 8j + a + 4h
__host__ __device__ __forceinline__ int perm_rank(int k) {
  const int j = k >> 3, a = (k >> 1) & 3, h = k & 1;
  return 8 * j + a + 4 * h;
}

// 8 INT4 codes (one 32-bit word, ranks 8j..8j+7) -> 4 f16x2 = code * s + z,
// register a holding physical ranks (8j + a, 8j + a + 4).
__device__ __forceinline__ void dequant_word(uint32_t w, __half2 s2, __half2 z2, uint32_t* out) {
  const uint32_t kMagic = 0x64006400u;
  const __half2 k1024 = __halves2half2(__ushort_as_half(0x6400), __ushort_as_half(0x6400));
  const __half2 k16inv = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));
  const __half2 km64 = __halves2half2(__ushort_as_half(0xD400), __ushort_as_half(0xD400));
  const uint32_t w8 = w >> 8;
  uint32_t r[4];
  r[0] = (w & 0x000F000Fu) | kMagic;
  r[1] = (w & 0x00F000F0u) | kMagic;
  r[2] = (w8 & 0x000F000Fu) | kMagic;
  r[3] = (w8 & 0x00F000F0u) | kMagic;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    __half2 v = *reinterpret_cast<__half2*>(&r[a]);
    v = (a & 1) ? __hfma2(v, k16inv, km64) : __hsub2(v, k1024);   // exact integer code
    v = __hfma2(v, s2, z2);
    out[a] = *reinterpret_cast<uint32_t*>(&v);
  }
}

__device__ __forceinline__ void unit_of(const Params& p, const Work& w, int T, int* u, int* jt,
                                        int* nt) {
  *u = T / w.tpu;
  *jt = T % w.tpu;
  *nt = min(kTile, p.n_tokens - *jt * kTile);
}

__global__ void __launch_bounds__(kThreads, 1) rope_tc_kernel(Params p, Work wk, uint32_t* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  Bars& bars = *reinterpret_cast<Bars*>(sm + kSmBar);
  volatile int* abort = &bars.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const int t_first = cta * wk.W;
  const int n_tiles = min(wk.W, wk.total - t_first);
  const int lk_row = p.lk_row, lv_row = p.lv_row, lksz_row = p.lksz_row, lvsz_row = p.lvsz_row;
  const int stage_bytes = kTile * (lk_row + lksz_row + lv_row + lvsz_row);
  const int rv = p.rv;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 4);
    }
    for (int b = 0; b < kNB; ++b) {
      mbar_init(&bars.tile_in[b], 4);
      mbar_init(&bars.v_done[b], 1);
      mbar_init(&bars.alk_free[b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.recon_done[b], 1);
      mbar_init(&bars.kq_full[b], 256);
      mbar_init(&bars.score_done[b], 1);
      mbar_init(&bars.p_full[b], 256);
      mbar_init(&bars.epi_sync[b], 128);
      for (int k = 0; k < 3; ++k) bars.flag[b][k] = 0;
    }
    mbar_init(&bars.acc_free, 256);
    mbar_init(&bars.mma_drain, 1);
    bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&bars.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  // static zeros of the operand buffers (padding heads / rows)
  for (int i = threadIdx.x; i < (2 * 4096 + kNB * 16384 + 2 * 4096) / 16; i += kThreads)
    reinterpret_cast<uint4*>(sm + kSmQ)[i] = make_uint4(0, 0, 0, 0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp == kWarpProd) {
    // ------------------------------------------------------------ producer
    int issued_upto = 0;  // tiles issued
    for (int jj = 0; jj < n_tiles && !*abort; ++jj) {
      const int s = jj % kStages;
      if (!mbar_wait(&bars.empty[s], ((jj / kStages) & 1) ^ 1, abort, err)) break;
      int u, jt, nt;
      unit_of(p, wk, t_first + jj, &u, &jt, &nt);
      const size_t row0 = (size_t)u * p.tmax + (size_t)jt * kTile;
      uint8_t* st = sm + kSmStage + s * kStageMax;
      const uint8_t* src[4] = {p.lk + row0 * lk_row,
                               reinterpret_cast<const uint8_t*>(p.lksz) + row0 * lksz_row,
                               p.lv + row0 * lv_row,
                               reinterpret_cast<const uint8_t*>(p.lvsz) + row0 * lvsz_row};
      const int rowb[4] = {lk_row, lksz_row, lv_row, lvsz_row};
      // bulk copies need 16-byte aligned sources: a unit base u * max_tokens * row
      // is aligned only when max_tokens * row is a multiple of 16
      bool aligned = true;
      for (int c = 0; c < 4; ++c) aligned &= (reinterpret_cast<uintptr_t>(src[c]) & 15u) == 0;
      if (nt == kTile && aligned) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&bars.full[s], stage_bytes);
          int off = 0;
          for (int c = 0; c < 4; ++c) {
            bulk_g2s(st + off, src[c], kTile * rowb[c], &bars.full[s]);
            off += kTile * rowb[c];
          }
        }
      } else {
        // ragged last tile of a unit, or unaligned rows: plain copies of the nt
        // valid rows
        int off = 0;
        for (int c = 0; c < 4; ++c) {
          const int n = nt * rowb[c];
          for (int i = lane; i < n; i += 32) st[off + i] = src[c][i];
          off += kTile * rowb[c];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.full[s]);
      }
      issued_upto = jj + 1;
    }
    // drain: every issued stage must have landed before the CTA may exit
    if (*abort && lane == 0) {
      for (int jj = max(0, issued_upto - kStages); jj < issued_upto; ++jj) {
        volatile int no_abort = 0;
        mbar_wait(&bars.full[jj % kStages], (jj / kStages) & 1, &no_abort, nullptr);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issue
    // Non-blocking scheduler: issue whichever of (value nv, score ns,
    // reconstruction nr) is ready, in tile order within each kind.  recon(nr)
    // overwrites the K_hat buffer of tile nr - 2, which the epilogue has read
    // once score(nr - 2) could be issued.
    if (lane == 0) {
      const uint32_t id_recon = idesc_f16(kTile, kD, 0, 0);
      const uint32_t id_score = idesc_f16(kTile, kN, 0, 0);
      const uint32_t id_val = idesc_f16(kVM, kN, 1, 1);
      const int ksteps_recon = p.rk / 16;
      int nr = 0, ns = 0, nv = 0;
      int v_unit = -1, v_started = 0;
      uint64_t idle_since = 0;
      uint32_t idle = 0;
      while (nv < n_tiles) {
        bool prog = false;
        if (nv < ns && mbar_test(&bars.p_full[nv & 1], (nv >> 1) & 1)) {
          int u, jt, nt;
          unit_of(p, wk, t_first + nv, &u, &jt, &nt);
          const bool first = u != v_unit;
          bool ready = true;
          if (first && v_started > 0) ready = mbar_test(&bars.acc_free, (v_started - 1) & 1);
          if (ready) {
            if (first) v_unit = u, ++v_started;
            const int bd = nv % kNB, pb = nv & 1;
            tc_fence_after();
            for (int kk = 0; kk < kTile / 16; ++kk)
              mma_ss(tmem + kColAcc, smem_desc(sm + kSmLV + bd * 16384 + kk * 256, 128, 2048),
                     smem_desc(sm + kSmP + pb * 4096 + kk * 256, 128, 2048), id_val,
                     (first && kk == 0) ? 0u : 1u);
            tc_commit(&bars.v_done[bd]);
            ++nv;
            prog = true;
          }
        }
        if (ns < nr && mbar_test(&bars.kq_full[ns & 1], (ns >> 1) & 1)) {
          const int sb = ns & 1;
          tc_fence_after();
          for (int kk = 0; kk < kD / 16; ++kk)
            mma_ts(tmem + kColS + sb * 16, tmem + kColAK + sb * 64 + kk * 8,
                   smem_desc(sm + kSmQ + sb * 4096 + kk * 256, 128, 2048), id_score, kk > 0);
          tc_commit(&bars.score_done[sb]);
          ++ns;
          prog = true;
        }
        if (nr < n_tiles && nr - ns < 2 &&
            mbar_test(&bars.tile_in[nr % kNB], (nr / kNB) & 1)) {
          const int kb = nr & 1, bd = nr % kNB;
          tc_fence_after();
          for (int kk = 0; kk < ksteps_recon; ++kk)
            mma_ts(tmem + kColDr + kb * 128, tmem + kColALk + bd * 16 + kk * 8,
                   smem_desc(sm + kSmBk + kk * 256, 128, 512), id_recon, kk > 0);
          tc_commit(&bars.recon_done[kb]);
          tc_commit(&bars.alk_free[bd]);
          ++nr;
          prog = true;
        }
        if (prog) {
          idle = 0;
        } else if ((++idle & 255u) == 0) {
          if (*abort) break;
          const uint64_t now = globaltimer();
          if (idle == 256) idle_since = now;
          else if (now - idle_since > kWaitLimitNs) {
            *abort = 1;
            atomicOr(err, kErrTimeout);
            break;
          }
        }
      }
      // every MMA this thread issued must complete before TMEM is released
      tc_commit(&bars.mma_drain);
      volatile int no_abort = 0;
      mbar_wait(&bars.mma_drain, 0, &no_abort, nullptr);
    }
    __syncwarp();
  } else if (warp >= kWarpDeq) {
    // ------------------------------------------------------------ dequantization
    const int q4 = warp & 3;                 // TMEM lane quadrant
    const int row = 32 * q4 + lane;          // token row in the tile
    int cur_u = -1;
    const __half2 one_h2 = __floats2half2_rn(1.f, 0.f);
    for (int jj = 0; jj < n_tiles; ++jj) {
      int u, jt, nt;
      unit_of(p, wk, t_first + jj, &u, &jt, &nt);
      const int bd = jj % kNB, s = jj % kStages;
      if (u != cur_u) {
        if (jj > 0 && !mbar_wait(&bars.alk_free[(jj - 1) % kNB], ((jj - 1) / kNB) & 1, abort, err))
          break;
        // B operand of the reconstruction: N = 128 dims x K = rk (logical ranks),
        // K-major core matrices, logical k holds Bk row perm_rank(k)
        const int kvh = u % p.Hkv;
        const __half* bk = p.bk + (size_t)kvh * p.rk * kD;
        __half* dst = reinterpret_cast<__half*>(sm + kSmBk);
        for (int e = threadIdx.x - 32 * kWarpDeq; e < p.rk * kD; e += 128) {
          const int k = e / kD, n = e % kD;
          dst[((n >> 3) * 512 + (k >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2) / 2] =
              bk[(size_t)perm_rank(k) * kD + n];
        }
        fence_proxy_async_smem();
        cur_u = u;
      }
      if (!mbar_wait(&bars.full[s], (jj / kStages) & 1, abort, err)) break;
      if (jj >= kNB) {
        // recon(jj - kNB) read this A buffer, value(jj - kNB) this L_v buffer
        if (!mbar_wait(&bars.alk_free[bd], ((jj - kNB) / kNB) & 1, abort, err)) break;
        if (!mbar_wait(&bars.v_done[bd], ((jj - kNB) / kNB) & 1, abort, err)) break;
      }
      tc_fence_after();
      const bool valid = row < nt;
      const uint8_t* st = sm + kSmStage + s * kStageMax;
      // ---- keys: rk/8 words -> TMEM columns (A operand of the reconstruction)
      uint32_t ka[16];
      {
        const uint32_t* codes = reinterpret_cast<const uint32_t*>(st + row * lk_row);
        const __half2* sz = reinterpret_cast<const __half2*>(st + kTile * lk_row + row * lksz_row);
        const __half2 sz0 = sz[0];
        const __half2 s2 = __low2half2(sz0), z2 = __high2half2(sz0);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (j < p.rk / 8 && valid) {
            dequant_word(codes[j], s2, z2, ka + 4 * j);
          } else {
            ka[4 * j] = ka[4 * j + 1] = ka[4 * j + 2] = ka[4 * j + 3] = 0u;
          }
        }
      }
      tmem_st16(tmem + ((uint32_t)(32 * q4) << 16) + kColALk + bd * 16, ka);
      // ---- values: rv/8 words -> shared memory (A of the value MMA, MN-major)
      {
        const uint8_t* vbase = st + kTile * (lk_row + lksz_row);
        const uint32_t* codes = reinterpret_cast<const uint32_t*>(vbase + row * lv_row);
        const __half2* sz = reinterpret_cast<const __half2*>(vbase + kTile * lv_row + row * lvsz_row);
        uint8_t* lv = sm + kSmLV + bd * 16384 + (row >> 3) * 128 + (row & 7) * 16;
        for (int j = 0; j < rv / 8; ++j) {
          uint32_t r[4] = {0u, 0u, 0u, 0u};
          if (valid) {
            const __half2 szg = sz[j / 4];          // group of 32 ranks = 4 words
            dequant_word(codes[j], __low2half2(szg), __high2half2(szg), r);
          }
          *reinterpret_cast<uint4*>(lv + j * 2048) = make_uint4(r[0], r[1], r[2], r[3]);
        }
        // the constant-one row (logical rank rv) sums P into the softmax denominator
        const __half2 on = valid ? one_h2 : __floats2half2_rn(0.f, 0.f);
        *reinterpret_cast<uint4*>(lv + (rv / 8) * 2048) =
            make_uint4(*reinterpret_cast<const uint32_t*>(&on), 0u, 0u, 0u);
      }
      tmem_wait_st();
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars.empty[s]);
        mbar_arrive(&bars.tile_in[bd]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int h = (warp - kWarpEpi) >> 2;    // group: RoPE pairs 32h.., heads 2h, 2h+1
    const int ew = (warp - kWarpEpi) & 3;    // warp index within the group
    const int q4 = warp & 3;
    const int row = 32 * q4 + lane;
    const int gtid = ew * 32 + lane;         // 0..127 within the group
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    // RoPE rotation of this row (delta = row) for the group's pairs, as f16x2
    // over consecutive frequencies (i, i + 1), i = 32h + 2k
    uint32_t cs[16], sn[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float c0, s0, c1, s1;
      const int i = 32 * h + 2 * k;
      const double t0 = (double)row * p.rope_f[i], t1 = (double)row * p.rope_f[i + 1];
      sincospif(2.f * (float)(t0 - rint(t0)), &s0, &c0);
      sincospif(2.f * (float)(t1 - rint(t1)), &s1, &c1);
      cs[k] = pack_h2(c0, c1);
      sn[k] = pack_h2(s0, s1);
    }
    // q-side rotation: this thread rotates pair qi of head qh
    const int qi = 32 * h + (gtid & 31), qh = gtid >> 5;
    float qlo = 0.f, qhi = 0.f;
    int rope_u = -1;
    // softmax state of the group's two heads
    float m_ref[2] = {-INFINITY, -INFINITY};
    int sm_u = -1, sm_b = 0, sm_kvh = 0, sm_slot = 0, sm_last = -1;
    const size_t rows_q = (size_t)p.B * p.Hq;
    const int pst = p.vdim + 2;
    uint32_t epi_phase = 0;
    auto epi_sync = [&]() -> bool {
      mbar_arrive(&bars.epi_sync[h]);
      const bool r = mbar_wait(&bars.epi_sync[h], epi_phase & 1, abort, err);
      ++epi_phase;
      return r;
    };
    // the accumulator of the finished unit -> partials of the group's heads
    auto finish_unit = [&](int jj_last) -> bool {
      if (!mbar_wait(&bars.v_done[jj_last % kNB], (jj_last / kNB) & 1, abort, err)) return false;
      tc_fence_after();
      uint32_t r[2];
      tmem_ld2(tmem + lane_base + kColAcc + 2 * h, r);
      tmem_wait_ld();
      reg_fence(r);
      if (lane < 16) {
        const int m = 16 * q4 + lane;          // logical value row
        for (int e = 0; e < 2; ++e) {
          const size_t qr = (size_t)sm_b * p.Hq + sm_kvh * kG + 2 * h + e;
          float* dst = p.part + ((size_t)sm_slot * rows_q + qr) * pst;
          const float v = __uint_as_float(r[e]);
          if (m < rv) dst[perm_rank(m)] = v;
          else if (m == rv) {
            dst[p.vdim] = m_ref[e];
            dst[p.vdim + 1] = v;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars.acc_free);
      return true;
    };

    // ---- stage 1: q_rot and RoPE of the reconstructed keys (in place)
    auto rope_stage = [&](int jj) -> bool {
      int u, jt, nt;
      unit_of(p, wk, t_first + jj, &u, &jt, &nt);
      if (u != rope_u) {
        rope_u = u;
        const __nv_bfloat16* qq =
            p.q + ((size_t)(u / p.Hkv) * p.Hq + (u % p.Hkv) * kG + qh) * kD;
        qlo = bf2f(qq[qi]);
        qhi = bf2f(qq[qi + kHalf]);
      }
      {
        // q_rot = R_t0^T q (B operand of the score MMA); this buffer was last
        // read by score(jj - 2), whose completion the softmax stage of jj - 2 saw
        const double turns = (double)(jt * kTile) * p.rope_f[qi];
        float sa, ca;
        sincospif(2.f * (float)(turns - rint(turns)), &sa, &ca);
        __half* qd = reinterpret_cast<__half*>(sm + kSmQ + (jj & 1) * 4096);
        const float rl = ca * qlo + sa * qhi;
        const float rh = ca * qhi - sa * qlo;
        qd[((qh >> 3) * 2048 + (qi >> 3) * 128 + (qh & 7) * 16 + (qi & 7) * 2) / 2] =
            __float2half_rn(rl);
        const int qj = qi + kHalf;
        qd[((qh >> 3) * 2048 + (qj >> 3) * 128 + (qh & 7) * 16 + (qj & 7) * 2) / 2] =
            __float2half_rn(rh);
      }
      if (!mbar_wait(&bars.recon_done[jj & 1], (jj >> 1) & 1, abort, err)) return false;
      tc_fence_after();
      // K_hat (fp32, column = dim) -> K'' (f16x2, column c = dims 2c, 2c+1).
      // This group rotates the low dims 32h..32h+31 against 64+32h..64+32h+31,
      // in two halves of 16 pairs.
      const uint32_t dr = tmem + lane_base + kColDr + (jj & 1) * 128;
      const uint32_t ak = tmem + lane_base + kColAK + (jj & 1) * 64;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t lo[16], hi[16];
        tmem_ld16(dr + 32 * h + 16 * half, lo);
        tmem_ld16(dr + kHalf + 32 * h + 16 * half, hi);
        tmem_wait_ld();
        reg_fence(lo);
        reg_fence(hi);
        uint32_t xo[8], yo[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const __half2 x = __floats2half2_rn(__uint_as_float(lo[2 * k]), __uint_as_float(lo[2 * k + 1]));
          const __half2 y = __floats2half2_rn(__uint_as_float(hi[2 * k]), __uint_as_float(hi[2 * k + 1]));
          const __half2 C = *reinterpret_cast<const __half2*>(&cs[8 * half + k]);
          const __half2 S = *reinterpret_cast<const __half2*>(&sn[8 * half + k]);
          const __half2 xr = __hfma2(C, x, __hneg2(__hmul2(S, y)));   // k_i cos - k_{i+64} sin
          const __half2 yr = __hfma2(C, y, __hmul2(S, x));            // k_{i+64} cos + k_i sin
          xo[k] = *reinterpret_cast<const uint32_t*>(&xr);
          yo[k] = *reinterpret_cast<const uint32_t*>(&yr);
        }
        tmem_st8(ak + 16 * h + 8 * half, xo);
        tmem_st8(ak + 32 + 16 * h + 8 * half, yo);
      }
      tmem_wait_st();
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(&bars.kq_full[jj & 1]);
      return true;
    };

    // ---- stage 2: scores, online softmax, P
    auto softmax_stage = [&](int jj) -> bool {
      int u, jt, nt;
      unit_of(p, wk, t_first + jj, &u, &jt, &nt);
      if (u != sm_u) {
        if (sm_u >= 0 && !finish_unit(sm_last)) return false;
        sm_u = u;
        sm_b = u / p.Hkv;
        sm_kvh = u % p.Hkv;
        sm_slot = cta - (int)(((long long)u * wk.tpu) / wk.W);
        m_ref[0] = m_ref[1] = -INFINITY;
      }
      const int sb = jj & 1;
      if (!mbar_wait(&bars.score_done[sb], (jj >> 1) & 1, abort, err)) return false;
      tc_fence_after();
      uint32_t sr[2];
      tmem_ld2(tmem + lane_base + kColS + sb * 16 + 2 * h, sr);
      tmem_wait_ld();
      reg_fence(sr);
      const bool valid = row < nt;
      float s2[2];
      bool need = false;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        s2[e] = valid ? __uint_as_float(sr[e]) * p.scale_log2 : -INFINITY;
        need |= s2[e] > m_ref[e] + 8.f;
      }
      // P buffer sb was read by value(jj - 2)
      if (jj >= 2 && !mbar_wait(&bars.v_done[(jj - 2) % kNB], ((jj - 2) / kNB) & 1, abort, err))
        return false;
      // a flag is reset two tiles after its last read (every thread of the
      // group has passed the synchronisation in between)
      const int fl = jj % 3;
      if (gtid == 0) bars.flag[h][(jj + 1) % 3] = 0;
      if (__any_sync(0xffffffffu, need) && lane == 0) atomicOr(&bars.flag[h][fl], 1);
      if (!epi_sync()) return false;
      if (bars.flag[h][fl]) {
        // raise the reference maximum to the tile maximum, rescale acc
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float tm = warp_max(s2[e]);
          if (lane == 0) bars.wmax[h][ew][e] = tm;
        }
        if (!epi_sync()) return false;
        float alpha[2];
        bool any_scale = false;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float mt = fmaxf(fmaxf(bars.wmax[h][0][e], bars.wmax[h][1][e]),
                                 fmaxf(bars.wmax[h][2][e], bars.wmax[h][3][e]));
          const float mn = fmaxf(m_ref[e], mt);
          alpha[e] = (m_ref[e] == -INFINITY) ? 1.f : exp2f(m_ref[e] - mn);
          any_scale |= (m_ref[e] != -INFINITY) && (mn > m_ref[e]);
          m_ref[e] = mn;
        }
        // while m_ref was -inf there is no earlier value MMA of this unit;
        // any_scale is the same in every thread of the group
        if (any_scale) {
          if (!mbar_wait(&bars.v_done[(jj - 1) % kNB], ((jj - 1) / kNB) & 1, abort, err))
            return false;
          tc_fence_after();
          uint32_t r[2];
          tmem_ld2(tmem + lane_base + kColAcc + 2 * h, r);
          tmem_wait_ld();
          reg_fence(r);
          r[0] = __float_as_uint(__uint_as_float(r[0]) * alpha[0]);
          r[1] = __float_as_uint(__uint_as_float(r[1]) * alpha[1]);
          tmem_st2(tmem + lane_base + kColAcc + 2 * h, r);
          tmem_wait_st();
          tc_fence_before();
        }
        if (!epi_sync()) return false;   // wmax is read by everyone before it is reused
      }
      const float p0 = valid ? exp2f(s2[0] - m_ref[0]) : 0.f;
      const float p1 = valid ? exp2f(s2[1] - m_ref[1]) : 0.f;
      *reinterpret_cast<uint32_t*>(sm + kSmP + sb * 4096 + (row >> 3) * 128 + (row & 7) * 16 +
                                   4 * h) = pack_h2(p0, p1);
      fence_proxy_async_smem();
      mbar_arrive(&bars.p_full[sb]);
      sm_last = jj;
      return true;
    };

    bool ok = true;
    for (int jj = 0; jj <= n_tiles && ok; ++jj) {
      if (jj < n_tiles) ok = rope_stage(jj);
      if (ok && jj >= 1) ok = softmax_stage(jj - 1);
    }
    if (ok && sm_u >= 0) finish_unit(sm_last);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool rope_tc_supported(const Params& p) {
  return p.kind == KVC_LOWRANK && p.rope && p.bits == 4 && !p.resid && !p.page &&
         p.d == kD && p.G == kG && (p.rk == 16 || p.rk == 32) && p.g == 32 &&
         p.rv % 8 == 0 && p.rv + 1 <= kVM && !p.seq_lens && p.n_tokens > 0 && p.L == 1 &&
         kTile * (p.lk_row + p.lksz_row + p.lv_row + p.lvsz_row) <= kStageMax;
}

// Persistent partition: grid CTAs of W tiles each; a unit of tpu tiles spans
// at most ceil(tpu / W) + 1 CTAs, each with one partial per unit.
void rope_tc_plan(const Params& p, int* grid, int* W, int* tpu, int* slots) {
  const int t = (p.n_tokens + kTile - 1) / kTile;
  const int units = p.B * p.Hkv;
  const int total = units * t;
  int gr = total < kNumSMs ? total : kNumSMs;
  const int w = (total + gr - 1) / gr;
  gr = (total + w - 1) / w;
  *grid = gr;
  *W = w;
  *tpu = t;
  *slots = (t + w - 1) / w + 1;
}

cudaError_t launch_rope_tc(const Params& p, uint32_t* err, cudaStream_t s) {
  int grid, W, tpu, slots;
  rope_tc_plan(p, &grid, &W, &tpu, &slots);
  Work wk{W, tpu, p.B * p.Hkv * tpu};
  cudaError_t e = cudaFuncSetAttribute(rope_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmAlloc);
  if (e != cudaSuccess) return e;
  static_assert(kSmTotal + 1024 <= kSmAlloc, "shared memory carve-up exceeds the allocation");
  static_assert(sizeof(Bars) <= 1024, "barrier block exceeds its slot");
  rope_tc_kernel<<<grid, kThreads, kSmAlloc, s>>>(p, wk, err);
  return cudaGetLastError();
}

}  // namespace kvc
