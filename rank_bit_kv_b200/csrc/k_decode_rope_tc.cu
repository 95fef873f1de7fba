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
//      N = 128 dims, K = rk) into TMEM,
//   4. applies RoPE as R_t = R_t0 R_delta (delta = row in the tile): each
//      epilogue thread owns one row, so R_delta is a per-thread constant
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
// Warp roles (320 threads, one CTA per SM):
//   warp 0     bulk-copy producer (6-stage ring of compressed tiles)
//   warp 1     TMEM allocation + MMA issue (one elected lane)
//   warps 2-5  epilogue: RoPE, scores, softmax, P, partials (thread = row)
//   warps 6-9  dequantization (thread = row)
// Every wait is bounded; on a timeout the CTA sets an error bit in the
// workspace, drains its own bulk copies, frees TMEM and exits.
#include <math.h>

#include "kvc_device.cuh"
#include "tc_util.cuh"

namespace kvc {
namespace {

using namespace tc;

constexpr int kTile = 128;
constexpr int kStages = 6;
constexpr int kThreads = 320;
constexpr int kWarpProd = 0, kWarpMma = 1, kWarpEpi = 2, kWarpDeq = 6;
constexpr int kD = 128;            // head dim
constexpr int kHalf = 64;          // RoPE pairs
constexpr int kG = 4;              // query heads per KV head
constexpr int kVM = 64;            // M of the value MMA (rank_v + 1 <= 64)
constexpr int kN = 16;             // N of score / value MMAs (4 heads padded)

// TMEM columns (512 allocated)
constexpr uint32_t kColALk = 0;    // 2 x 16  recon A (128 x rk fp16, rk <= 32)
constexpr uint32_t kColS = 32;     // 2 x 16  scores (fp32)
constexpr uint32_t kColAcc = 64;   // 16      value accumulator (M = 64 layout)
constexpr uint32_t kColDr = 128;   // 2 x 128 reconstructed keys (fp32)
constexpr uint32_t kColAK = 384;   // 2 x 64  rotated keys (fp16, A of the score MMA)
constexpr uint32_t kTmemCols = 512;

// Shared memory carve-up (bytes, from a 1024-aligned base)
constexpr int kSmStage = 0;                           // kStages x stage bytes
constexpr int kStageMax = 8192;
constexpr int kSmBk = kSmStage + kStages * kStageMax;  // 8 KB  B of recon (128 x 32)
constexpr int kSmQ = kSmBk + 8192;                    // 2 x 4 KB  B of score (16 x 128)
constexpr int kSmLV = kSmQ + 2 * 4096;                // 2 x 16 KB A of value (64 x 128)
constexpr int kSmP = kSmLV + 2 * 16384;               // 2 x 4 KB  B of value (128 x 16)
constexpr int kSmBar = kSmP + 2 * 4096;               // barriers + scratch
constexpr int kSmTotal = kSmBar + 1024;
constexpr int kSmAlloc = 120 * 1024 + 1024;           // forces one CTA per SM

struct Bars {
  uint64_t full[kStages], empty[kStages];
  uint64_t tile_in[2], recon_done[2], kq_full[2], score_done[2], p_full[2], v_done[2];
  uint64_t acc_free;
  uint64_t epi_sync;     // bounded barrier among the 128 epilogue threads
  uint64_t mma_drain;    // last MMAs of the CTA completed
  uint32_t tmem_base;
  int abort;
  int flag[3];
  float wmax[4][kG];
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
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.tile_in[b], 4);
      mbar_init(&bars.recon_done[b], 1);
      mbar_init(&bars.kq_full[b], 128);
      mbar_init(&bars.score_done[b], 1);
      mbar_init(&bars.p_full[b], 128);
      mbar_init(&bars.v_done[b], 1);
    }
    mbar_init(&bars.acc_free, 128);
    mbar_init(&bars.epi_sync, 128);
    mbar_init(&bars.mma_drain, 1);
    bars.abort = 0;
    bars.flag[0] = bars.flag[1] = bars.flag[2] = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&bars.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  // static zeros of the operand buffers (padding heads / rows)
  for (int i = threadIdx.x; i < (2 * 4096 + 2 * 16384 + 2 * 4096) / 16; i += kThreads)
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
      const uint8_t* src[4] = {p.lk + row0 * lk_row, reinterpret_cast<const uint8_t*>(p.lksz) + row0 * lksz_row,
                               p.lv + row0 * lv_row, reinterpret_cast<const uint8_t*>(p.lvsz) + row0 * lvsz_row};
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
    if (lane == 0) {
      const uint32_t id_recon = idesc_f16(kTile, kD, 0, 0);
      const uint32_t id_score = idesc_f16(kTile, kN, 0, 0);
      const uint32_t id_val = idesc_f16(kVM, kN, 1, 1);
      const int ksteps_recon = p.rk / 16;
      int unit_idx = -1, cur_u = -1;
      auto recon = [&](int jj) -> bool {
        const int b = jj & 1;
        if (!mbar_wait(&bars.tile_in[b], (jj >> 1) & 1, abort, err)) return false;
        tc_fence_after();
        for (int kk = 0; kk < ksteps_recon; ++kk)
          mma_ts(tmem + kColDr + b * 128, tmem + kColALk + b * 16 + kk * 8,
                 smem_desc(sm + kSmBk + kk * 256, 128, 512), id_recon, kk > 0);
        tc_commit(&bars.recon_done[b]);
        return true;
      };
      auto score = [&](int jj) -> bool {
        const int b = jj & 1;
        if (!mbar_wait(&bars.kq_full[b], (jj >> 1) & 1, abort, err)) return false;
        tc_fence_after();
        for (int kk = 0; kk < kD / 16; ++kk)
          mma_ts(tmem + kColS + b * 16, tmem + kColAK + b * 64 + kk * 8,
                 smem_desc(sm + kSmQ + b * 4096 + kk * 256, 128, 2048), id_score, kk > 0);
        tc_commit(&bars.score_done[b]);
        return true;
      };
      auto value = [&](int jj) -> bool {
        const int b = jj & 1;
        if (!mbar_wait(&bars.p_full[b], (jj >> 1) & 1, abort, err)) return false;
        int u, jt, nt;
        unit_of(p, wk, t_first + jj, &u, &jt, &nt);
        bool first = false;
        if (u != cur_u) {
          first = true;
          cur_u = u;
          ++unit_idx;
          if (unit_idx > 0 && !mbar_wait(&bars.acc_free, (unit_idx - 1) & 1, abort, err))
            return false;
        }
        tc_fence_after();
        for (int kk = 0; kk < kTile / 16; ++kk)
          mma_ss(tmem + kColAcc, smem_desc(sm + kSmLV + b * 16384 + kk * 256, 128, 2048),
                 smem_desc(sm + kSmP + b * 4096 + kk * 256, 128, 2048), id_val,
                 (first && kk == 0) ? 0u : 1u);
        tc_commit(&bars.v_done[b]);
        return true;
      };
      bool ok = n_tiles > 0 ? recon(0) : true;
      for (int j = 0; j < n_tiles && ok; ++j) {
        if (j >= 1) ok = value(j - 1);
        if (ok && j + 1 < n_tiles) ok = recon(j + 1);
        if (ok) ok = score(j);
      }
      if (ok && n_tiles > 0) value(n_tiles - 1);
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
      const int b = jj & 1, s = jj % kStages;
      if (u != cur_u) {
        if (jj > 0 && !mbar_wait(&bars.recon_done[(jj - 1) & 1], ((jj - 1) >> 1) & 1, abort, err))
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
      if (jj >= 2) {
        if (!mbar_wait(&bars.recon_done[b], ((jj - 2) >> 1) & 1, abort, err)) break;
        if (!mbar_wait(&bars.v_done[b], ((jj - 2) >> 1) & 1, abort, err)) break;
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
          if (j < p.rk / 8) {
            dequant_word(valid ? codes[j] : 0u, s2, z2, ka + 4 * j);
            if (!valid) ka[4 * j] = ka[4 * j + 1] = ka[4 * j + 2] = ka[4 * j + 3] = 0u;
          } else {
            ka[4 * j] = ka[4 * j + 1] = ka[4 * j + 2] = ka[4 * j + 3] = 0u;
          }
        }
      }
      tmem_st16(tmem + ((uint32_t)(32 * q4) << 16) + kColALk + b * 16, ka);
      // ---- values: rv/8 words -> shared memory (A of the value MMA, MN-major)
      {
        const uint8_t* vbase = st + kTile * (lk_row + lksz_row);
        const uint32_t* codes = reinterpret_cast<const uint32_t*>(vbase + row * lv_row);
        const __half2* sz = reinterpret_cast<const __half2*>(vbase + kTile * lv_row + row * lvsz_row);
        uint8_t* lv = sm + kSmLV + b * 16384 + (row >> 3) * 128 + (row & 7) * 16;
        for (int j = 0; j < rv / 8; ++j) {
          const __half2 szg = sz[j / 4];          // group of 32 ranks = 4 words
          uint32_t r[4];
          dequant_word(valid ? codes[j] : 0u, __low2half2(szg), __high2half2(szg), r);
          if (!valid) r[0] = r[1] = r[2] = r[3] = 0u;
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
        mbar_arrive(&bars.tile_in[b]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;
    const int row = 32 * q4 + lane;
    const int ew = warp - kWarpEpi;           // 0..3 epilogue warp index
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    // RoPE rotation of this row (delta = row) for every pair, as f16x2 over
    // consecutive frequencies (i, i + 1)
    uint32_t cs[32], sn[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      float c0, s0, c1, s1;
      const double t0 = (double)row * p.rope_f[2 * k], t1 = (double)row * p.rope_f[2 * k + 1];
      sincospif(2.f * (float)(t0 - rint(t0)), &s0, &c0);
      sincospif(2.f * (float)(t1 - rint(t1)), &s1, &c1);
      cs[k] = pack_h2(c0, c1);
      sn[k] = pack_h2(s0, s1);
    }
    // queries of the current unit for the q-side rotation: this thread rotates
    // pair i = row % 64 of heads 2 * (row / 64) and 2 * (row / 64) + 1
    const int qi = row & (kHalf - 1), qh0 = 2 * (row >> 6);
    float qlo[2], qhi[2];
    float m_ref[kG];
    int cur_u = -1, unit_idx = -1, cur_b = 0, cur_kvh = 0, cur_slot = 0;
    const size_t rows_q = (size_t)p.B * p.Hq;
    const int pst = p.vdim + 2;

    auto finish_unit = [&](int jj_last) -> bool {
      if (!mbar_wait(&bars.v_done[jj_last & 1], (jj_last >> 1) & 1, abort, err)) return false;
      tc_fence_after();
      uint32_t r[16];
      tmem_ld16(tmem + lane_base + kColAcc, r);
      tmem_wait_ld();
      reg_fence(r);
      if (lane < 16) {
        const int m = 16 * q4 + lane;          // logical value row
        for (int h = 0; h < kG; ++h) {
          const size_t qr = (size_t)cur_b * p.Hq + cur_kvh * kG + h;
          float* dst = p.part + ((size_t)cur_slot * rows_q + qr) * pst;
          const float v = __uint_as_float(r[h]);
          if (m < rv) dst[perm_rank(m)] = v;
          else if (m == rv) {
            dst[p.vdim] = m_ref[h];
            dst[p.vdim + 1] = v;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars.acc_free);
      return true;
    };

    uint32_t epi_phase = 0;
    auto epi_sync = [&]() -> bool {
      mbar_arrive(&bars.epi_sync);
      const bool r = mbar_wait(&bars.epi_sync, epi_phase & 1, abort, err);
      ++epi_phase;
      return r;
    };

    bool ok = true;
    int jj = 0;
    for (; jj < n_tiles && ok; ++jj) {
      int u, jt, nt;
      unit_of(p, wk, t_first + jj, &u, &jt, &nt);
      const int b = jj & 1;
      if (u != cur_u) {
        if (cur_u >= 0 && !(ok = finish_unit(jj - 1))) break;
        cur_u = u;
        ++unit_idx;
        cur_b = u / p.Hkv;
        cur_kvh = u % p.Hkv;
        cur_slot = cta - (int)(((long long)u * wk.tpu) / wk.W);
        const __nv_bfloat16* qq = p.q + ((size_t)cur_b * p.Hq + cur_kvh * kG) * kD;
        for (int h = 0; h < 2; ++h) {
          qlo[h] = bf2f(qq[(qh0 + h) * kD + qi]);
          qhi[h] = bf2f(qq[(qh0 + h) * kD + qi + kHalf]);
        }
#pragma unroll
        for (int h = 0; h < kG; ++h) m_ref[h] = -INFINITY;
      }
      // ---- q_rot = R_t0^T q for this tile (B operand of the score MMA)
      {
        const double turns = (double)(jt * kTile) * p.rope_f[qi];
        float sa, ca;
        sincospif(2.f * (float)(turns - rint(turns)), &sa, &ca);
        __half* qd = reinterpret_cast<__half*>(sm + kSmQ + b * 4096);
        for (int h = 0; h < 2; ++h) {
          const int hh = qh0 + h;
          const float rl = ca * qlo[h] + sa * qhi[h];
          const float rh = ca * qhi[h] - sa * qlo[h];
          qd[((hh >> 3) * 2048 + (qi >> 3) * 128 + (hh & 7) * 16 + (qi & 7) * 2) / 2] =
              __float2half_rn(rl);
          const int qj = qi + kHalf;
          qd[((hh >> 3) * 2048 + (qj >> 3) * 128 + (hh & 7) * 16 + (qj & 7) * 2) / 2] =
              __float2half_rn(rh);
        }
      }
      // ---- RoPE of the reconstructed keys: K'' = R_delta K_hat, into TMEM (fp16)
      if (!(ok = mbar_wait(&bars.recon_done[b], (jj >> 1) & 1, abort, err))) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        // dims 8c..8c+7 (low half) and 64+8c..64+8c+7 (high half): 4 f16x2 each,
        // stored at columns 4c.. and 32+4c.. (column k holds dims 2k, 2k+1)
        uint32_t lo[8], hi[8];
        tmem_ld8(tmem + lane_base + kColDr + b * 128 + 8 * c, lo);
        tmem_ld8(tmem + lane_base + kColDr + b * 128 + kHalf + 8 * c, hi);
        tmem_wait_ld();
        reg_fence(lo);
        reg_fence(hi);
        uint32_t xo[4], yo[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const __half2 x = __floats2half2_rn(__uint_as_float(lo[2 * k]), __uint_as_float(lo[2 * k + 1]));
          const __half2 y = __floats2half2_rn(__uint_as_float(hi[2 * k]), __uint_as_float(hi[2 * k + 1]));
          const __half2 C = *reinterpret_cast<const __half2*>(&cs[4 * c + k]);
          const __half2 S = *reinterpret_cast<const __half2*>(&sn[4 * c + k]);
          const __half2 xr = __hfma2(C, x, __hneg2(__hmul2(S, y)));   // k_i cos - k_{i+64} sin
          const __half2 yr = __hfma2(C, y, __hmul2(S, x));            // k_{i+64} cos + k_i sin
          xo[k] = *reinterpret_cast<const uint32_t*>(&xr);
          yo[k] = *reinterpret_cast<const uint32_t*>(&yr);
        }
        tmem_st4(tmem + lane_base + kColAK + b * 64 + 4 * c, xo);
        tmem_st4(tmem + lane_base + kColAK + b * 64 + 32 + 4 * c, yo);
      }
      tmem_wait_st();
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(&bars.kq_full[b]);

      // ---- scores and the online softmax
      if (!(ok = mbar_wait(&bars.score_done[b], (jj >> 1) & 1, abort, err))) break;
      tc_fence_after();
      uint32_t sr[4];
      tmem_ld4(tmem + lane_base + kColS + b * 16, sr);
      tmem_wait_ld();
      reg_fence(sr);
      const bool valid = row < nt;
      float s2[kG];
      bool need = false;
#pragma unroll
      for (int h = 0; h < kG; ++h) {
        s2[h] = valid ? __uint_as_float(sr[h]) * p.scale_log2 : -INFINITY;
        need |= s2[h] > m_ref[h] + 8.f;
      }
      // a flag is reset two tiles after its last read (every thread has passed
      // the synchronisation of the tile in between)
      const int fl = jj % 3;
      if (threadIdx.x == 32 * kWarpEpi) bars.flag[(jj + 1) % 3] = 0;
      if (__any_sync(0xffffffffu, need) && lane == 0) atomicOr(&bars.flag[fl], 1);
      if (!(ok = epi_sync())) break;
      if (bars.flag[fl]) {
        // raise the reference maximum to the tile maximum, rescale acc
#pragma unroll
        for (int h = 0; h < kG; ++h) {
          const float tm = warp_max(s2[h]);
          if (lane == 0) bars.wmax[ew][h] = tm;
        }
        if (!(ok = epi_sync())) break;
        float alpha[kG];
        bool any_scale = false;
#pragma unroll
        for (int h = 0; h < kG; ++h) {
          const float mt = fmaxf(fmaxf(bars.wmax[0][h], bars.wmax[1][h]),
                                 fmaxf(bars.wmax[2][h], bars.wmax[3][h]));
          const float mn = fmaxf(m_ref[h], mt);
          alpha[h] = (m_ref[h] == -INFINITY) ? 1.f : exp2f(m_ref[h] - mn);
          any_scale |= (m_ref[h] != -INFINITY) && (mn > m_ref[h]);
          m_ref[h] = mn;
        }
        // no earlier value MMA of this unit exists while m_ref was -inf; any_scale
        // is the same in every thread (same wmax, same m_ref)
        if (any_scale) {
          ok = mbar_wait(&bars.v_done[(jj - 1) & 1], ((jj - 1) >> 1) & 1, abort, err);
          if (ok) {
            tc_fence_after();
            uint32_t r[16];
            tmem_ld16(tmem + lane_base + kColAcc, r);
            tmem_wait_ld();
            reg_fence(r);
#pragma unroll
            for (int h = 0; h < kG; ++h) r[h] = __float_as_uint(__uint_as_float(r[h]) * alpha[h]);
            tmem_st16(tmem + lane_base + kColAcc, r);
            tmem_wait_st();
            tc_fence_before();
          }
        }
        if (!epi_sync() || !ok) {   // wmax is read by everyone before it is reused
          ok = false;
          break;
        }
      }
      // ---- P (fp16) into the B operand of the value MMA: row -> 8 bytes
      if (jj >= 2 && !(ok = mbar_wait(&bars.v_done[b], ((jj - 2) >> 1) & 1, abort, err))) break;
      {
        float pv[kG];
#pragma unroll
        for (int h = 0; h < kG; ++h) pv[h] = valid ? exp2f(s2[h] - m_ref[h]) : 0.f;
        uint2 w2 = make_uint2(pack_h2(pv[0], pv[1]), pack_h2(pv[2], pv[3]));
        *reinterpret_cast<uint2*>(sm + kSmP + b * 4096 + (row >> 3) * 128 + (row & 7) * 16) = w2;
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars.p_full[b]);
    }
    if (ok && n_tiles > 0 && cur_u >= 0) finish_unit(n_tiles - 1);
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

// Partial slots a unit spans under the persistent partition.
void rope_tc_plan(const Params& p, int* grid, int* W, int* tpu, int* slots) {
  const int t = (p.n_tokens + kTile - 1) / kTile;
  const int units = p.B * p.Hkv;
  const int total = units * t;
  int g = total < kNumSMs ? total : kNumSMs;
  const int w = (total + g - 1) / g;
  g = (total + w - 1) / w;
  *grid = g;
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
  rope_tc_kernel<<<grid, kThreads, kSmAlloc, s>>>(p, wk, err);
  return cudaGetLastError();
}

}  // namespace kvc
