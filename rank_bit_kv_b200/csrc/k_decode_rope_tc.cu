// Split-T fused decode for low-rank INT4 caches with keys stored before RoPE.
//
// Per KV head the cache holds INT4 latents L_k (T x rk) and L_v (T x rv) with
// per-group fp16 (scale, zero); keys are k_t = l_t Bk rotated by RoPE at slot
// t ("JoLT: Near-Lossless KV Cache Compression", Key findings: the method works
// pre-RoPE; the FlashJoLT decode "attends directly on the stored core,
// factors and residual").  For a tile of 128 tokens starting at t0 the kernel
//   1. stages the compressed rows with 1-D bulk copies (no multicast),
//   2. dequantizes L_k into TMEM and L_v into shared memory,
//   3. reconstructs K_hat = L_k Bk with one tcgen05 MMA per 16 ranks
//      (M = 128 tokens, N = 128 dims, f16 accumulator in TMEM),
//   4. applies RoPE as R_t = R_t0 R_delta (delta = row in the tile): R_delta is
//      a per-thread constant rotation (each thread always owns the same rows),
//      R_t0 is folded into the queries (q_rot = R_t0^T q, so
//      q . R_t k = q_rot . R_delta k) -- no per-token sin/cos,
//   5. scores S = K'' q_rot^T and accumulates acc^T += L_v^T P with warp-level
//      mma.sync (m16n8k16): these products have N = 4 query heads, and a
//      tcgen05 MMA with M = 128 keeps the tensor pipe busy for about N / 2
//      cycles per K = 16 step but no fewer than ~48 (measured: 48 at N = 64,
//      65 at N = 128, 128 at N = 256), so only the N = 128 reconstruction runs
//      on tcgen05,
//   6. keeps an online softmax per warp with a lazily raised reference
//      maximum (rescaling only when a score exceeds it by 2^8),
// and writes one partial (acc, m, l) per warp and unit that the split combine
// merges and up-projects by Bv once per head.
//
// TMEM -> registers uses the 16x256b shape with 16-bit packing: each warp gets
// its 16 rows of K_hat with four consecutive f16 columns per thread and row,
// which become the A fragments of the score MMA once the k order inside every
// 16-wide step is permuted the same way on the query side (the query
// fragments are stored in that order).
//
// The grid is persistent: the tiles of all (batch row, KV head) units are cut
// into equal contiguous ranges, one per CTA, so every SM streams the same
// number of bytes; a range may cross a unit boundary (a partial per part).
//
// Warp roles (480 threads, one CTA per SM):
//   warp 0      producer: 8-stage ring of compressed tiles, four 1-D bulk
//               copies per tile (no multicast)
//   warp 1      TMEM allocation + tcgen05 reconstruction MMAs (one lane)
//   warps 2-5   dequantization (thread = token row), software-pipelined: the
//               stage words of tile jj + 1 are loaded before tile jj is stored
//   warps 6-13  epilogue: each owns 16 rows of every tile, in its TMEM lane
//               quadrant; iteration jj scores tile jj + 1 and runs the softmax
//               and value product of tile jj
//   warp 14     q_rot of every tile
// Every wait is bounded; on a timeout the CTA sets an error bit in the
// workspace, drains its own bulk copies and MMAs, frees TMEM and exits.
#include <math.h>

#include "kvc_device.cuh"
#include "tc_util.cuh"

namespace kvc {
namespace {

using namespace tc;

constexpr int kTile = 128;
constexpr int kStagesLog2 = 3, kStages = 1 << kStagesLog2;
constexpr int kThreads = 480;
constexpr int kWarpProd = 0, kWarpMma = 1, kWarpDeq = 2, kWarpEpi = 6, kEpiWarps = kRopeTcParts,
              kWarpQrot = 14;
constexpr int kD = 128;            // head dim
constexpr int kHalf = 64;          // RoPE pairs
constexpr int kG = 4;              // query heads per KV head
constexpr int kRvMax = 48;         // value rank handled (3 m16 tiles)
constexpr int kLvStride = 56;      // halves per L_v row in shared memory (48 + pad)
constexpr int kNBLog2 = 3, kNB = 1 << kNBLog2;   // dequantized operand buffers (tile jj uses jj % kNB)

// TMEM columns (512 allocated)
constexpr uint32_t kColALk = 0;    // kNB x 16   recon A (128 x rk fp16, rk <= 32)
constexpr int kNDr = 3;            // K_hat buffers (tile jj uses jj % kNDr)
constexpr uint32_t kColDr = 128;   // kNDr x 128 reconstructed keys K_hat (f16, one per column)
constexpr uint32_t kTmemCols = 512;

// Shared memory carve-up (bytes, from a 1024-aligned base)
constexpr int kSmStage = 0;                              // kStages x stage bytes
constexpr int kStageMax = 8192;
constexpr int kSmBk = kSmStage + kStages * kStageMax;     // 8 KB  B of recon (128 x 32)
constexpr int kLvBytes = kTile * kLvStride * 2;           // 14 KB per buffer
constexpr int kSmLV = kSmBk + 8192;                      // kNB x L_v tile [128][56] fp16
constexpr int kQfBytes = 2048;                           // q_rot fragments of a tile (8 heads, 4..7 zero)
constexpr int kSmQF = kSmLV + kNB * kLvBytes;            // kNB x 2 KB
constexpr int kSmBar = kSmQF + kNB * kQfBytes;           // barriers
constexpr int kSmTotal = kSmBar + 1024;
constexpr int kSmAlloc = kSmTotal + 2048 > 120 * 1024 ? kSmTotal + 2048 : 120 * 1024;

struct Bars {
  uint64_t full[kStages], empty[kStages];
  uint64_t tile_in[kNB];     // L_k in TMEM, L_v and q_rot in shared memory (4 dequant warps)
  uint64_t alk_free[kNB];    // recon of the buffer's last tile completed (tcgen05.commit)
  uint64_t lv_free[kNB];     // every epilogue warp is done with L_v / q_rot of the buffer
  uint64_t recon_done[kNDr]; // K_hat buffer written
  uint64_t dr_free[kNDr];    // every epilogue warp has loaded the K_hat buffer
  uint64_t mma_drain;        // last MMAs of the CTA completed
  uint32_t tmem_base;
  int abort;
};

// slot and phase parity of tile j in a ring of 2^lg buffers
template <int lg>
__device__ __forceinline__ int slot_of(int j) { return j & ((1 << lg) - 1); }
template <int lg>
__device__ __forceinline__ uint32_t phase_of(int j) { return ((uint32_t)j >> lg) & 1u; }
__device__ __forceinline__ int dr_slot(int j) { return (int)((uint32_t)j % kNDr); }
__device__ __forceinline__ uint32_t dr_phase(int j) { return ((uint32_t)j / kNDr) & 1u; }

struct Work {
  int W, tpu, total;     // tiles per CTA, tiles per unit, all tiles
};

// Position of a CTA's tile in its unit, advanced one tile at a time.
struct TileCursor {
  int u, jt, tpu;
  __device__ TileCursor(int t, int tiles_per_unit)
      : u(t / tiles_per_unit), jt(t % tiles_per_unit), tpu(tiles_per_unit) {}
  __device__ void next() {
    if (++jt == tpu) {
      jt = 0;
      ++u;
    }
  }
  __device__ int valid_rows(int n_tokens) const { return min(kTile, n_tokens - jt * kTile); }
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

// Byte offset of the f16 pair q_rot[h][d], q_rot[h][d + 1] (d even) in a
// tile's query-fragment buffer.  Epilogue thread (g = head, c4) reads 64
// contiguous bytes: for every 16-wide k step kk the dims kk*16 + 4*c4 + 0..3
// (b0 = first two, b1 = last two), 16-byte chunks XOR-swizzled so that the
// 8 threads of a load phase hit distinct banks.
__device__ __forceinline__ int qf_offset(int h, int d) {
  const int kk = d >> 4, w = d & 15, c4 = w >> 2, e = w & 3;
  const int blk = h * 4 + c4;
  const int sw = (blk >> 1) & 3;
  return blk * 64 + (((kk >> 1) ^ sw) << 4) + (kk & 1) * 8 + e * 2;
}

template <int RK>
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
      mbar_init(&bars.tile_in[b], 5);
      mbar_init(&bars.alk_free[b], 1);
      mbar_init(&bars.lv_free[b], kEpiWarps);
    }
    for (int b = 0; b < kNDr; ++b) {
      mbar_init(&bars.recon_done[b], 1);
      mbar_init(&bars.dr_free[b], kEpiWarps);
    }
    mbar_init(&bars.mma_drain, 1);
    bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&bars.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  // zero the L_v tiles and query fragments once: the pad columns, ranks >= rv
  // and the padding heads 4..7 stay zero (L_v and the fragments are adjacent)
  static_assert(kSmQF == kSmLV + kNB * kLvBytes, "L_v and query fragments must be adjacent");
  for (int i = threadIdx.x; i < (kNB * kLvBytes + kNB * kQfBytes) / 16; i += kThreads)
    reinterpret_cast<uint4*>(sm + kSmLV)[i] = make_uint4(0, 0, 0, 0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp == kWarpProd) {
    // ------------------------------------------------------------ producer
    // one lane issues the tile's four components as 1-D bulk copies (no
    // multicast) completing on the stage's full barrier
    int issued_upto = 0;  // tiles issued
    TileCursor cur(t_first, wk.tpu);
    // (test switch: with no copies issued, every consumer's bounded wait runs
    // out and the CTA takes its abort path)
    const int n_issue = p.test_no_copies ? 0 : n_tiles;
    for (int jj = 0; jj < n_issue && !*abort; ++jj, cur.next()) {
      const int s = slot_of<kStagesLog2>(jj);
      if (!mbar_wait(&bars.empty[s], phase_of<kStagesLog2>(jj) ^ 1, abort, err)) break;
      const int nt = cur.valid_rows(p.n_tokens);
      const size_t row0 = (size_t)cur.u * p.tmax + (size_t)cur.jt * kTile;
      uint8_t* st = sm + kSmStage + s * kStageMax;
      const uint8_t* src[4] = {p.lk + row0 * lk_row,
                               reinterpret_cast<const uint8_t*>(p.lksz) + row0 * lksz_row,
                               p.lv + row0 * lv_row,
                               reinterpret_cast<const uint8_t*>(p.lvsz) + row0 * lvsz_row};
      const int rowb[4] = {lk_row, lksz_row, lv_row, lvsz_row};
      // bulk copies need 16-byte aligned sources: a unit base u * max_tokens * row
      // is aligned only when max_tokens * row is a multiple of 16
      bool aligned = true;
#pragma unroll
      for (int c = 0; c < 4; ++c) aligned &= (reinterpret_cast<uintptr_t>(src[c]) & 15u) == 0;
      if (nt == kTile && aligned) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&bars.full[s], stage_bytes);
          int off = 0;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            bulk_g2s(st + off, src[c], kTile * rowb[c], &bars.full[s]);
            off += kTile * rowb[c];
          }
        }
      } else {
        // ragged last tile of a unit, or unaligned rows: plain copies of the nt
        // valid rows
        int off = 0;
#pragma unroll
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
        mbar_wait(&bars.full[slot_of<kStagesLog2>(jj)], phase_of<kStagesLog2>(jj), &no_abort, nullptr);
      }
    }
  } else if (warp == kWarpQrot) {
    // ------------------------------------------------------------ q_rot of every tile
    // lane m rotates pairs 2m, 2m + 1.  The angle of pair i at t0 = 128 jt is
    // jt * frac(128 f_i) turns; frac(128 f_i) is held in 32-bit fixed point so
    // that jt * F mod 2^32 is exact.
    uint32_t Fq[2];
    float qv[kG][4];                         // q[h][2m], [2m+1], [2m+64], [2m+65] * scale
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      double x = 128.0 * p.rope_f[(2 * lane + e) & (kHalf - 1)];
      x -= floor(x);
      Fq[e] = (uint32_t)(unsigned long long)llrint(x * 4294967296.0);
    }
#pragma unroll
    for (int h = 0; h < kG; ++h) qv[h][0] = qv[h][1] = qv[h][2] = qv[h][3] = 0.f;
    TileCursor cur(t_first, wk.tpu);
    for (int jj = 0; jj < n_tiles; ++jj, cur.next()) {
      const int bd = slot_of<kNBLog2>(jj);
      if (jj == 0 || cur.jt == 0) {
        const int kvh = cur.u % p.Hkv, b = cur.u / p.Hkv;
        const __nv_bfloat16* qq = p.q + ((size_t)b * p.Hq + kvh * kG) * kD;
#pragma unroll
        for (int h = 0; h < kG; ++h) {
          qv[h][0] = bf2f(qq[h * kD + 2 * lane]) * p.scale_log2;
          qv[h][1] = bf2f(qq[h * kD + 2 * lane + 1]) * p.scale_log2;
          qv[h][2] = bf2f(qq[h * kD + 2 * lane + kHalf]) * p.scale_log2;
          qv[h][3] = bf2f(qq[h * kD + 2 * lane + kHalf + 1]) * p.scale_log2;
        }
      }
      // the epilogue warps are done with this buffer's previous tile
      if (jj >= kNB && !mbar_wait(&bars.lv_free[bd], phase_of<kNBLog2>(jj - kNB), abort, err)) break;
      float ca[2], sa[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int turns = (int)((uint32_t)cur.jt * Fq[e]);      // in 2^-32 turns
        __sincosf((float)turns * 1.4629180792671596e-09f, &sa[e], &ca[e]);   // 2 pi / 2^32
      }
      uint8_t* qf = sm + kSmQF + bd * kQfBytes;
#pragma unroll
      for (int h = 0; h < kG; ++h) {
        const float lo0 = ca[0] * qv[h][0] + sa[0] * qv[h][2];
        const float lo1 = ca[1] * qv[h][1] + sa[1] * qv[h][3];
        const float hi0 = ca[0] * qv[h][2] - sa[0] * qv[h][0];
        const float hi1 = ca[1] * qv[h][3] - sa[1] * qv[h][1];
        *reinterpret_cast<uint32_t*>(qf + qf_offset(h, 2 * lane)) = pack_h2(lo0, lo1);
        *reinterpret_cast<uint32_t*>(qf + qf_offset(h, 2 * lane + kHalf)) = pack_h2(hi0, hi1);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.tile_in[bd]);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ reconstruction MMAs
    if (lane == 0) {
      const uint32_t id_recon = idesc_f16(kTile, kD, 0, 0, /*d_f16=*/1);
      for (int nr = 0; nr < n_tiles; ++nr) {
        const int kb = dr_slot(nr), bd = slot_of<kNBLog2>(nr);
        if (!mbar_wait(&bars.tile_in[bd], phase_of<kNBLog2>(nr), abort, err)) break;
        // the K_hat buffer of tile nr - kNDr has been read by every epilogue warp
        if (nr >= kNDr && !mbar_wait(&bars.dr_free[kb], dr_phase(nr - kNDr), abort, err)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < RK / 16; ++kk)
          mma_ts(tmem + kColDr + kb * 128, tmem + kColALk + bd * 16 + kk * 8,
                 smem_desc(sm + kSmBk + kk * 256, 128, 512), id_recon, kk > 0);
        tc_commit(&bars.recon_done[kb]);
        tc_commit(&bars.alk_free[bd]);
      }
      // every MMA this thread issued must complete before TMEM is released
      tc_commit(&bars.mma_drain);
      volatile int no_abort = 0;
      mbar_wait(&bars.mma_drain, 0, &no_abort, nullptr);
    }
    __syncwarp();
  } else if (warp < kWarpEpi) {
    // ------------------------------------------------------------ dequantization
    // thread = token row.  Software-pipelined: the stage words of tile jj + 1
    // are loaded into registers before tile jj is dequantized and stored.
    const int q4 = warp & 3;                 // TMEM lane quadrant
    const int row = 32 * q4 + lane;          // token row in the tile
    const int dt = threadIdx.x - 32 * kWarpDeq;   // 0..127
    const int nwv = rv / 8;
    // raw words of one tile's row: key codes, key (scale, zero), value codes,
    // value (scale, zero) of both groups
    struct RowWords {
      uint32_t kc[RK / 8], ksz, vc[kRvMax / 8], vsz[2];
    };
    auto load_row = [&](int jj, RowWords& w) {
      const uint8_t* st = sm + kSmStage + slot_of<kStagesLog2>(jj) * kStageMax;
      if constexpr (RK == 32) {
        const uint4 v = *reinterpret_cast<const uint4*>(st + row * (RK / 2));
        w.kc[0] = v.x;
        w.kc[1] = v.y;
        w.kc[2] = v.z;
        w.kc[3] = v.w;
      } else {
        const uint2 v = *reinterpret_cast<const uint2*>(st + row * (RK / 2));
        w.kc[0] = v.x;
        w.kc[1] = v.y;
      }
      w.ksz = *reinterpret_cast<const uint32_t*>(st + kTile * (RK / 2) + row * lksz_row);
      const uint8_t* vbase = st + kTile * (lk_row + lksz_row);
      const uint32_t* codes = reinterpret_cast<const uint32_t*>(vbase + row * lv_row);
      const uint32_t* sz = reinterpret_cast<const uint32_t*>(vbase + kTile * lv_row + row * lvsz_row);
      // words past rv read neighbouring bytes of the stage and are dropped
#pragma unroll
      for (int j = 0; j < kRvMax / 8; ++j) w.vc[j] = codes[j];
      w.vsz[0] = sz[0];
      w.vsz[1] = sz[1];
    };
    RowWords cw, nw;
    bool ok = n_tiles > 0 && mbar_wait(&bars.full[0], 0, abort, err);
    if (ok) load_row(0, cw);
    TileCursor cur(t_first, wk.tpu);
    for (int jj = 0; jj < n_tiles && ok; ++jj, cur.next()) {
      const int nt = cur.valid_rows(p.n_tokens);
      const int bd = slot_of<kNBLog2>(jj), s = slot_of<kStagesLog2>(jj);
      // prefetch the next tile's words (their latency hides behind this tile)
      if (jj + 1 < n_tiles) {
        if (!(ok = mbar_wait(&bars.full[slot_of<kStagesLog2>(jj + 1)], phase_of<kStagesLog2>(jj + 1),
                             abort, err)))
          break;
        load_row(jj + 1, nw);
      }
      if (jj == 0 || cur.jt == 0) {
        // new unit: Bk is rewritten once the previous tile's recon is done
        if (jj > 0 && !(ok = mbar_wait(&bars.alk_free[slot_of<kNBLog2>(jj - 1)],
                                       phase_of<kNBLog2>(jj - 1), abort, err)))
          break;
        const int kvh = cur.u % p.Hkv;
        // B operand of the reconstruction: N = 128 dims x K = rk (logical ranks),
        // K-major core matrices, logical k holds Bk row perm_rank(k)
        const __half* bk = p.bk + (size_t)kvh * RK * kD;
        __half* dst = reinterpret_cast<__half*>(sm + kSmBk);
        for (int e = dt; e < RK * kD; e += 128) {
          const int k = e / kD, n = e % kD;
          dst[((n >> 3) * 512 + (k >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2) / 2] =
              bk[(size_t)perm_rank(k) * kD + n];
        }
        fence_proxy_async_smem();
      }
      if (jj >= kNB) {
        // recon(jj - kNB) read this A buffer; the epilogue warps are done with
        // this L_v buffer
        if (!(ok = mbar_wait(&bars.alk_free[bd], phase_of<kNBLog2>(jj - kNB), abort, err))) break;
        if (!(ok = mbar_wait(&bars.lv_free[bd], phase_of<kNBLog2>(jj - kNB), abort, err))) break;
      }
      tc_fence_after();
      // rows past the end get scale = zero = 0 (bitwise: the stage bytes of
      // such rows are stale and may hold any fp16 pattern), hence zero latents
      const uint32_t vmask = row < nt ? 0xFFFFFFFFu : 0u;
      // ---- keys: rk/8 words -> TMEM columns (A operand of the reconstruction)
      {
        const uint32_t szw = cw.ksz & vmask;
        const __half2 sz0 = *reinterpret_cast<const __half2*>(&szw);
        const __half2 s2 = __low2half2(sz0), z2 = __high2half2(sz0);
        uint32_t ka[RK / 2];
#pragma unroll
        for (int j = 0; j < RK / 8; ++j) dequant_word(cw.kc[j], s2, z2, ka + 4 * j);
        const uint32_t ta = tmem + ((uint32_t)(32 * q4) << 16) + kColALk + bd * 16;
        if constexpr (RK == 32) tmem_st16(ta, ka);
        else tmem_st8(ta, ka);
      }
      // ---- values: rv/8 words -> shared memory rows [token][logical rank]
      {
        uint8_t* lv = sm + kSmLV + bd * kLvBytes + row * (kLvStride * 2);
        const uint32_t gw[2] = {cw.vsz[0] & vmask, cw.vsz[1] & vmask};   // groups of 32 ranks
#pragma unroll
        for (int j = 0; j < kRvMax / 8; ++j) {
          if (j < nwv) {
            const __half2 szg = *reinterpret_cast<const __half2*>(&gw[j < 4 ? 0 : 1]);
            uint32_t r[4];
            dequant_word(cw.vc[j], __low2half2(szg), __high2half2(szg), r);
            *reinterpret_cast<uint4*>(lv + j * 16) = make_uint4(r[0], r[1], r[2], r[3]);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars.empty[s]);       // tile jj's words were consumed above
        mbar_arrive(&bars.tile_in[bd]);
      }
      cw = nw;
    }
  } else {
    // ------------------------------------------------------------ epilogue warps
    const int ew = warp - kWarpEpi;          // partial index of this warp
    const int q4 = warp & 3;                 // this warp's TMEM lane quadrant
    const int m_base = 32 * q4 + 16 * (ew >> 2);   // inside the warp's lane quadrant
    const int g = lane >> 2, c4 = lane & 3;  // fragment row / column group
    const int r0 = m_base + g, r1 = r0 + 8;  // the two rows this thread holds
    const uint32_t taddr0 = tmem + ((uint32_t)m_base << 16);
    // RoPE rotation R_delta of rows r0 and r1 for the pairs this thread holds:
    // dims i = 16 kk + 4 c4 + {0,1} (hf 0) and {2,3} (hf 1), kk = 0..3, against
    // i + 64, as f16x2 over the two dims
    uint32_t cs[4][2][2], sn[4][2][2];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int i = 16 * kk + 4 * c4 + 2 * hf;
          const int delta = rr ? r1 : r0;
          float c0, s0, c1, s1;
          double t0 = (double)delta * p.rope_f[i], t1 = (double)delta * p.rope_f[i + 1];
          t0 -= rint(t0);
          t1 -= rint(t1);
          __sincosf(6.283185307179586f * (float)t0, &s0, &c0);
          __sincosf(6.283185307179586f * (float)t1, &s1, &c1);
          cs[kk][hf][rr] = pack_h2(c0, c1);
          sn[kk][hf][rr] = pack_h2(s0, s1);
        }
    // query-fragment block of this thread (g = head; heads 4..7 are zero)
    const int qblk = g * 4 + c4;
    const int qsw = (qblk >> 1) & 3;
    // ldmatrix row address of this lane in an L_v buffer
    const int lv_off = (m_base + (lane & 7) + ((lane >> 4) << 3)) * (kLvStride * 2) +
                       ((lane >> 3) & 1) * 16;
    // per-warp softmax state for heads 2*c4, 2*c4 + 1 (real heads when c4 < 2)
    float m_ref[2], m_thr[2], l_sum[2];
    float acc[3][4];
    int cur_b = 0, cur_kvh = 0, cur_slot = 0;
    const size_t rows_q = (size_t)p.B * p.Hq;
    const int pst = p.vdim + 2;
    auto reset = [&]() {
      m_ref[0] = m_ref[1] = -INFINITY;
      m_thr[0] = m_thr[1] = -INFINITY;
      l_sum[0] = l_sum[1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < 3; ++mt)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[mt][k] = 0.f;
    };
    // partial of this warp for the finished unit
    auto write_partial = [&]() {
      float l0 = l_sum[0], l1 = l_sum[1];
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o);
      }
      if (c4 < 2) {
        const int slot = cur_slot * kEpiWarps + ew;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const size_t qr = (size_t)cur_b * p.Hq + cur_kvh * kG + 2 * c4 + e;
          float* dst = p.part + ((size_t)slot * rows_q + qr) * pst;
#pragma unroll
          for (int mt = 0; mt < 3; ++mt) {
            const int m0 = 16 * mt + g;
            if (m0 < rv) dst[perm_rank(m0)] = acc[mt][e];
            if (m0 + 8 < rv) dst[perm_rank(m0 + 8)] = acc[mt][2 + e];
          }
          if (g == 0) {
            dst[p.vdim] = m_ref[e];
            dst[p.vdim + 1] = e ? l1 : l0;
          }
        }
      }
    };

    // K_hat of this warp's 16 rows of tile jj (f16, four 32-column loads),
    // issued one iteration ahead so that the TMEM latency hides behind work
    uint32_t klo[2][8], khi[2][8];
    auto issue_k = [&](int jj) -> bool {
      const int kb = dr_slot(jj);
      if (!mbar_wait(&bars.recon_done[kb], dr_phase(jj), abort, err)) return false;
      tc_fence_after();
      const uint32_t dr = taddr0 + kColDr + kb * 128;
      tmem_ld16x256_x2_pack16(dr + 0, klo[0]);
      tmem_ld16x256_x2_pack16(dr + 32, klo[1]);
      tmem_ld16x256_x2_pack16(dr + kHalf, khi[0]);
      tmem_ld16x256_x2_pack16(dr + kHalf + 32, khi[1]);
      return true;
    };

    // K_hat of tile jj is in registers: every epilogue warp releases its buffer
    auto k_ready = [&](int jj) -> bool {
      if (!mbar_wait(&bars.tile_in[slot_of<kNBLog2>(jj)], phase_of<kNBLog2>(jj), abort, err))
        return false;
      tmem_wait_ld();
      reg_fence(klo[0]);
      reg_fence(klo[1]);
      reg_fence(khi[0]);
      reg_fence(khi[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.dr_free[dr_slot(jj)]);
      return true;
    };
    // RoPE in registers, then the score MMA (k steps kk and kk + 4 in two
    // independent accumulator chains); the query fragments of k steps
    // {2h, 2h+1} and {2h+4, 2h+5} sit in 16-byte chunks h and h + 2.  Scores
    // come out in log2 units (the softmax scale is folded into q_rot).
    auto score_tile = [&](int bd, float (&out)[4]) {
      const uint4* qf = reinterpret_cast<const uint4*>(sm + kSmQF + bd * kQfBytes + qblk * 64);
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const uint4 qlo = qf[hh ^ qsw], qhi = qf[(hh + 2) ^ qsw];
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2) {
          const int kk = 2 * hh + k2;
          uint32_t xr[4], yr[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) {          // r: (row r >> 1, dims pair-couple r & 1)
            const __half2 x = *reinterpret_cast<const __half2*>(&klo[hh][4 * k2 + r]);
            const __half2 y = *reinterpret_cast<const __half2*>(&khi[hh][4 * k2 + r]);
            const __half2 C = *reinterpret_cast<const __half2*>(&cs[kk][r & 1][r >> 1]);
            const __half2 S = *reinterpret_cast<const __half2*>(&sn[kk][r & 1][r >> 1]);
            const __half2 xo = __hfma2(C, x, __hneg2(__hmul2(S, y)));   // k_i cos - k_{i+64} sin
            const __half2 yo = __hfma2(C, y, __hmul2(S, x));            // k_{i+64} cos + k_i sin
            xr[r] = *reinterpret_cast<const uint32_t*>(&xo);
            yr[r] = *reinterpret_cast<const uint32_t*>(&yo);
          }
          const uint32_t alo[4] = {xr[0], xr[2], xr[1], xr[3]};
          const uint32_t ahi[4] = {yr[0], yr[2], yr[1], yr[3]};
          mma16816(sa, alo, k2 ? qlo.z : qlo.x, k2 ? qlo.w : qlo.y);
          mma16816(sb, ahi, k2 ? qhi.z : qhi.x, k2 ? qhi.w : qhi.y);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) out[i] = sa[i] + sb[i];
    };

    // Software pipeline: iteration jj scores tile jj + 1 and runs the softmax
    // and value product of tile jj, so the two dependency chains interleave.
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
    bool ok = n_tiles > 0 && issue_k(0) && k_ready(0);
    if (ok) {
      score_tile(0, sc);
      if (n_tiles > 1) ok = issue_k(1);
    }
    TileCursor cur(t_first, wk.tpu);
    for (int jj = 0; jj < n_tiles && ok; ++jj, cur.next()) {
      const int nt = cur.valid_rows(p.n_tokens);
      if (jj == 0 || cur.jt == 0) {
        if (jj > 0) write_partial();
        reset();
        cur_b = cur.u / p.Hkv;
        cur_kvh = cur.u % p.Hkv;
        cur_slot = cta - (int)(((long long)cur.u * wk.tpu) / wk.W);
      }
      const int bd = slot_of<kNBLog2>(jj);
      if (jj + 1 < n_tiles && !(ok = k_ready(jj + 1))) break;
      // ---- score of tile jj + 1 (after the last tile: stale registers, dropped)
      float sn1[4];
      score_tile(slot_of<kNBLog2>(jj + 1), sn1);
      // ---- online softmax of tile jj (rows r0, r1; heads 2c4, 2c4 + 1)
      const bool v0 = r0 < nt, v1 = r1 < nt;     // rows past the end weigh nothing
      const float s0 = v0 ? sc[0] : -INFINITY, s1 = v0 ? sc[1] : -INFINITY;
      const float s2 = v1 ? sc[2] : -INFINITY, s3 = v1 ? sc[3] : -INFINITY;
      const bool need = s0 > m_thr[0] || s2 > m_thr[0] || s1 > m_thr[1] || s3 > m_thr[1];
      float pv[4];
      pv[0] = ex2_approx(s0 - m_ref[0]);
      pv[1] = ex2_approx(s1 - m_ref[1]);
      pv[2] = ex2_approx(s2 - m_ref[0]);
      pv[3] = ex2_approx(s3 - m_ref[1]);
      if (__any_sync(0xffffffffu, need)) {
        float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
        }
        const float n0 = fmaxf(m_ref[0], mx0), n1 = fmaxf(m_ref[1], mx1);
        // a = 2^(m_old - m_new); 0 for a first maximum (m_old = -inf)
        const float a0 = ex2_approx(m_ref[0] - n0), a1 = ex2_approx(m_ref[1] - n1);
        l_sum[0] *= a0;
        l_sum[1] *= a1;
#pragma unroll
        for (int mt = 0; mt < 3; ++mt) {
          acc[mt][0] *= a0;
          acc[mt][2] *= a0;
          acc[mt][1] *= a1;
          acc[mt][3] *= a1;
        }
        m_ref[0] = n0;
        m_ref[1] = n1;
        m_thr[0] = n0 + 8.f;
        m_thr[1] = n1 + 8.f;
        pv[0] = ex2_approx(s0 - n0);
        pv[1] = ex2_approx(s1 - n1);
        pv[2] = ex2_approx(s2 - n0);
        pv[3] = ex2_approx(s3 - n1);
      }
      // masked rows: select, not multiply (-inf - -inf is NaN while no row of
      // this warp has been seen)
      if (!v0) pv[0] = pv[1] = 0.f;
      if (!v1) pv[2] = pv[3] = 0.f;
      l_sum[0] += pv[0] + pv[2];
      l_sum[1] += pv[1] + pv[3];
      // P as the B operand (k = token, n = head): transpose the two 8x8 blocks
      const uint32_t pb0 = movmatrix_trans(pack_h2(pv[0], pv[1]));
      const uint32_t pb1 = movmatrix_trans(pack_h2(pv[2], pv[3]));
      // ---- acc^T (rank x head) += L_v^T (rank x token) P (token x head)
      {
        const uint8_t* lvt = sm + kSmLV + bd * kLvBytes + lv_off;
#pragma unroll
        for (int mt = 0; mt < 3; ++mt) {
          if (16 * mt < rv) {
            uint32_t a[4];
            ldmatrix_x4_trans(a, lvt + 32 * mt);
            mma16816(acc[mt], a, pb0, pb1);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.lv_free[bd]);
      // the K_hat loads of tile jj + 2 fly during the next iteration's waits
      if (jj + 2 < n_tiles && !(ok = issue_k(jj + 2))) break;
#pragma unroll
      for (int i = 0; i < 4; ++i) sc[i] = sn1[i];
    }
    if (ok && n_tiles > 0) write_partial();
    if (!ok) tmem_wait_ld();   // no load of this thread may be in flight at exit
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
         p.rv % 8 == 0 && p.rv <= kRvMax && !p.seq_lens && p.n_tokens > 0 && p.L == 1 &&
         kTile * (p.lk_row + p.lksz_row + p.lv_row + p.lvsz_row) <= kStageMax;
}

// Persistent partition: grid CTAs of W tiles each; a unit of tpu tiles spans
// at most ceil(tpu / W) + 1 CTAs, each writing one partial per epilogue warp.
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
  *slots = ((t + w - 1) / w + 1) * kEpiWarps;
}

cudaError_t launch_rope_tc(const Params& p, uint32_t* err, cudaStream_t s) {
  int grid, W, tpu, slots;
  rope_tc_plan(p, &grid, &W, &tpu, &slots);
  Work wk{W, tpu, p.B * p.Hkv * tpu};
  static_assert(kSmTotal + 1024 <= kSmAlloc, "shared memory carve-up exceeds the allocation");
  static_assert(sizeof(Bars) <= 1024, "barrier block exceeds its slot");
  static_assert(kColALk + kNB * 16 <= kColDr && kColDr + kNDr * 128 <= kTmemCols,
                "TMEM columns exceed the allocation");
  auto kern = p.rk == 32 ? rope_tc_kernel<32> : rope_tc_kernel<16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmAlloc);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmAlloc, s>>>(p, wk, err);
  return cudaGetLastError();
}

}  // namespace kvc
