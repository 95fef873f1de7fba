// Split-T decode on INT4 low-rank caches whose keys are stored before RoPE,
// with the key reconstruction on the fifth-generation tensor cores.
//
// Keys are k_t = l_t Bk, rotated by RoPE at slot t ("JoLT: Near-Lossless KV
// Cache Compression", Key findings: the method works pre-RoPE; attention runs
// over the stored factors without dense K/V, "A JoLT for the KV cache ...",
// Abstract).  The GQA group of a KV head shares every reconstructed key, so
// the reconstruction K = L Bk (128 tokens x 128 dims x rank 32 per tile) is the
// one dense contraction of the step; it runs as two tcgen05 MMAs
// (M = 128 tokens, N = 128 dims, K = 16) with an fp32 accumulator in TMEM.
//
// Warpgroup-autonomous streaming: a persistent CTA per SM holds kWG
// warpgroups; the 128-token tiles of all (batch row, KV head) units are cut
// into equal contiguous ranges, one per warpgroup (a range may cross a unit
// boundary: one partial per warp and unit part).  Warp w of a group owns token
// rows 32w .. 32w + 31 of every tile of its range: it copies exactly those
// rows' compressed bytes (16-byte cp.async into its own part of the group's
// ring) and reads nothing another warp copied, so the tile loop has no block or
// group barrier.  Per tile:
//   1. every thread dequantises its token's key latent (x = c s + z, f16) into
//      the group's A tile (canonical K-major, no swizzle) and a quarter of the
//      rotated-query fragments, then arrives on the tile's "A ready" mbarrier;
//   2. warp 0 of the group, one tile ahead, waits for "A ready" and for the
//      TMEM buffer to be free, issues the two reconstruction MMAs (M = 128
//      tokens, N = 128 dims, K = 16 each, fp32 accumulator in one of two TMEM
//      buffers) and commits them to the tile's "ready" mbarrier, so the MMAs
//      of tile j + 1 run while the group works on tile j;
//   3. each warp waits for "ready", reads its 32 rows of K from TMEM with the
//      16x256b shape (the m16n8 accumulator-fragment layout), releases the
//      buffer, rounds to f16 once and applies the rotation R_delta of the row
//      inside the tile (cos / sin from a per-CTA table); the tile's own
//      rotation R_t0 is folded into the queries (R_t = R_t0 R_delta);
//   4. scores K' q^T on mma.sync with the GQA group as N, online softmax with
//      a lazily raised maximum, and acc^T += Lv^T P' with the value codes as
//      centred f16 subnormal operands and the value scales folded into P'.
// The release / acquire chain of the mbarriers (a warp's arrive on "A ready",
// warp 0's wait on it and its arrive on "ready", the other warps' wait on
// "ready") orders every warp's query fragments before every other warp's
// reads.  Every wait is bounded: a wait that gives up sets the workspace error
// word and the group stops.
// The split combine merges the partials and maps acc through Bv.
#include <math.h>

#include <type_traits>

#include "kvc_device.cuh"
#include "tc_util.cuh"

namespace kvc {
namespace {

using namespace tc;

constexpr int kWG = 2;                  // warpgroups per CTA (2 x 2 TMEM buffers of 128 columns)
constexpr int kWThreads = 128 * kWG;
constexpr int kTT = 128;                // tokens per tile (M of the MMA)
constexpr int kSub = 16;                // tokens per sub-stage (one warp half)
template <int RV>
constexpr int stages_of() { return RV == 64 ? 5 : 6; }   // staged tiles per warpgroup
constexpr int kRank = 32;               // key rank (one scale group)
constexpr int kD = 128;
constexpr int kMaxHkv = 8;
constexpr int kBkBytes = kD * kRank * 2;            // one head's B operand (8 KB)
constexpr int kATile = kTT * kRank * 2;             // A operand of one tile (8 KB)
constexpr int kTrigBytes = 4 * kTT * 4 * 16;        // R_delta table (32 KB)
constexpr int kQfBytes = 4 * 32 * 16;               // rotated-query fragments of a tile (2 KB)
constexpr uint32_t kN0 = 0x000F000Fu;
constexpr uint32_t kN1 = 0x00F000F0u;
constexpr uint32_t kMagic = 0x64006400u;            // f16 1024 in both halves
constexpr uint32_t kC0 = 0x00080008u;               // 8 * 2^-24 (centring, eps 1)
constexpr uint32_t kC1 = 0x00800080u;               // 8 * 16 * 2^-24 (eps 16)

// One 16-token sub-stage: key codes, key (scale, zero), value (scale, zero)
// pairs, value codes -- the layout of the warp-level pre-RoPE kernel.
template <int RV>
struct WSub {
  static constexpr int NVG = (RV + 31) / 32;
  static constexpr int LK = 0;
  static constexpr int LKS = LK + kSub * kRank / 2;
  static constexpr int LVS = LKS + kSub * 4;
  static constexpr int LV = LVS + kSub * NVG * 4;
  static constexpr int BYTES = LV + kSub * RV / 2;
  static constexpr int CHUNKS = BYTES / 16;
  static constexpr int STAGE = 8 * BYTES;             // a 128-token tile
  static constexpr int WCHUNKS = 2 * CHUNKS;           // a warp's two sub-stages
  static constexpr int CPL = (WCHUNKS + 31) / 32;     // copy chunks per lane
  static constexpr int S = stages_of<RV>();
  // per warpgroup: ring, two A tiles, four sets of query fragments (a warp may
  // write tile j + 2's while a slower one still reads tile j's; tile j + 4's
  // waits, through the TMEM-free barrier of tile j + 1, until every warp is
  // past tile j)
  static constexpr int WG_BYTES = S * STAGE + 2 * kATile + 4 * kQfBytes;
  static constexpr int OFF_BK = 0;
  static constexpr int OFF_TRIG = OFF_BK + kMaxHkv * kBkBytes;
  static constexpr int OFF_WG = OFF_TRIG + kTrigBytes;
  static constexpr int OFF_BAR = OFF_WG + kWG * WG_BYTES;
  // per warpgroup: a_ready[2], tmem_free[2], ready[2] mbarriers, abort flag
  static constexpr int BAR_WG = 64;
  static constexpr int SMEM = OFF_BAR + 16 + kWG * BAR_WG;
  static_assert(BYTES % 16 == 0, "sub-stage must be a whole number of 16-byte chunks");
  static_assert(SMEM + 1024 <= 227 * 1024, "shared memory per CTA");
};

struct WWork {
  int W, tpu, total;   // tiles per warpgroup, tiles per unit, all tiles
};

template <int OFF>
__device__ __forceinline__ void cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0+%2], [%1], 16;" ::"r"(dst), "l"(src), "n"(OFF)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}
__device__ __forceinline__ __half2 u2h2(uint32_t x) { return *reinterpret_cast<__half2*>(&x); }
__device__ __forceinline__ uint32_t h2u(__half2 x) { return *reinterpret_cast<uint32_t*>(&x); }
__device__ __forceinline__ uint32_t lds32(const uint8_t* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}
__device__ __forceinline__ uint4 lds128(const uint8_t* p) {
  return *reinterpret_cast<const uint4*>(p);
}
__device__ __forceinline__ uint32_t cen(uint32_t x, uint32_t c) {
  return h2u(__hsub2(u2h2(x), u2h2(c)));
}

// Rank held by logical K index k of the A / B operands: a code word of ranks
// 8c .. 8c + 7 unpacks (nibble masks 0 and 4, 8 and 12 bits apart) into the
// f16 pairs (8c + a, 8c + a + 4), a = 0..3, stored as k = 8c + 2a + {0, 1}.
__host__ __device__ __forceinline__ int perm_rank(int k) {
  const int c = k >> 3, a = (k >> 1) & 3, h = k & 1;
  return 8 * c + a + 4 * h;
}

// Byte offset of element (row, k) in a K-major no-swizzle operand tile: 8 x 16
// byte core matrices, K-adjacent cores 128 bytes apart (LBO), row-adjacent
// groups of 8 rows 512 bytes apart (SBO).
__host__ __device__ __forceinline__ int kmajor_off(int row, int k) {
  return (row >> 3) * 512 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2;
}

template <int RV>
__global__ void __launch_bounds__(kWThreads, 1) rope_wg_kernel(Params p, WWork wk) {
  using L = WSub<RV>;
  constexpr int NVG = L::NVG, VT = RV / 16, RVB = RV / 2;
  constexpr bool kHalfGroup = (RV % 32) != 0;
  extern __shared__ __align__(1024) uint8_t wsm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(wsm_raw) + 1023) &
                                           ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wg = warp >> 2, wq = warp & 3, wt = tid & 127;   // warpgroup, warp in group, thread in group
  const int g = lane >> 2, c4 = lane & 3;
  const int Hkv = p.Hkv, G = p.G;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::OFF_BAR);
  uint8_t* const wbar = sm + L::OFF_BAR + 16 + wg * L::BAR_WG;
  uint64_t* a_ready = reinterpret_cast<uint64_t*>(wbar);        // [2], 4 warps arrive
  uint64_t* tmem_free = a_ready + 2;                             // [2], 4 warps arrive
  uint64_t* ready = a_ready + 4;                                 // [2], MMA commit + warp 0
  // a wait that gives up stops only its own group (the other groups finish)
  volatile int* abort_flag = reinterpret_cast<volatile int*>(wbar + 48);

  // ---- CTA setup: B operands of every KV head (logical k holds Bk row
  // perm_rank(k)), the R_delta table, barriers, TMEM
  for (int e = tid; e < Hkv * kD * kRank; e += kWThreads) {
    const int h = e / (kD * kRank), k = (e / kD) % kRank, n = e % kD;   // n fastest: coalesced
    *reinterpret_cast<__half*>(sm + L::OFF_BK + h * kBkBytes + kmajor_off(n, k)) =
        p.bk[((size_t)h * kRank + perm_rank(k)) * kD + n];
  }
  // R_delta table: entry (j, delta, c4) = (cos, sin) of delta * omega_i as f16x2
  // over dims i = 16 j + 2 c4 + {0, 1} (n-tile 2j) and i + 8 (n-tile 2j + 1)
  for (int e = tid; e < 4 * kTT * 4; e += kWThreads) {
    const int j = e / (kTT * 4), dl = (e / 4) % kTT, c = e % 4;
    uint32_t w[4];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      float cs[2], sn[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int i = 16 * j + 8 * m + 2 * c + q;
        const double turns = (double)dl * p.rope_f[i];
        sincospif(2.f * (float)(turns - rint(turns)), &sn[q], &cs[q]);
      }
      w[2 * m] = h2u(__floats2half2_rn(cs[0], cs[1]));
      w[2 * m + 1] = h2u(__floats2half2_rn(sn[0], sn[1]));
    }
    *reinterpret_cast<uint4*>(sm + L::OFF_TRIG + ((j * kTT + dl) * 4 + c) * 16) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (wt == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&a_ready[b], 4);
      mbar_init(&tmem_free[b], 4);
      mbar_init(&ready[b], 2);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();       // B operands written by threads, read by the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot + (uint32_t)(256 * wg);   // this group's two buffers

  uint8_t* const wsm = sm + L::OFF_WG + wg * L::WG_BYTES;
  uint8_t* const ring = wsm;
  uint8_t* const atile = wsm + L::S * L::STAGE;            // [2] A tiles
  uint8_t* const qfb = atile + 2 * kATile;                 // [4] query fragments
  const uint32_t ring_s = smem_u32(ring);

  const int gwg = blockIdx.x * kWG + wg;
  const int t_first = gwg * wk.W;
  const int n_tiles = max(0, min(wk.W, wk.total - t_first));
  const size_t rows_q = (size_t)p.B * p.Hq;
  const int pst = p.vdim + 2;

  // ---- this lane's copy chunks: chunk c = lane + 32 i of the warp's two
  // sub-stages (2 wq, 2 wq + 1); sub-stage, source component, offset in its rows
  const uint8_t* c_src[L::CPL];
  int c_rowb[L::CPL], c_sub[L::CPL];
#pragma unroll
  for (int i = 0; i < L::CPL; ++i) {
    const int c = lane + 32 * i;
    const int sub = 2 * wq + c / L::CHUNKS, o = 16 * (c % L::CHUNKS);
    const uint8_t* base = nullptr;
    int off = 0, rowb = 0;
    if (c < L::WCHUNKS) {
      if (o < L::LKS) base = p.lk, off = L::LK, rowb = kRank / 2;
      else if (o < L::LVS) base = reinterpret_cast<const uint8_t*>(p.lksz), off = L::LKS, rowb = 4;
      else if (o < L::LV) base = reinterpret_cast<const uint8_t*>(p.lvsz), off = L::LVS, rowb = NVG * 4;
      else base = p.lv, off = L::LV, rowb = RVB;
    }
    c_src[i] = base ? base + (o - off) : nullptr;
    c_rowb[i] = rowb;
    c_sub[i] = sub;
  }
  // first row of 16-token block jb (0 .. tmax/16 - 1) of unit u in the cache
  auto block_row = [&](int u, int jb) -> long long {
    if (p.page) {
      const int b = u / Hkv, kvh = u % Hkv;
      const int pg = min(max(__ldg(p.page_table + (size_t)b * (p.tmax / kSub) + jb), 0),
                         p.n_pages - 1);
      return ((long long)pg * Hkv + kvh) * kSub;
    }
    return (long long)u * p.tmax + (long long)jb * kSub;
  };
  auto issue = [&](int jj) {
    if (jj < n_tiles) {
      const int t = t_first + jj;
      const int u = t / wk.tpu, jt = t % wk.tpu;
      const uint32_t dst = ring_s + (jj % L::S) * L::STAGE + 2 * wq * L::BYTES;
#pragma unroll
      for (int i = 0; i < L::CPL; ++i) {
        const int c = lane + 32 * i;
        const int jb = 8 * jt + c_sub[i];
        // blocks past the capacity are never attended (rows past n_tokens)
        if (c < L::WCHUNKS && jb * kSub < p.tmax) {
          const uint8_t* src = c_src[i] + block_row(u, jb) * c_rowb[i];
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + 16 * c),
                       "l"(src)
                       : "memory");
        }
      }
    }
    cp_commit();
  };

  // ---- rotated queries: warp wq forms k-steps wq and wq + 4 of the score
  // MMA's B fragments (head g; dims 16 wq + 8 h + 2 c4 + {0, 1} and + 64)
  uint32_t Fq[2][2];                     // frac(128 f_i) of this lane's dims, in 2^-32 turns
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      double x = 128.0 * p.rope_f[16 * wq + 8 * h + 2 * c4 + q];
      x -= floor(x);
      Fq[h][q] = (uint32_t)(unsigned long long)llrint(x * 4294967296.0);
    }
  float qv[2][4];                        // q[d], q[d + 1], q[d + 64], q[d + 65] of head g (scaled)
  int q_unit = -1;
  auto load_q = [&](int u) {
    const int b = u / Hkv, kvh = u % Hkv;
    const float sl = g < G ? p.scale_log2 : 0.f;
    const __nv_bfloat16* qg = p.q + ((size_t)b * p.Hq + kvh * G + min(g, G - 1)) * kD;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int d0 = 16 * wq + 8 * h + 2 * c4;
      const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(qg + d0));
      const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(qg + d0 + 64));
      qv[h][0] = lo.x * sl;
      qv[h][1] = lo.y * sl;
      qv[h][2] = hi.x * sl;
      qv[h][3] = hi.y * sl;
    }
    q_unit = u;
  };
  // (R_t0^T q)_i = q_i c + q_{i+64} s ; (R_t0^T q)_{i+64} = q_{i+64} c - q_i s
  auto rotate_q = [&](int jt, uint8_t* qf) {
    uint32_t w[2][2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float cs[2], sn[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int turns = (int)((uint32_t)jt * Fq[h][q]);
        __sincosf((float)turns * 1.4629180792671596e-09f, &sn[q], &cs[q]);   // 2 pi / 2^32
      }
      w[0][h] = h2u(__floats2half2_rn(fmaf(qv[h][0], cs[0], qv[h][2] * sn[0]),
                                      fmaf(qv[h][1], cs[1], qv[h][3] * sn[1])));
      w[1][h] = h2u(__floats2half2_rn(fmaf(qv[h][2], cs[0], -qv[h][0] * sn[0]),
                                      fmaf(qv[h][3], cs[1], -qv[h][1] * sn[1])));
    }
    // fragments [k-step pair][lane][k-step parity][h]: k-steps wq (low dims) and wq + 4
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int j = wq + 4 * e;
      *reinterpret_cast<uint2*>(qf + ((j >> 1) * 32 + lane) * 16 + (j & 1) * 8) =
          make_uint2(w[e][0], w[e][1]);
    }
  };

  // ---- per-warp softmax state for heads 2 c4, 2 c4 + 1 (rows g, g + 8 of each half)
  float m_ref[2], m_thr[2], l_sum[2];
  float accV[VT][4];
  float zs[NVG][2];
  auto reset = [&]() {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      m_ref[e] = m_thr[e] = -INFINITY;
      l_sum[e] = 0.f;
#pragma unroll
      for (int v = 0; v < NVG; ++v) zs[v][e] = 0.f;
    }
#pragma unroll
    for (int mt = 0; mt < VT; ++mt) accV[mt][0] = accV[mt][1] = accV[mt][2] = accV[mt][3] = 0.f;
  };
  auto write_partial = [&](int u) {
    float l2[2] = {l_sum[0], l_sum[1]};
    float z2[NVG][2];
#pragma unroll
    for (int v = 0; v < NVG; ++v) z2[v][0] = zs[v][0], z2[v][1] = zs[v][1];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        l2[e] += __shfl_xor_sync(0xffffffffu, l2[e], o);
#pragma unroll
        for (int v = 0; v < NVG; ++v) z2[v][e] += __shfl_xor_sync(0xffffffffu, z2[v][e], o);
      }
    }
    const int b = u / Hkv, kvh = u % Hkv;
    const int slot = (gwg - (int)(((long long)u * wk.tpu) / wk.W)) * 4 + wq;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = 2 * c4 + e;
      if (h >= G) continue;
      float* dst = p.part + ((size_t)slot * rows_q + (size_t)b * p.Hq + kvh * G + h) * pst;
#pragma unroll
      for (int mt = 0; mt < VT; ++mt) {
        const int v = mt >> 1;
        int r0;
        if (kHalfGroup && mt == VT - 1) r0 = 32 * v + 2 * g;
        else r0 = 32 * v + 4 * g + 2 * (mt & 1);
        dst[r0] = accV[mt][e] * 16777216.f + z2[v][e];
        dst[r0 + 1] = accV[mt][2 + e] * (16777216.f / 16.f) + z2[v][e];
      }
      if (g == 0) {
        dst[p.vdim] = m_ref[e];
        dst[p.vdim + 1] = l2[e];
      }
    }
  };

  // ---- softmax + value product of one 16-token sub-stage (rows g, g + 8)
  const uint32_t sel_v = (g & 1) ? 0x7632u : 0x5410u;
  const uint32_t bh = g & 3;
  const uint32_t sel_h = bh | (bh << 4) | ((4 + bh) << 8) | ((4 + bh) << 12);
  const int o_lv = L::LV + RVB * 2 * c4 + 4 * (g >> 1);
  const int o_lvh = L::LV + RVB * 2 * c4 + 4 * (g >> 2);
  auto values = [&](const uint8_t* st, int nt, const float (&s)[4]) {
    const bool ok0 = g < nt, ok1 = g + 8 < nt;
    const bool need = s[0] > m_thr[0] || s[2] > m_thr[0] || s[1] > m_thr[1] || s[3] > m_thr[1];
    if (__any_sync(0xffffffffu, need)) {
      float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      const float n0 = fmaxf(m_ref[0], mx0), n1 = fmaxf(m_ref[1], mx1);
      // a = 2^(m_old - m_new): 0 for a first maximum (m_old = -inf)
      const float al[2] = {ex2_approx(m_ref[0] - n0), ex2_approx(m_ref[1] - n1)};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        l_sum[e] *= al[e];
#pragma unroll
        for (int v = 0; v < NVG; ++v) zs[v][e] *= al[e];
#pragma unroll
        for (int mt = 0; mt < VT; ++mt) accV[mt][e] *= al[e], accV[mt][2 + e] *= al[e];
      }
      m_ref[0] = n0;
      m_ref[1] = n1;
      m_thr[0] = n0 + 8.f;
      m_thr[1] = n1 + 8.f;
    }
    float pv[4];
    pv[0] = ok0 ? ex2_approx(s[0] - m_ref[0]) : 0.f;
    pv[1] = ok0 ? ex2_approx(s[1] - m_ref[1]) : 0.f;
    pv[2] = ok1 ? ex2_approx(s[2] - m_ref[0]) : 0.f;
    pv[3] = ok1 ? ex2_approx(s[3] - m_ref[1]) : 0.f;
    l_sum[0] += pv[0] + pv[2];
    l_sum[1] += pv[1] + pv[3];
    const __half2 hp01 = __floats2half2_rn(pv[0], pv[1]);
    const __half2 hp23 = __floats2half2_rn(pv[2], pv[3]);
    const __half2 k8 = __float2half2_rn(8.f);
#pragma unroll
    for (int v = 0; v < NVG; ++v) {
      __half2 sz_0 = u2h2(lds32(st + L::LVS + NVG * 4 * g + 4 * v));
      __half2 sz_1 = u2h2(lds32(st + L::LVS + NVG * 4 * (g + 8) + 4 * v));
      if (!ok0) sz_0 = __float2half2_rn(0.f);   // rows past the end may hold any bits
      if (!ok1) sz_1 = __float2half2_rn(0.f);
      // zero term of the centred codes: p * (z + 8 s)
      const __half2 zc0 = __hfma2(__low2half2(sz_0), k8, __high2half2(sz_0));
      const __half2 zc1 = __hfma2(__low2half2(sz_1), k8, __high2half2(sz_1));
      const float2 ztf = __half22float2(__hfma2(hp23, zc1, __hmul2(hp01, zc0)));
      zs[v][0] += ztf.x;
      zs[v][1] += ztf.y;
      const uint32_t b0 = movmatrix_trans(h2u(__hmul2(hp01, __low2half2(sz_0))));
      const uint32_t b1 = movmatrix_trans(h2u(__hmul2(hp23, __low2half2(sz_1))));
      const bool half = kHalfGroup && v == NVG - 1;
      const uint8_t* lv = st + (half ? o_lvh : o_lv) + 16 * v;
      const uint32_t sel = half ? sel_h : sel_v;
      const uint32_t xA = prmt(lds32(lv), lds32(lv + RVB), sel);
      const uint32_t xB = prmt(lds32(lv + 8 * RVB), lds32(lv + 9 * RVB), sel);
      {
        const uint32_t av[4] = {cen(xA & kN0, kC0), cen(xA & kN1, kC1), cen(xB & kN0, kC0),
                                cen(xB & kN1, kC1)};
        mma16816(accV[2 * v], av, b0, b1);
      }
      if (!half) {
        const uint32_t yA = xA >> 8, yB = xB >> 8;
        const uint32_t av[4] = {cen(yA & kN0, kC0), cen(yA & kN1, kC1), cen(yB & kN0, kC0),
                                cen(yB & kN1, kC1)};
        mma16816(accV[2 * v + 1], av, b0, b1);
      }
    }
  };

  // ---- 1. this warp's rows of tile jj -> A tile (buffer jj & 1) and query
  // fragments (buffer jj & 3)
  const uint32_t k1024 = 0x64006400u;
  auto prepare = [&](int jj) {
    const int t = t_first + jj;
    const int u = t / wk.tpu, jt = t % wk.tpu;
    const int nt = min(kTT, p.n_tokens - jt * kTT);
    const uint8_t* st = ring + (jj % L::S) * L::STAGE;
    uint8_t* at = atile + (jj & 1) * kATile;
    const int row = 32 * wq + lane;                      // token row of this thread
    const uint8_t* sb = st + (row >> 4) * L::BYTES;
    const int r = row & 15;
    const uint4 w = lds128(sb + L::LK + 16 * r);
    const uint32_t vm = row < nt ? 0xFFFFFFFFu : 0u;     // zero rows past the end
    const __half2 sz = u2h2(lds32(sb + L::LKS + 4 * r) & vm);
    const __half2 s2 = __low2half2(sz), z2 = __high2half2(sz);
    const uint32_t ws4[4] = {w.x, w.y, w.z, w.w};
    const uint32_t rowoff = (row >> 3) * 512 + (row & 7) * 16;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t o[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const uint32_t x = ((ws4[c] >> (4 * a)) & kN0) | kMagic;
        o[a] = h2u(__hfma2(__hsub2(u2h2(x), u2h2(k1024)), s2, z2));
      }
      *reinterpret_cast<uint4*>(at + rowoff + c * 128) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (u != q_unit) load_q(u);
    rotate_q(jt, qfb + (jj & 3) * kQfBytes);
    fence_proxy_async_smem();              // A written by threads, read by the tensor core
    __syncwarp();
    if (lane == 0) mbar_arrive(&a_ready[jj & 1]);
  };
  // ---- 2. warp 0: the reconstruction MMAs of tile jj (after every warp's rows,
  // and after every warp has read the TMEM buffer's previous tile jj - 2)
  auto issue_mma = [&](int jj) -> bool {
    const int b = jj & 1;
    if (!mbar_wait(&a_ready[b], (uint32_t)(jj >> 1) & 1u, abort_flag, p.err)) return false;
    if (jj >= 2 && !mbar_wait(&tmem_free[b], (uint32_t)((jj - 2) >> 1) & 1u, abort_flag, p.err))
      return false;
    tc_fence_after();
    if (lane == 0) {
      const int t = t_first + jj;
      const uint32_t idesc = idesc_f16(kTT, kD, 0, 0);
      const uint8_t* bk = sm + L::OFF_BK + ((t / wk.tpu) % Hkv) * kBkBytes;
      const uint8_t* at = atile + b * kATile;
#pragma unroll
      for (int kk = 0; kk < kRank / 16; ++kk)
        mma_ss(tmem + 128 * b, smem_desc(at + kk * 256, 128, 512),
               smem_desc(bk + kk * 256, 128, 512), idesc, kk > 0);
      tc_commit(&ready[b]);
      mbar_arrive(&ready[b]);              // releases warp 0's own writes with the chain
    }
    __syncwarp();
    return true;
  };

  // ---- the warpgroup's tiles
#pragma unroll
  for (int i = 0; i < L::S - 1; ++i) issue(i);
  int cur_u = -1;
  bool ok = true;
  int issued = 0;                          // tiles whose MMAs warp 0 has issued
  if (n_tiles > 0) {
    cp_wait<L::S - 2>();                   // this lane's copies of tile 0
    __syncwarp();
    prepare(0);
    if (wq == 0) ok = issue_mma(0), issued = ok ? 1 : 0;
  }
  for (int jj = 0; jj < n_tiles && ok; ++jj) {
    const int t = t_first + jj;
    const int u = t / wk.tpu, jt = t % wk.tpu;
    const int nt = min(kTT, p.n_tokens - jt * kTT);     // valid rows of this tile
    // refill the stage of tile jj - 1 (this warp's part), then tile jj + 1's rows
    issue(jj + L::S - 1);
    if (jj + 1 < n_tiles) {
      cp_wait<L::S - 2>();
      __syncwarp();
      prepare(jj + 1);
      if (wq == 0) {
        ok = issue_mma(jj + 1);
        if (ok) issued = jj + 2;
      }
    }
    if (!ok) break;
    if (u != cur_u) {
      if (cur_u >= 0) write_partial(cur_u);
      reset();
      cur_u = u;
    }
    const int b = jj & 1;
    if (!mbar_wait(&ready[b], (uint32_t)(jj >> 1) & 1u, abort_flag, p.err)) {
      ok = false;
      break;
    }
    tc_fence_after();
    const uint8_t* qf = qfb + (jj & 3) * kQfBytes;
    uint32_t qb[8][2];
#pragma unroll
    for (int jp = 0; jp < 4; ++jp) {
      const uint4 v = lds128(qf + (jp * 32 + lane) * 16);
      qb[2 * jp][0] = v.x;
      qb[2 * jp][1] = v.y;
      qb[2 * jp + 1][0] = v.z;
      qb[2 * jp + 1][1] = v.w;
    }
    const uint8_t* st = ring + (jj % L::S) * L::STAGE;
    // 3.-4. per 16-row half of this warp's 32 rows
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh) {
      const int row0 = 32 * wq + 16 * hh;              // first row of the half in the tile
      const uint32_t ta = tmem + 128 * b + ((uint32_t)row0 << 16);
      uint32_t klo[4][8], khi[4][8];                   // n-tiles 2j, 2j+1 and 2j+8, 2j+9 (fp32)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        tmem_ld16x256_x2(ta + 16 * j, klo[j]);
        tmem_ld16x256_x2(ta + 64 + 16 * j, khi[j]);
      }
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        reg_fence(klo[j]);
        reg_fence(khi[j]);
      }
      if (hh == 1) {                                   // this warp is done with the buffer
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tmem_free[b]);
      }
      // R_delta of rows row0 + g and row0 + g + 8, rounded to f16 once before
      uint32_t kf[16][2];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const uint4 tr = lds128(sm + L::OFF_TRIG + ((j * kTT + row0 + g + 8 * r) * 4 + c4) * 16);
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            const __half2 cs = u2h2(m ? tr.z : tr.x), sn = u2h2(m ? tr.w : tr.y);
            const __half2 lo = __floats2half2_rn(__uint_as_float(klo[j][4 * m + 2 * r]),
                                                 __uint_as_float(klo[j][4 * m + 2 * r + 1]));
            const __half2 hi = __floats2half2_rn(__uint_as_float(khi[j][4 * m + 2 * r]),
                                                 __uint_as_float(khi[j][4 * m + 2 * r + 1]));
            kf[2 * j + m][r] = h2u(__hfma2(lo, cs, __hneg2(__hmul2(hi, sn))));
            kf[2 * j + m + 8][r] = h2u(__hfma2(hi, cs, __hmul2(lo, sn)));
          }
        }
      }
      // scores: k-step j takes n-tiles 2j, 2j + 1 as the A fragment
      float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t af[4] = {kf[2 * j][0], kf[2 * j][1], kf[2 * j + 1][0], kf[2 * j + 1][1]};
        if (j & 1) mma16816(s1, af, qb[j][0], qb[j][1]);
        else mma16816(s0, af, qb[j][0], qb[j][1]);
      }
      float s[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) s[i] = s0[i] + s1[i];
      const int nth = nt - row0;                       // valid rows of this half
      if (g >= nth) s[0] = s[1] = -INFINITY;
      if (g + 8 >= nth) s[2] = s[3] = -INFINITY;
      values(st + (2 * wq + hh) * L::BYTES, nth, s);
    }
  }
  if (ok && cur_u >= 0) write_partial(cur_u);
  // on a wait that gave up: let the MMAs warp 0 issued finish before TMEM is freed
  if (!ok && wq == 0 && issued > 0) {
    volatile int no_abort = 0;
    mbar_wait(&ready[(issued - 1) & 1], (uint32_t)((issued - 1) >> 1) & 1u, &no_abort, nullptr);
  }
  cp_wait<0>();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, 512);
  }
}

template <int RV>
cudaError_t launch_w(const Params& p, const WWork& wk, int grid, cudaStream_t s) {
  using L = WSub<RV>;
  cudaError_t e = cudaFuncSetAttribute(rope_wg_kernel<RV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM + 1024);
  if (e != cudaSuccess) return e;
  rope_wg_kernel<RV><<<grid, kWThreads, L::SMEM + 1024, s>>>(p, wk);
  return cudaGetLastError();
}

}  // namespace

bool rope_wg_supported(const Params& p) {
  if (p.kind != KVC_LOWRANK || !p.rope || p.bits != 4 || p.g != 32 || p.d != kD) return false;
  if (p.rk != kRank || (p.rv != 32 && p.rv != 48 && p.rv != 64) || p.resid) return false;
  if (p.page != 0 && p.page != kSub) return false;
  if (p.L != 1 || p.seq_lens || p.n_tokens <= 0 || p.G < 1 || p.G > 8) return false;
  if (p.Hkv > kMaxHkv || p.tmax % kSub) return false;
  const long long rows = p.page ? (long long)p.n_pages * p.Hkv * kSub : (long long)p.B * p.Hkv * p.tmax;
  return rows < (1LL << 31) && p.vdim == p.rv;
}

void rope_wg_plan(const Params& p, int* grid, int* W, int* tpu, int* slots) {
  const int t = (p.n_tokens + kTT - 1) / kTT;
  const long long total = (long long)p.B * p.Hkv * t;
  const long long groups_max = (long long)kNumSMs * kWG;
  const long long w = (total + groups_max - 1) / groups_max;
  const long long n_groups = (total + w - 1) / w;
  *grid = (int)((n_groups + kWG - 1) / kWG);
  *W = (int)w;
  *tpu = t;
  *slots = (int)((t + w - 1) / w + 1) * 4;
}

int rope_wg_slots(int batch, int n_kv_heads, int n_tokens) {
  const int t = (n_tokens + kTT - 1) / kTT;
  const long long total = (long long)batch * n_kv_heads * t;
  const long long groups_max = (long long)kNumSMs * kWG;
  const long long w = (total + groups_max - 1) / groups_max;
  return (int)((t + w - 1) / w + 1) * 4;
}

cudaError_t launch_rope_wg(const Params& p, cudaStream_t s) {
  int grid, W, tpu, slots;
  rope_wg_plan(p, &grid, &W, &tpu, &slots);
  const WWork wk{W, tpu, p.B * p.Hkv * tpu};
  switch (p.rv) {
    case 32: return launch_w<32>(p, wk, grid, s);
    case 48: return launch_w<48>(p, wk, grid, s);
    default: return launch_w<64>(p, wk, grid, s);
  }
}

}  // namespace kvc
