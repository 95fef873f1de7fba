// Split-T decode on INT4 low-rank caches whose keys carry no RoPE, with or
// without the 2-bit residual in the rotated (signed Walsh-Hadamard) basis,
// contiguous or paged (16-token pages).  Attention runs in the latent space:
//   s_t = q~ . l^k_t (+ q^ . y^k_t),   acc += sum_t p_t l^v_t (+ p_t y^v_t),
// with q~ = Bk q and q^ = Q q from the query projection, and the combine
// kernel maps acc back through Bv (and Q^T).
//
// Every warp streams its own contiguous range of 16-token tiles (one page of a
// (batch row, KV head) unit) through a private ring of shared-memory stages
// filled with 16-byte cp.async copies, and runs both contractions on mma.sync
// m16n8k16 (f16 operands, fp32 accumulate) with the GQA group as N:
//   - No code is dequantized element by element.  An INT4 or 2-bit code c,
//     masked into the low mantissa bits of an f16 (exponent field zero), is
//     the subnormal c * 2^-24 (times a power of two eps <= 256 for the fields
//     that sit higher up in the mantissa, undone on the other operand or at the
//     end).  The per-token scale and zero are applied after the score MMA
//     (s = scale * (c . q~) + zero * sum(q~)) and, on the value side, folded
//     into the probabilities (P' = p * scale as the B operand; the zero term
//     sum_t p_t zero_t is kept on the CUDA cores).
//   - The ordering of rank indices inside an MMA's K dimension is free (the
//     query operand uses the same order), and so is the ordering of value rows
//     (undone when the partials are written); both are chosen so that one
//     32-bit shared-memory word feeds whole operand registers.
//   - MMA row slot i holds token (i & 8) | ((i & 7) >> 1) | ((i & 1) << 2), so
//     that the value operand's token slots read tokens c4, c4 + 4, c4 + 8,
//     c4 + 12 of lane c4 (every shared-memory load is a per-thread base plus an
//     immediate, conflict-free); the residual key rows are stored in slot order.
//   - Scores are kept in units of 2^-24 log2; online softmax with a lazily
//     raised reference maximum (raised only when a score exceeds it by more
//     than 8 in log2 units); the scores of tile k + 1 are formed before the
//     softmax and value update of tile k.
#include <math.h>

#include <type_traits>

#include "kvc_device.cuh"
#include "tc_util.cuh"

namespace kvc {
namespace {

using namespace tc;

constexpr int kLT = 16;                  // tokens per tile (one page)
constexpr int kLWarps = 12;
constexpr int kLThreads = 32 * kLWarps;
constexpr int kLStages = 8;
constexpr int kDist = kLStages - 2;      // tiles in flight ahead of the one computed
constexpr int kLRank = 32;               // key rank handled (one scale group)
constexpr float kTwo24 = 16777216.f;     // code c held as the f16 bit pattern c is c * 2^-24

// Stage layout of one tile: each component of the cache as the tile's 16
// consecutive rows; the small ones first, then (residual layouts) the residual
// key codes at byte 512, so that one copy instruction of the warp moves them
// and places their rows in MMA-slot order, then the value codes.
template <int RV, bool RES>
struct Stage {
  static constexpr int NVG = (RV + 31) / 32;          // value scale groups
  static constexpr int VT = RV / 16;                  // latent value M-tiles
  static constexpr int LK = 0;
  static constexpr int LKS = LK + kLT * kLRank / 2;
  static constexpr int LVS = LKS + kLT * 4;
  static constexpr int RKS = LVS + kLT * NVG * 4;
  static constexpr int RVS = RKS + (RES ? kLT * 2 : 0);
  static constexpr int RKC = RES ? 512 : RVS;
  static constexpr int LV = RKC + (RES ? kLT * 32 : 0);
  static constexpr int RVC = LV + kLT * RV / 2;
  static constexpr int BYTES = RVC + (RES ? kLT * 32 : 0);
  static constexpr int CHUNKS = BYTES / 16;          // 16-byte copy chunks
  static constexpr int CPL = (CHUNKS + 31) / 32;      // chunks per lane
  static constexpr int SMEM = kLWarps * kLStages * BYTES;
  static_assert(!RES || RVS + kLT * 2 <= 512, "residual keys must start at byte 512");
};

struct LWork {
  int W, tpu, total;                     // tiles per warp, tiles per unit, all tiles
};


// 16-byte cp.async to shared byte address dst + OFF
template <int OFF>
__device__ __forceinline__ void cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0+%2], [%1], 16;" ::"r"(dst), "l"(src), "n"(OFF)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float2 unpack_h2(uint32_t x) {
  return __half22float2(*reinterpret_cast<const __half2*>(&x));
}

__device__ __forceinline__ __half2 u2h2(uint32_t x) { return *reinterpret_cast<__half2*>(&x); }
__device__ __forceinline__ uint32_t h2u(__half2 x) { return *reinterpret_cast<uint32_t*>(&x); }

__device__ __forceinline__ uint32_t lds32(const uint8_t* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}

// 2-bit field mu (0..7) of both 16-bit halves, scaled by eps2(mu)
__host__ __device__ constexpr uint32_t mask2(int mu) {
  return mu < 5 ? 0x00030003u << (2 * mu) : 0x00030003u << (2 * (mu - 3));
}
__host__ __device__ constexpr float eps2(int mu) {
  return mu == 0 ? 1.f : mu == 1 ? 4.f : mu == 2 ? 16.f : mu == 3 ? 64.f
       : mu == 4 ? 256.f : mu == 5 ? 16.f : mu == 6 ? 64.f : 256.f;
}
__device__ __forceinline__ uint32_t field2(uint32_t x, uint32_t x6, int mu) {
  return (mu < 5 ? x : x6) & mask2(mu);
}
constexpr uint32_t kN0 = 0x000F000Fu;    // nibble 0 of both halves (eps 1)
constexpr uint32_t kN1 = 0x00F000F0u;    // nibble 1 of both halves (eps 16)
// Code centring, exact in f16 subnormals: an INT4 value operand c * eps * 2^-24
// becomes (c - 8) * eps * 2^-24.  The long fp32 MMA accumulations then hold sums
// near the result instead of a large common part that the zero terms cancel
// afterwards, so the rounding of the tensor-core accumulation (which is not
// round-to-nearest) is not amplified.  (The 2-bit residual values, a tenth of
// the latent's in size, keep their plain codes.)
constexpr uint32_t kC0 = 0x00080008u;    // 8 * 2^-24 in both halves (eps 1)
constexpr uint32_t kC1 = 0x00800080u;    // 8 * 16 * 2^-24 (eps 16)
__device__ __forceinline__ uint32_t hsub_u32(uint32_t x, uint32_t c) {
  return h2u(__hsub2(*reinterpret_cast<__half2*>(&x), *reinterpret_cast<__half2*>(&c)));
}

template <int RV, bool RES>
__global__ void __launch_bounds__(kLThreads, 1) latent_tc_kernel(Params p, LWork wk) {
  // the combine may launch now: its blocks take SMs as this grid's CTAs exit and
  // wait (griddepcontrol.wait) for the whole grid before reading the partials
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  using L = Stage<RV, RES>;
  constexpr int NVG = L::NVG, VT = L::VT;
  constexpr int RVB = RV / 2;                   // latent value row bytes
  constexpr bool kHalfGroup = (RV % 32) != 0;   // last value group holds 16 ranks
  extern __shared__ __align__(128) uint8_t lsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * kLWarps + warp;
  const int t_first = gw * wk.W;
  const int n_tiles = min(wk.W, wk.total - t_first);
  if (n_tiles <= 0) return;
  const uint32_t ring_s = smem_u32(lsm) + warp * (kLStages * L::BYTES);
  const uint8_t* const ring = lsm + warp * (kLStages * L::BYTES);
  const int G = p.G, Hkv = p.Hkv;
  const int g = lane >> 2, c4 = lane & 3;
  const size_t rows_q = (size_t)p.B * p.Hq;
  const int pst = p.vdim + 2;
  const int npp = p.tmax / kLT;                 // tiles (pages) per batch row

  // ---- chunk c = lane + 32 i (16 bytes) of every stage: source component,
  // the chunk's offset inside the component's 16 rows, and its row bytes;
  // each copy instruction of the warp moves 512 contiguous stage bytes
  const uint8_t* c_src[L::CPL];
  int c_rowb[L::CPL];
#pragma unroll
  for (int i = 0; i < L::CPL; ++i) {
    const int o = 16 * (lane + 32 * i);
    const uint8_t* base = nullptr;
    int off = 0, rowb = 0;
    if (o < L::LKS) base = p.lk, off = L::LK, rowb = kLRank / 2;
    else if (o < L::LVS) base = reinterpret_cast<const uint8_t*>(p.lksz), off = L::LKS, rowb = 4;
    else if (o < L::RKS) base = reinterpret_cast<const uint8_t*>(p.lvsz), off = L::LVS, rowb = NVG * 4;
    else if (RES && o < L::RVS) base = reinterpret_cast<const uint8_t*>(p.rks), off = L::RKS, rowb = 2;
    else if (RES && o < L::RVS + kLT * 2) base = reinterpret_cast<const uint8_t*>(p.rvs), off = L::RVS, rowb = 2;
    else if (o < L::RKC) base = nullptr;               // padding before the residual keys
    else if (o < L::LV) base = p.rkc, off = L::RKC, rowb = 32;
    else if (o < L::RVC) base = p.lv, off = L::LV, rowb = RVB;
    else if (o < L::BYTES) base = p.rvc, off = L::RVC, rowb = 32;
    c_src[i] = base ? base + (o - off) : nullptr;
    c_rowb[i] = rowb;
  }

  // ---- first cache row of tile t of the range (page table or contiguous),
  // produced 32 tiles at a time, one per lane, a block ahead of its use
  auto tile_row = [&](int jj) -> int {
    const int t = t_first + jj;
    if (jj >= n_tiles) return 0;
    const int u = t / wk.tpu, jt = t % wk.tpu;
    const int b = u / Hkv, kvh = u % Hkv;
    if (p.page) {
      // a page id outside the cache is clamped (never read out of bounds)
      const int pg = min(max(__ldg(p.page_table + (size_t)b * npp + jt), 0), p.n_pages - 1);
      return (pg * Hkv + kvh) * kLT;
    }
    return u * p.tmax + jt * kLT;
  };
  int rows_cur = tile_row(lane), rows_next = tile_row(32 + lane);

  // whole 16-row blocks are copied, also on a unit's last, partial tile: the
  // rows past its end exist (the capacity is a multiple of 16 and pages are
  // whole), and their values are never used unmasked
  // residual key rows are stored in MMA-slot order: chunk j (token j / 2,
  // half j % 2) of that component goes to slot (token) ^-1 -- see tg below
  const int rk_tok = lane >> 1;
  const int rk_dst = L::RKC + 32 * ((rk_tok & 8) | ((rk_tok & 3) << 1) | ((rk_tok >> 2) & 1)) +
                     16 * (lane & 1);
  auto issue = [&](int stage, int row0) {
    const uint32_t dst = ring_s + stage * L::BYTES + 16 * lane;
#pragma unroll
    for (int i = 0; i < L::CPL; ++i) {
      if (lane + 32 * i < L::CHUNKS && (16 * (lane + 32 * i) >= L::RKC || 16 * (lane + 32 * i) < L::RVS + (RES ? kLT * 2 : 0))) {
        const uint8_t* src = c_src[i] + (size_t)row0 * c_rowb[i];
        switch (i) {
          case 0: cp16<0>(dst, src); break;
          case 1:
            if (RES) cp16<0>(ring_s + stage * L::BYTES + rk_dst, src);
            else cp16<512>(dst, src);
            break;
          case 2: cp16<1024>(dst, src); break;
          default: cp16<1536>(dst, src); break;
        }
      }
    }
  };

  // prologue: kDist tiles in flight
#pragma unroll
  for (int i = 0; i < kDist; ++i) {
    const int r = __shfl_sync(0xffffffffu, rows_cur, i);
    if (i < n_tiles) issue(i, r);
    cp_async_commit();
  }

  // the projected queries come from the kernel launched just before this one
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- per-unit state (scores are kept in units of 2^-24 log2)
  uint32_t bq[2][2];                     // q~ (latent key) B fragments
  uint32_t br[RES ? 8 : 1][2];           // q^ (residual key) B fragments
  float sumL[2], kR[2];                  // 2^-24 sum q~ ; -1.5 * 2^-24 sum q^ (columns 2c4 + e)
  float m_ref[2], m_thr[2], l_sum[2], nm[2];   // nm = -m_ref * 2^24
  float accV[VT][4];
  float accR[RES ? 8 : 1][4];
  float zs[NVG][2];                      // sum_t p_t zero_t per value group
  float sR[2];                           // sum_t p_t scale_t of the residual
  int cur_u = -1, cur_slot = 0;

  auto reset = [&](int u) {
    const int b = u / Hkv, kvh = u % Hkv;
    const float sl = p.scale_log2;
    const bool vq = g < G;
    const float* qr = p.qt + ((size_t)b * p.Hq + kvh * G + min(g, G - 1)) * p.qdim;
    float own_l = 0.f, own_r = 0.f;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int r0 = 8 * c4 + 2 * s;
      const float x0 = vq ? qr[r0] * sl : 0.f, x4 = vq ? qr[r0 + 4] * sl : 0.f;
      const float x1 = vq ? qr[r0 + 1] * sl * (1.f / 16.f) : 0.f;
      const float x5 = vq ? qr[r0 + 5] * sl * (1.f / 16.f) : 0.f;
      bq[s][0] = pack_h2(x0, x4);
      bq[s][1] = pack_h2(x1, x5);
      const float2 e0 = unpack_h2(bq[s][0]), e1 = unpack_h2(bq[s][1]);
      own_l += e0.x + e0.y + 16.f * (e1.x + e1.y);
    }
    if constexpr (RES) {
      const float* qh = qr + kLRank;
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int w = 2 * c4 + (s >> 2), k = s & 3;
        const int d0 = 16 * w + 2 * k;
        const float e_a = eps2(2 * k), e_b = eps2(2 * k + 1);
        const float y0 = vq ? qh[d0] * sl / e_a : 0.f, y8 = vq ? qh[d0 + 8] * sl / e_a : 0.f;
        const float y1 = vq ? qh[d0 + 1] * sl / e_b : 0.f, y9 = vq ? qh[d0 + 9] * sl / e_b : 0.f;
        br[s][0] = pack_h2(y0, y8);
        br[s][1] = pack_h2(y1, y9);
        const float2 f0 = unpack_h2(br[s][0]), f1 = unpack_h2(br[s][1]);
        own_r += e_a * (f0.x + f0.y) + e_b * (f1.x + f1.y);
      }
    }
    own_l += __shfl_xor_sync(0xffffffffu, own_l, 1);
    own_l += __shfl_xor_sync(0xffffffffu, own_l, 2);
    own_r += __shfl_xor_sync(0xffffffffu, own_r, 1);
    own_r += __shfl_xor_sync(0xffffffffu, own_r, 2);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      sumL[e] = __shfl_sync(0xffffffffu, own_l, 4 * (2 * c4 + e)) * (1.f / kTwo24);
      kR[e] = __shfl_sync(0xffffffffu, own_r, 4 * (2 * c4 + e)) * (-1.5f / kTwo24);
      m_ref[e] = m_thr[e] = -INFINITY;
      nm[e] = INFINITY;
      l_sum[e] = 0.f;
      sR[e] = 0.f;
#pragma unroll
      for (int v = 0; v < NVG; ++v) zs[v][e] = 0.f;
    }
#pragma unroll
    for (int mt = 0; mt < VT; ++mt) accV[mt][0] = accV[mt][1] = accV[mt][2] = accV[mt][3] = 0.f;
#pragma unroll
    for (int mt = 0; mt < (RES ? 8 : 1); ++mt)
      accR[mt][0] = accR[mt][1] = accR[mt][2] = accR[mt][3] = 0.f;
  };

  auto write_partial = [&]() {
    float l2[2] = {l_sum[0], l_sum[1]}, s2[2] = {sR[0], sR[1]};
    float z2[NVG][2];
#pragma unroll
    for (int v = 0; v < NVG; ++v) z2[v][0] = zs[v][0], z2[v][1] = zs[v][1];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        l2[e] += __shfl_xor_sync(0xffffffffu, l2[e], o);
        s2[e] += __shfl_xor_sync(0xffffffffu, s2[e], o);
#pragma unroll
        for (int v = 0; v < NVG; ++v) z2[v][e] += __shfl_xor_sync(0xffffffffu, z2[v][e], o);
      }
    }
    const int b = cur_u / Hkv, kvh = cur_u % Hkv;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = 2 * c4 + e;
      if (h >= G) continue;
      float* dst = p.part + ((size_t)cur_slot * rows_q + (size_t)b * p.Hq + kvh * G + h) * pst;
#pragma unroll
      for (int mt = 0; mt < VT; ++mt) {
        const int v = mt >> 1;
        int r0;
        if (kHalfGroup && mt == VT - 1) r0 = 32 * v + 2 * g;
        else r0 = 32 * v + 4 * g + 2 * (mt & 1);
        dst[r0] = accV[mt][e] * kTwo24 + z2[v][e];
        dst[r0 + 1] = accV[mt][2 + e] * (kTwo24 / 16.f) + z2[v][e];
      }
      if constexpr (RES) {
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const int k0 = 2 * mt;
          dst[RV + 16 * g + k0] = accR[mt][e] * (kTwo24 / eps2(k0 & 7)) - 1.5f * s2[e];
          dst[RV + 16 * g + k0 + 1] = accR[mt][2 + e] * (kTwo24 / eps2((k0 + 1) & 7)) - 1.5f * s2[e];
        }
      }
      if (g == 0) {
        dst[p.vdim] = m_ref[e] * kTwo24;
        dst[p.vdim + 1] = l2[e];
      }
    }
  };

  // MMA row slot i holds token (i & 8) | ((i & 7) >> 1) | ((i & 1) << 2):
  // score rows g, g + 8 read tokens tg, tg + 8, and the value operand's token
  // slots 2c4, 2c4 + 1, 2c4 + 8, 2c4 + 9 read tokens c4, c4 + 4, c4 + 8,
  // c4 + 12, so every shared-memory load is a per-thread base plus a constant
  // and the value loads of a warp hit 32 distinct banks
  const int tg = (g >> 1) | ((g & 1) << 2);
  const int o_lk = L::LK + 16 * tg + 4 * c4;
  const int o_lks = L::LKS + 4 * tg;
  const int o_rk = L::RKC + 32 * g + 8 * c4;     // rows stored in slot order
  const int o_rks = L::RKS + 2 * tg;
  const int o_lvs = L::LVS + NVG * 4 * tg;
  const int o_rv = L::RVC + 32 * c4 + 4 * g;
  const int o_rvs = L::RVS + 2 * tg;
  // latent value words: full group v -> word 4v + g/2 (half g & 1), half group
  // -> word 4v + g/4 (byte g & 3)
  const int o_lv = L::LV + RVB * c4 + 4 * (g >> 1);
  const int o_lvh = L::LV + RVB * c4 + 4 * (g >> 2);
  const uint32_t sel_v = (g & 1) ? 0x7632u : 0x5410u;
  const uint32_t bh = g & 3;
  const uint32_t sel_h = bh | (bh << 4) | ((4 + bh) << 8) | ((4 + bh) << 12);

  // ---- one tile of the current unit from stage s_use; TAIL: the unit's last
  // tile holds nt < 16 tokens (rows past nt are masked out)
  auto scores = [&](auto tail_tag, const uint8_t* st, int nt, float (&s)[4]) {
    constexpr bool TAIL = decltype(tail_tag)::value;
    const bool ok0 = !TAIL || tg < nt, ok1 = !TAIL || tg + 8 < nt;
    // rows g, g + 8 = token slots; columns 2c4, 2c4 + 1 = heads
    {
      const uint32_t k0 = lds32(st + o_lk), k1 = lds32(st + o_lk + 128);
      float aL[4] = {0.f, 0.f, 0.f, 0.f};
      {
        const uint32_t a[4] = {k0 & kN0, k1 & kN0, k0 & kN1, k1 & kN1};
        mma16816(aL, a, bq[0][0], bq[0][1]);
        const uint32_t y0 = k0 >> 8, y1 = k1 >> 8;
        const uint32_t a2[4] = {y0 & kN0, y1 & kN0, y0 & kN1, y1 & kN1};
        mma16816(aL, a2, bq[1][0], bq[1][1]);
      }
      const float2 sz0 = unpack_h2(lds32(st + o_lks));
      const float2 sz1 = unpack_h2(lds32(st + o_lks + 32));
      if constexpr (RES) {
        // the -1.5 offset of the residual levels enters as the chain's start value
        float aR0[4] = {kR[0], kR[1], kR[0], kR[1]}, aR1[4] = {0.f, 0.f, 0.f, 0.f};
        const uint2 r0 = *reinterpret_cast<const uint2*>(st + o_rk);
        const uint2 r1 = *reinterpret_cast<const uint2*>(st + o_rk + 256);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t w0 = h ? r0.y : r0.x, w1 = h ? r1.y : r1.x;
          const uint32_t w06 = w0 >> 6, w16 = w1 >> 6;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t a[4] = {field2(w0, w06, 2 * k), field2(w1, w16, 2 * k),
                                   field2(w0, w06, 2 * k + 1), field2(w1, w16, 2 * k + 1)};
            if (k & 1) mma16816(aR1, a, br[4 * h + k][0], br[4 * h + k][1]);
            else mma16816(aR0, a, br[4 * h + k][0], br[4 * h + k][1]);
          }
        }
        const float sr0 = __half2float(*reinterpret_cast<const __half*>(st + o_rks));
        const float sr1 = __half2float(*reinterpret_cast<const __half*>(st + o_rks + 16));
        s[0] = fmaf(sz0.x, aL[0], fmaf(sr0, aR0[0] + aR1[0], sz0.y * sumL[0]));
        s[1] = fmaf(sz0.x, aL[1], fmaf(sr0, aR0[1] + aR1[1], sz0.y * sumL[1]));
        s[2] = fmaf(sz1.x, aL[2], fmaf(sr1, aR0[2] + aR1[2], sz1.y * sumL[0]));
        s[3] = fmaf(sz1.x, aL[3], fmaf(sr1, aR0[3] + aR1[3], sz1.y * sumL[1]));
      } else {
        s[0] = fmaf(sz0.x, aL[0], sz0.y * sumL[0]);
        s[1] = fmaf(sz0.x, aL[1], sz0.y * sumL[1]);
        s[2] = fmaf(sz1.x, aL[2], sz1.y * sumL[0]);
        s[3] = fmaf(sz1.x, aL[3], sz1.y * sumL[1]);
      }
      if constexpr (TAIL) {
        if (!ok0) s[0] = s[1] = -INFINITY;
        if (!ok1) s[2] = s[3] = -INFINITY;
      }
    }

  };

  auto values = [&](auto tail_tag, const uint8_t* st, int nt, const float (&s)[4]) {
    constexpr bool TAIL = decltype(tail_tag)::value;
    const bool ok0 = !TAIL || tg < nt, ok1 = !TAIL || tg + 8 < nt;
    // ---------------- online softmax (lazy maximum, raised by more than 2^8)
    const bool need = s[0] > m_thr[0] || s[2] > m_thr[0] || s[1] > m_thr[1] || s[3] > m_thr[1];
    if (__any_sync(0xffffffffu, need)) {
      float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      const float n0 = fmaxf(m_ref[0], mx0), n1 = fmaxf(m_ref[1], mx1);
      const float al[2] = {ex2_approx((m_ref[0] - n0) * kTwo24),
                           ex2_approx((m_ref[1] - n1) * kTwo24)};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        l_sum[e] *= al[e];
        sR[e] *= al[e];
#pragma unroll
        for (int v = 0; v < NVG; ++v) zs[v][e] *= al[e];
#pragma unroll
        for (int mt = 0; mt < VT; ++mt) accV[mt][e] *= al[e], accV[mt][2 + e] *= al[e];
        if constexpr (RES) {
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) accR[mt][e] *= al[e], accR[mt][2 + e] *= al[e];
        }
      }
      m_ref[0] = n0;
      m_ref[1] = n1;
      m_thr[0] = n0 + 8.f / kTwo24;
      m_thr[1] = n1 + 8.f / kTwo24;
      nm[0] = -n0 * kTwo24;
      nm[1] = -n1 * kTwo24;
    }
    float pv[4];
    pv[0] = ex2_approx(fmaf(s[0], kTwo24, nm[0]));
    pv[1] = ex2_approx(fmaf(s[1], kTwo24, nm[1]));
    pv[2] = ex2_approx(fmaf(s[2], kTwo24, nm[0]));
    pv[3] = ex2_approx(fmaf(s[3], kTwo24, nm[1]));
    if constexpr (TAIL) {
      if (!ok0) pv[0] = pv[1] = 0.f;
      if (!ok1) pv[2] = pv[3] = 0.f;
    }
    l_sum[0] += pv[0] + pv[2];
    l_sum[1] += pv[1] + pv[3];
    // probabilities of the rows' tokens, packed per row: (head 2c4, head 2c4 + 1)
    const __half2 hp01 = __floats2half2_rn(pv[0], pv[1]);
    const __half2 hp23 = __floats2half2_rn(pv[2], pv[3]);

    // ---------------- values: acc^T (value row x head) += V^T (row x token) P'
    // P' = p * scale and the zero term p * zero are formed in f16x2 per tile
    // (scale and zero are fp16 already); the zero terms are summed in fp32
#pragma unroll
    for (int v = 0; v < NVG; ++v) {
      __half2 sz_0 = u2h2(lds32(st + o_lvs + 4 * v));
      __half2 sz_1 = u2h2(lds32(st + o_lvs + NVG * 32 + 4 * v));
      if constexpr (TAIL) {          // rows past the end may hold any bits
        if (!ok0) sz_0 = __float2half2_rn(0.f);
        if (!ok1) sz_1 = __float2half2_rn(0.f);
      }
      // zero term of the centred codes: p * (z + 8 s)
      const __half2 k8 = __float2half2_rn(8.f);
      const __half2 zc0 = __hfma2(__low2half2(sz_0), k8, __high2half2(sz_0));
      const __half2 zc1 = __hfma2(__low2half2(sz_1), k8, __high2half2(sz_1));
      const __half2 zt = __hfma2(hp23, zc1, __hmul2(hp01, zc0));
      const float2 ztf = __half22float2(zt);
      zs[v][0] += ztf.x;
      zs[v][1] += ztf.y;
      const uint32_t b0 = movmatrix_trans(h2u(__hmul2(hp01, __low2half2(sz_0))));
      const uint32_t b1 = movmatrix_trans(h2u(__hmul2(hp23, __low2half2(sz_1))));
      const bool half = kHalfGroup && v == NVG - 1;
      const uint8_t* lv = st + (half ? o_lvh : o_lv) + 16 * v;
      const uint32_t sel = half ? sel_h : sel_v;
      const uint32_t xA = prmt(lds32(lv), lds32(lv + 4 * RVB), sel);
      const uint32_t xB = prmt(lds32(lv + 8 * RVB), lds32(lv + 12 * RVB), sel);
      {
        const uint32_t a[4] = {hsub_u32(xA & kN0, kC0), hsub_u32(xA & kN1, kC1),
                               hsub_u32(xB & kN0, kC0), hsub_u32(xB & kN1, kC1)};
        mma16816(accV[2 * v], a, b0, b1);
      }
      if (!half) {
        const uint32_t yA = xA >> 8, yB = xB >> 8;
        const uint32_t a[4] = {hsub_u32(yA & kN0, kC0), hsub_u32(yA & kN1, kC1),
                               hsub_u32(yB & kN0, kC0), hsub_u32(yB & kN1, kC1)};
        mma16816(accV[2 * v + 1], a, b0, b1);
      }
    }
    if constexpr (RES) {
      __half2 rs_0 = __half2half2(*reinterpret_cast<const __half*>(st + o_rvs));
      __half2 rs_1 = __half2half2(*reinterpret_cast<const __half*>(st + o_rvs + 16));
      if constexpr (TAIL) {
        if (!ok0) rs_0 = __float2half2_rn(0.f);
        if (!ok1) rs_1 = __float2half2_rn(0.f);
      }
      const __half2 q01 = __hmul2(hp01, rs_0), q23 = __hmul2(hp23, rs_1);
      // the sum of the very operands the MMA uses, in fp32
      const float2 qa = __half22float2(q01), qb = __half22float2(q23);
      sR[0] += qa.x + qb.x;
      sR[1] += qa.y + qb.y;
      const uint32_t b0 = movmatrix_trans(h2u(q01));
      const uint32_t b1 = movmatrix_trans(h2u(q23));
      const uint32_t wA0 = lds32(st + o_rv), wA1 = lds32(st + o_rv + 128);
      const uint32_t wB0 = lds32(st + o_rv + 256), wB1 = lds32(st + o_rv + 384);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const uint32_t sl = hh ? 0x7632u : 0x5410u;
        const uint32_t xA = prmt(wA0, wA1, sl), xB = prmt(wB0, wB1, sl);
        const uint32_t xA6 = xA >> 6, xB6 = xB >> 6;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t a[4] = {field2(xA, xA6, 2 * k), field2(xA, xA6, 2 * k + 1),
                                 field2(xB, xB6, 2 * k), field2(xB, xB6, 2 * k + 1)};
          mma16816(accR[4 * hh + k], a, b0, b1);
        }
      }
    }
  };

  // ---- next copy: keep kDist tiles in flight, then wait for the oldest; the
  // stage of the tile before the oldest is refilled (the oldest's values are
  // still to be computed); the cache rows come 32 tiles at a time
  int ji = kDist, s_iss = kDist, s_use = 0;
  auto step = [&]() -> const uint8_t* {
    __syncwarp();                        // every lane is done with the stage refilled now
    if ((ji & 31) == 0) {
      rows_cur = rows_next;
      rows_next = tile_row(ji + 32 + lane);
    }
    const int r = __shfl_sync(0xffffffffu, rows_cur, ji & 31);
    if (ji < n_tiles) issue(s_iss, r);
    cp_async_commit();
    ++ji;
    s_iss = s_iss + 1 == kLStages ? 0 : s_iss + 1;
    cp_async_wait<kDist>();
    __syncwarp();
    const uint8_t* st = ring + s_use * L::BYTES;
    s_use = s_use + 1 == kLStages ? 0 : s_use + 1;
    return st;
  };

  // ---- the units of this warp's range, one partial each
  const int tail_nt = p.n_tokens % kLT;          // tokens of a unit's last tile, 0 = whole
  int u = t_first / wk.tpu, jt0 = t_first % wk.tpu;
  for (int jj = 0; jj < n_tiles;) {
    const int cnt = min(wk.tpu - jt0, n_tiles - jj);
    const bool tail = tail_nt != 0 && jt0 + cnt == wk.tpu;
    cur_u = u;
    cur_slot = gw - (int)(((long long)u * wk.tpu) / wk.W);
    reset(u);
    // software pipeline: the scores of tile k + 1 are formed before the
    // softmax and value update of tile k
    float s_cur[4], s_nxt[4];
    const uint8_t* st_cur = step();
    if (tail && cnt == 1) scores(std::true_type(), st_cur, tail_nt, s_cur);
    else scores(std::false_type(), st_cur, kLT, s_cur);
    for (int k = 0; k + 2 < cnt; ++k) {
      const uint8_t* st_nxt = step();
      scores(std::false_type(), st_nxt, kLT, s_nxt);
      values(std::false_type(), st_cur, kLT, s_cur);
      st_cur = st_nxt;
#pragma unroll
      for (int i = 0; i < 4; ++i) s_cur[i] = s_nxt[i];
    }
    if (cnt >= 2) {
      const uint8_t* st_nxt = step();
      if (tail) scores(std::true_type(), st_nxt, tail_nt, s_nxt);
      else scores(std::false_type(), st_nxt, kLT, s_nxt);
      values(std::false_type(), st_cur, kLT, s_cur);
      st_cur = st_nxt;
#pragma unroll
      for (int i = 0; i < 4; ++i) s_cur[i] = s_nxt[i];
    }
    if (tail) values(std::true_type(), st_cur, tail_nt, s_cur);
    else values(std::false_type(), st_cur, kLT, s_cur);
    write_partial();
    jj += cnt;
    ++u;
    jt0 = 0;
  }
  cp_async_wait<0>();
}

template <int RV, bool RES>
cudaError_t launch_t(const Params& p, const LWork& wk, int grid, cudaStream_t s) {
  using L = Stage<RV, RES>;
  cudaError_t e = cudaFuncSetAttribute(latent_tc_kernel<RV, RES>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  // a programmatic dependent of the query projection: its prologue copies
  // overlap the projection's tail
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kLThreads);
  cfg.dynamicSmemBytes = L::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, latent_tc_kernel<RV, RES>, p, wk);
}

}  // namespace

bool latent_tc_supported(const Params& p) {
  if (p.kind != KVC_LOWRANK || p.rope || p.bits != 4 || p.g != 32 || p.d != 128) return false;
  if (p.rk != kLRank || (p.rv != 32 && p.rv != 48 && p.rv != 64)) return false;
  if (p.resid != 0 && p.resid != 2) return false;
  if (p.page != 0 && p.page != kLT) return false;
  if (p.L != 1 || p.seq_lens || p.n_tokens <= 0 || p.G < 1 || p.G > 8) return false;
  if (p.tmax % kLT) return false;
  const long long rows = p.page ? (long long)p.n_pages * p.Hkv * kLT : (long long)p.B * p.Hkv * p.tmax;
  return rows < (1LL << 31) && p.vdim == p.rv + (p.resid ? kResidDim : 0) &&
         p.qdim == p.rk + (p.resid ? kResidDim : 0);
}

// Equal contiguous tile ranges per warp; a unit of tpu tiles spans at most
// ceil(tpu / W) + 1 warps, each writing one partial.
void latent_tc_plan(const Params& p, int* grid, int* W, int* tpu, int* slots) {
  const int t = (p.n_tokens + kLT - 1) / kLT;
  const long long total = (long long)p.B * p.Hkv * t;
  const long long warps_max = (long long)kNumSMs * kLWarps;
  const long long w = (total + warps_max - 1) / warps_max;
  const long long n_warps = (total + w - 1) / w;
  *grid = (int)((n_warps + kLWarps - 1) / kLWarps);
  *W = (int)w;
  *tpu = t;
  *slots = (int)((t + w - 1) / w + 1);
}

int latent_tc_slots(int batch, int n_kv_heads, int n_tokens) {
  const int t = (n_tokens + kLT - 1) / kLT;
  const long long total = (long long)batch * n_kv_heads * t;
  const long long warps_max = (long long)kNumSMs * kLWarps;
  const long long w = (total + warps_max - 1) / warps_max;
  return (int)((t + w - 1) / w + 1);
}

cudaError_t launch_latent_tc(const Params& p, cudaStream_t s) {
  int grid, W, tpu, slots;
  latent_tc_plan(p, &grid, &W, &tpu, &slots);
  const LWork wk{W, tpu, p.B * p.Hkv * tpu};
  const bool res = p.resid != 0;
  switch (p.rv) {
    case 32: return res ? launch_t<32, true>(p, wk, grid, s) : launch_t<32, false>(p, wk, grid, s);
    case 48: return res ? launch_t<48, true>(p, wk, grid, s) : launch_t<48, false>(p, wk, grid, s);
    default: return res ? launch_t<64, true>(p, wk, grid, s) : launch_t<64, false>(p, wk, grid, s);
  }
}

}  // namespace kvc
