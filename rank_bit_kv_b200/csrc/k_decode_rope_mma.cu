// Split-T decode on INT4 low-rank caches whose keys are stored before RoPE,
// on warp-level MMAs.  Every warp streams its own contiguous range of 16-token
// tiles through a private ring of shared-memory stages (16-byte cp.async) and,
// per tile:
//   - dequantises the key latents into f16 operands (x = c s + z per token and
//     group) and reconstructs K = L Bk with mma.sync m16n8k16 (M = 16 tokens,
//     N = 128 dims, K = the rank; fp32 accumulate, each sum rounded to f16
//     once), the Bk fragments read from shared memory with ldmatrix.trans;
//   - applies the rotation of the token's position inside its group of 128 (or
//     64) tokens,
//     R_delta, in f16x2 (cos / sin of delta * omega_i from a per-CTA table);
//     the group's own rotation R_t0 is folded into the queries once per group
//     (R_t = R_t0 R_delta, rotate-half pairs (i, i + 64));
//   - scores K' q_rot^T on mma.sync (the reconstructed fragments are the A
//     operand as they are; the GQA group is N), online softmax with a lazily
//     raised maximum, and acc^T += Lv^T P' with the value codes as MMA
//     operands (f16 subnormals) and the value scales folded into P'.
// The combine kernel merges the per-unit partials and maps acc through Bv.
#include <math.h>

#include <type_traits>

#include "kvc_device.cuh"
#include "tc_util.cuh"

namespace kvc {
namespace {

using namespace tc;

constexpr int kPT = 16;                  // tokens per tile
constexpr int kPWarps = 12;
constexpr int kPThreads = 32 * kPWarps;
constexpr int kPStages = 8;
constexpr int kPDist = kPStages - 2;     // tiles in flight ahead of the one computed
constexpr int kPRank = 32;               // key rank handled (one scale group)
// tokens sharing one query rotation: 128 where the rotation table fits next to
// the rings (value rank <= 48), else 64
template <int RV>
constexpr int group_of() { return RV <= 48 ? 128 : 64; }
constexpr int kPMaxHkv = 8;
constexpr int kBkRow = 272;              // smem bytes per Bk row (128 f16 + 16 pad)
constexpr int kBkHead = kPRank * kBkRow; // one KV head's factor
constexpr int kRopeRow = 320;            // smem bytes per delta of the rotation table
constexpr int kQTab = 64 * 8;            // per-warp (cos, sin) of the group rotation
constexpr int kQStride = 136;            // bf16 per staged query row (padded: no bank conflicts)
constexpr int kQRows = 8 * kQStride * 2; // per-warp queries of the current unit (bf16)

template <int RV>
struct PStage {
  static constexpr int NVG = (RV + 31) / 32;
  static constexpr int VT = RV / 16;
  static constexpr int LK = 0;
  static constexpr int LKS = LK + kPT * kPRank / 2;
  static constexpr int LVS = LKS + kPT * 4;
  static constexpr int LV = LVS + kPT * NVG * 4;
  static constexpr int BYTES = LV + kPT * RV / 2;
  static constexpr int CHUNKS = BYTES / 16;
  static constexpr int CPL = (CHUNKS + 31) / 32;
  static constexpr int GROUP = group_of<RV>();
  // dynamic shared memory: factors, rotation table, per-warp group rotation, rings
  static constexpr int OFF_ROPE = kPMaxHkv * kBkHead;
  static constexpr int OFF_QTAB = OFF_ROPE + GROUP * kRopeRow;
  static constexpr int OFF_QROW = OFF_QTAB + kPWarps * kQTab;
  static constexpr int OFF_RING = OFF_QROW + kPWarps * kQRows;
  static constexpr int SMEM = OFF_RING + kPWarps * kPStages * BYTES;
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

struct PWork {
  int W, tpu, total;
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

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

constexpr uint32_t kN0 = 0x000F000Fu;    // nibble 0 of both halves
constexpr uint32_t kN1 = 0x00F000F0u;    // nibble 1 of both halves (x 16)
constexpr uint32_t kMagic = 0x64006400u; // f16 1024 in both halves
// Value codes enter the MMA centred, (c - 8) * eps * 2^-24 (exact in f16
// subnormals), so the long fp32 accumulation holds a sum near the result rather
// than a large common part that the zero term cancels afterwards.
constexpr uint32_t kC0 = 0x00080008u;    // 8 * 2^-24 in both halves (eps 1)
constexpr uint32_t kC1 = 0x00800080u;    // 8 * 16 * 2^-24 (eps 16)

// Rank held by k-slot kappa (0..15) of k-step ks of the reconstruction MMA:
// thread c4 turns word c4 of a latent row (ranks 8 c4 .. 8 c4 + 7) into its
// A registers (nibbles 0 / 4, 1 / 5 for step 0; 2 / 6, 3 / 7 for step 1).
__host__ __device__ constexpr int recon_rank(int ks, int kappa) {
  return 8 * ((kappa & 7) >> 1) + 4 * (kappa & 1) + 2 * ks + (kappa >> 3);
}

template <int RV>
__global__ void __launch_bounds__(kPThreads, 1) rope_mma_kernel(Params p, PWork wk) {
  // the combine may launch now: its blocks take SMs as this grid's CTAs exit and
  // wait (griddepcontrol.wait) for the whole grid before reading the partials
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  using L = PStage<RV>;
  constexpr int NVG = L::NVG, VT = L::VT;
  constexpr int RVB = RV / 2;
  constexpr bool kHalfGroup = (RV % 32) != 0;
  extern __shared__ __align__(128) uint8_t psm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hkv = p.Hkv, G = p.G;
  const uint32_t sm_s = smem_u32(psm);

  // ---- CTA setup: Bk of every KV head, rows in the k-slot order of the MMA
  for (int e = tid; e < Hkv * kPRank * 16; e += kPThreads) {
    const int h = e / (kPRank * 16), row = (e / 16) % kPRank, ch = e % 16;
    const int rank = recon_rank(row >> 4, row & 15);
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.bk + ((size_t)h * kPRank + rank) * 128) + ch);
    *reinterpret_cast<uint4*>(psm + h * kBkHead + row * kBkRow + ch * 16) = v;
  }
  // rotation table: delta in [0, GROUP), entry (m, c4) holds (cos, sin) of
  // delta * omega_i for dims i = 8 nt + 2 c4 + {0, 1}, nt = 2m, 2m + 1, packed f16x2
  for (int e = tid; e < L::GROUP * 16; e += kPThreads) {
    const int dl = e >> 4, m = (e >> 2) & 3, c = e & 3;
    uint32_t w[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float cs[2], sn[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int i = 8 * (2 * m + h) + 2 * c + q;
        const double turns = (double)dl * p.rope_f[i];
        sincospif(2.f * (float)(turns - rint(turns)), &sn[q], &cs[q]);
      }
      w[2 * h] = h2u(__floats2half2_rn(cs[0], cs[1]));
      w[2 * h + 1] = h2u(__floats2half2_rn(sn[0], sn[1]));
    }
    *reinterpret_cast<uint4*>(psm + L::OFF_ROPE + dl * kRopeRow + m * 64 + c * 16) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
  __syncthreads();

  const int gw = blockIdx.x * kPWarps + warp;
  const int t_first = gw * wk.W;
  const int n_tiles = min(wk.W, wk.total - t_first);
  if (n_tiles <= 0) return;
  const uint32_t ring_s = sm_s + L::OFF_RING + warp * (kPStages * L::BYTES);
  const uint8_t* const ring = psm + L::OFF_RING + warp * (kPStages * L::BYTES);
  float2* const qtab = reinterpret_cast<float2*>(psm + L::OFF_QTAB + warp * kQTab);
  __nv_bfloat16* const qsm = reinterpret_cast<__nv_bfloat16*>(psm + L::OFF_QROW + warp * kQRows);
  const int g = lane >> 2, c4 = lane & 3;
  const size_t rows_q = (size_t)p.B * p.Hq;
  const int pst = p.vdim + 2;

  // ---- copy chunks (c = lane + 32 i): component, offset inside its 16 rows
  const uint8_t* c_src[L::CPL];
  int c_rowb[L::CPL];
#pragma unroll
  for (int i = 0; i < L::CPL; ++i) {
    const int o = 16 * (lane + 32 * i);
    const uint8_t* base = nullptr;
    int off = 0, rowb = 0;
    if (o < L::LKS) base = p.lk, off = L::LK, rowb = kPRank / 2;
    else if (o < L::LVS) base = reinterpret_cast<const uint8_t*>(p.lksz), off = L::LKS, rowb = 4;
    else if (o < L::LV) base = reinterpret_cast<const uint8_t*>(p.lvsz), off = L::LVS, rowb = NVG * 4;
    else if (o < L::BYTES) base = p.lv, off = L::LV, rowb = RVB;
    c_src[i] = base ? base + (o - off) : nullptr;
    c_rowb[i] = rowb;
  }
  auto tile_row = [&](int jj) -> int {
    if (jj >= n_tiles) return 0;
    const int t = t_first + jj;
    const int u = t / wk.tpu, jt = t % wk.tpu;
    if (p.page) {
      const int b = u / Hkv, kvh = u % Hkv;
      // a page id outside the cache is clamped (never read out of bounds)
      const int pg = min(max(__ldg(p.page_table + (size_t)b * (p.tmax / kPT) + jt), 0), p.n_pages - 1);
      return (pg * Hkv + kvh) * kPT;
    }
    return u * p.tmax + jt * kPT;
  };
  int rows_cur = tile_row(lane), rows_next = tile_row(32 + lane);
  auto issue = [&](int stage, int row0) {
    const uint32_t dst = ring_s + stage * L::BYTES + 16 * lane;
#pragma unroll
    for (int i = 0; i < L::CPL; ++i) {
      if (lane + 32 * i < L::CHUNKS) {
        const uint8_t* src = c_src[i] + (size_t)row0 * c_rowb[i];
        if (i == 0) cp16<0>(dst, src);
        else if (i == 1) cp16<512>(dst, src);
        else cp16<1024>(dst, src);
      }
    }
  };
#pragma unroll
  for (int i = 0; i < kPDist; ++i) {
    const int r = __shfl_sync(0xffffffffu, rows_cur, i);
    if (i < n_tiles) issue(i, r);
    cp_commit();
  }

  // ---- per-unit state (scores in log2 units)
  uint32_t qb[8][2];                     // rotated queries, B fragments of the score MMA
  float m_ref[2], m_thr[2], l_sum[2];
  float accV[VT][4];
  float zs[NVG][2];
  int cur_u = -1, cur_slot = 0, cur_J = -1;

  auto reset = [&](int u) {
    const int b = u / Hkv, kvh = u % Hkv;
    // the unit's queries, once, into this warp's shared area
    __syncwarp();
    const __nv_bfloat16* qg = p.q + ((size_t)b * p.Hq + kvh * G) * 128;
    for (int e = lane; e < G * 16; e += 32)
      *reinterpret_cast<uint4*>(qsm + (e >> 4) * kQStride + 8 * (e & 15)) =
          __ldg(reinterpret_cast<const uint4*>(qg) + e);
    __syncwarp();
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      m_ref[e] = m_thr[e] = -INFINITY;
      l_sum[e] = 0.f;
#pragma unroll
      for (int v = 0; v < NVG; ++v) zs[v][e] = 0.f;
    }
#pragma unroll
    for (int mt = 0; mt < VT; ++mt) accV[mt][0] = accV[mt][1] = accV[mt][2] = accV[mt][3] = 0.f;
    cur_J = -1;
  };

  // queries rotated by R_t0, t0 = GROUP J, scaled by the softmax scale (log2 e
  // folded in), as the score MMA's B fragments
  auto rotate_q = [&](int J) {
    const double t0 = (double)J * L::GROUP;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int i = lane + 32 * k;
      const double turns = t0 * p.rope_f[i];
      float sn, cs;
      sincospif(2.f * (float)(turns - rint(turns)), &sn, &cs);
      qtab[i] = make_float2(cs, sn);
    }
    __syncwarp();
    const float sl = g < G ? p.scale_log2 : 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int d0 = 16 * j + 8 * h + 2 * c4;           // dims d0, d0 + 1 (< 64)
        const __nv_bfloat16* qr = qsm + min(g, G - 1) * kQStride;
        const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(qr + d0));
        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(qr + d0 + 64));
        const float2 t0c = qtab[d0], t1c = qtab[d0 + 1];
        const float l0 = lo.x, l1 = lo.y, h0 = hi.x, h1 = hi.y;
        // (R^T q)_i = q_i c + q_{i+64} s ; (R^T q)_{i+64} = q_{i+64} c - q_i s
        qb[j][h] = h2u(__floats2half2_rn(sl * fmaf(l0, t0c.x, h0 * t0c.y),
                                         sl * fmaf(l1, t1c.x, h1 * t1c.y)));
        qb[j + 4][h] = h2u(__floats2half2_rn(sl * fmaf(h0, t0c.x, -l0 * t0c.y),
                                             sl * fmaf(h1, t1c.x, -l1 * t1c.y)));
      }
    }
    __syncwarp();
  };

  auto write_partial = [&]() {
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
        dst[r0] = accV[mt][e] * 16777216.f + z2[v][e];
        dst[r0 + 1] = accV[mt][2 + e] * (16777216.f / 16.f) + z2[v][e];
      }
      if (g == 0) {
        dst[p.vdim] = m_ref[e];
        dst[p.vdim + 1] = l2[e];
      }
    }
  };

  const uint32_t sel_v = (g & 1) ? 0x7632u : 0x5410u;
  const uint32_t bh = g & 3;
  const uint32_t sel_h = bh | (bh << 4) | ((4 + bh) << 8) | ((4 + bh) << 12);
  const int o_lv = L::LV + RVB * 2 * c4 + 4 * (g >> 1);
  const int o_lvh = L::LV + RVB * 2 * c4 + 4 * (g >> 2);
  // ldmatrix row address of this lane inside a KV head's factor: matrix
  // lane / 8 -> (k-slot half, n-tile of the pair), row lane % 8
  const int ldsm_off = ((lane & 7) + 8 * ((lane >> 3) & 1)) * kBkRow + 16 * (lane >> 4);
  const uint32_t rope_s = sm_s + L::OFF_ROPE + 16 * c4;

  // ---- scores of one tile (rows g, g + 8 = tokens; columns 2c4, 2c4 + 1 = heads)
  auto scores = [&](auto tail_tag, const uint8_t* st, int jt, int nt, float (&s)[4]) {
    constexpr bool TAIL = decltype(tail_tag)::value;
    const int kvh = cur_u % Hkv;
    // dequantised key latents as the A operand: rows g, g + 8
    uint32_t a[2][4];
    {
      const uint32_t w0 = lds32(st + L::LK + 16 * g + 4 * c4);
      const uint32_t w1 = lds32(st + L::LK + 16 * (g + 8) + 4 * c4);
      const __half2 sz0 = u2h2(lds32(st + L::LKS + 4 * g));
      const __half2 sz1 = u2h2(lds32(st + L::LKS + 4 * (g + 8)));
      const __half2 s0 = __low2half2(sz0), z0 = __high2half2(sz0);
      const __half2 s1 = __low2half2(sz1), z1 = __high2half2(sz1);
      const __half2 k1024 = __float2half2_rn(1024.f);
      auto deq = [&](uint32_t x, __half2 sc, __half2 zz) -> uint32_t {
        return h2u(__hfma2(__hsub2(u2h2((x & kN0) | kMagic), k1024), sc, zz));
      };
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        const uint32_t x0 = w0 >> (8 * ks), x1 = w1 >> (8 * ks);
        a[ks][0] = deq(x0, s0, z0);
        a[ks][1] = deq(x1, s1, z1);
        a[ks][2] = deq(x0 >> 4, s0, z0);
        a[ks][3] = deq(x1 >> 4, s1, z1);
      }
    }
    // reconstruction K = L Bk (16 n-tiles of 8 dims) with fp32 accumulators,
    // one RoPE pair of n-tile couples at a time: n-tiles 2m, 2m + 1 hold dims
    // i and n-tiles 2m + 8, 2m + 9 dims i + 64.  Each sum is rounded to f16 once,
    // then R_delta rotates the pair (rows g and g + 8) in f16x2.
    uint32_t kf[16][2];
    const uint32_t bk_s = sm_s + kvh * kBkHead + ldsm_off;
    const int dl0 = (kPT * jt) % L::GROUP + g;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      float c[4][4];
#pragma unroll
      for (int x = 0; x < 4; ++x) c[x][0] = c[x][1] = c[x][2] = c[x][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        uint32_t b[4];
        ldsm_x4_trans(b, bk_s + ks * 16 * kBkRow + m * 32);
        mma16816(c[0], a[ks], b[0], b[1]);
        mma16816(c[1], a[ks], b[2], b[3]);
        ldsm_x4_trans(b, bk_s + ks * 16 * kBkRow + (m + 4) * 32);
        mma16816(c[2], a[ks], b[0], b[1]);
        mma16816(c[3], a[ks], b[2], b[3]);
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const uint4 t = lds128(rope_s + (dl0 + 8 * r) * kRopeRow + 64 * m);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int nt = 2 * m + h;
          const __half2 cs = u2h2(h ? t.z : t.x), sn = u2h2(h ? t.w : t.y);
          const __half2 lo = __floats2half2_rn(c[h][2 * r], c[h][2 * r + 1]);
          const __half2 hi = __floats2half2_rn(c[2 + h][2 * r], c[2 + h][2 * r + 1]);
          kf[nt][r] = h2u(__hfma2(lo, cs, __hneg2(__hmul2(hi, sn))));
          kf[nt + 8][r] = h2u(__hfma2(hi, cs, __hmul2(lo, sn)));
        }
      }
    }
    // scores: k-step j takes n-tiles 2j, 2j + 1 as they are
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t af[4] = {kf[2 * j][0], kf[2 * j][1], kf[2 * j + 1][0], kf[2 * j + 1][1]};
      if (j & 1) mma16816(s1, af, qb[j][0], qb[j][1]);
      else mma16816(s0, af, qb[j][0], qb[j][1]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) s[i] = s0[i] + s1[i];
    if constexpr (TAIL) {
      if (g >= nt) s[0] = s[1] = -INFINITY;
      if (g + 8 >= nt) s[2] = s[3] = -INFINITY;
    }
  };

  auto values = [&](auto tail_tag, const uint8_t* st, int nt, const float (&s)[4]) {
    constexpr bool TAIL = decltype(tail_tag)::value;
    const bool ok0 = !TAIL || g < nt, ok1 = !TAIL || g + 8 < nt;
    const bool need = s[0] > m_thr[0] || s[2] > m_thr[0] || s[1] > m_thr[1] || s[3] > m_thr[1];
    if (__any_sync(0xffffffffu, need)) {
      float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      const float n0 = fmaxf(m_ref[0], mx0), n1 = fmaxf(m_ref[1], mx1);
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
    pv[0] = ex2_approx(s[0] - m_ref[0]);
    pv[1] = ex2_approx(s[1] - m_ref[1]);
    pv[2] = ex2_approx(s[2] - m_ref[0]);
    pv[3] = ex2_approx(s[3] - m_ref[1]);
    if constexpr (TAIL) {
      if (!ok0) pv[0] = pv[1] = 0.f;
      if (!ok1) pv[2] = pv[3] = 0.f;
    }
    l_sum[0] += pv[0] + pv[2];
    l_sum[1] += pv[1] + pv[3];
    const __half2 hp01 = __floats2half2_rn(pv[0], pv[1]);
    const __half2 hp23 = __floats2half2_rn(pv[2], pv[3]);
#pragma unroll
    for (int v = 0; v < NVG; ++v) {
      __half2 sz_0 = u2h2(lds32(st + L::LVS + NVG * 4 * g + 4 * v));
      __half2 sz_1 = u2h2(lds32(st + L::LVS + NVG * 4 * (g + 8) + 4 * v));
      if constexpr (TAIL) {
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
      const uint32_t xA = prmt(lds32(lv), lds32(lv + RVB), sel);
      const uint32_t xB = prmt(lds32(lv + 8 * RVB), lds32(lv + 9 * RVB), sel);
      auto cen = [](uint32_t x, uint32_t c) { return h2u(__hsub2(u2h2(x), u2h2(c))); };
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

  int ji = kPDist, s_iss = kPDist, s_use = 0;
  auto step = [&]() -> const uint8_t* {
    __syncwarp();
    if ((ji & 31) == 0) {
      rows_cur = rows_next;
      rows_next = tile_row(ji + 32 + lane);
    }
    const int r = __shfl_sync(0xffffffffu, rows_cur, ji & 31);
    if (ji < n_tiles) issue(s_iss, r);
    cp_commit();
    ++ji;
    s_iss = s_iss + 1 == kPStages ? 0 : s_iss + 1;
    cp_wait<kPDist>();
    __syncwarp();
    const uint8_t* st = ring + s_use * L::BYTES;
    s_use = s_use + 1 == kPStages ? 0 : s_use + 1;
    return st;
  };
  auto score_tile = [&](bool tail, const uint8_t* st, int jt, int nt, float (&s)[4]) {
    const int J = (kPT * jt) / L::GROUP;
    if (J != cur_J) {
      rotate_q(J);
      cur_J = J;
    }
    if (tail) scores(std::true_type(), st, jt, nt, s);
    else scores(std::false_type(), st, jt, kPT, s);
  };

  const int tail_nt = p.n_tokens % kPT;
  int u = t_first / wk.tpu, jt0 = t_first % wk.tpu;
  for (int jj = 0; jj < n_tiles;) {
    const int cnt = min(wk.tpu - jt0, n_tiles - jj);
    const bool tail = tail_nt != 0 && jt0 + cnt == wk.tpu;
    cur_u = u;
    cur_slot = gw - (int)(((long long)u * wk.tpu) / wk.W);
    reset(u);
    float s_cur[4], s_nxt[4];
    const uint8_t* st_cur = step();
    score_tile(tail && cnt == 1, st_cur, jt0, tail_nt, s_cur);
    for (int k = 0; k + 1 < cnt; ++k) {
      const uint8_t* st_nxt = step();
      score_tile(tail && k + 2 == cnt, st_nxt, jt0 + k + 1, tail_nt, s_nxt);
      values(std::false_type(), st_cur, kPT, s_cur);
      st_cur = st_nxt;
#pragma unroll
      for (int i = 0; i < 4; ++i) s_cur[i] = s_nxt[i];
    }
    if (tail) values(std::true_type(), st_cur, tail_nt, s_cur);
    else values(std::false_type(), st_cur, kPT, s_cur);
    write_partial();
    jj += cnt;
    ++u;
    jt0 = 0;
  }
  cp_wait<0>();
}

template <int RV>
cudaError_t launch_p(const Params& p, const PWork& wk, int grid, cudaStream_t s) {
  using L = PStage<RV>;
  cudaError_t e = cudaFuncSetAttribute(rope_mma_kernel<RV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  rope_mma_kernel<RV><<<grid, kPThreads, L::SMEM, s>>>(p, wk);
  return cudaGetLastError();
}

}  // namespace

bool rope_mma_supported(const Params& p) {
  if (p.kind != KVC_LOWRANK || !p.rope || p.bits != 4 || p.g != 32 || p.d != 128) return false;
  if (p.rk != kPRank || (p.rv != 32 && p.rv != 48 && p.rv != 64) || p.resid) return false;
  if (p.page != 0 && p.page != kPT) return false;
  if (p.L != 1 || p.seq_lens || p.n_tokens <= 0 || p.G < 1 || p.G > 8) return false;
  if (p.Hkv > kPMaxHkv || p.tmax % kPT) return false;
  const long long rows = p.page ? (long long)p.n_pages * p.Hkv * kPT : (long long)p.B * p.Hkv * p.tmax;
  return rows < (1LL << 31) && p.vdim == p.rv;
}

void rope_mma_plan(const Params& p, int* grid, int* W, int* tpu, int* slots) {
  const int t = (p.n_tokens + kPT - 1) / kPT;
  const long long total = (long long)p.B * p.Hkv * t;
  const long long warps_max = (long long)kNumSMs * kPWarps;
  const long long w = (total + warps_max - 1) / warps_max;
  const long long n_warps = (total + w - 1) / w;
  *grid = (int)((n_warps + kPWarps - 1) / kPWarps);
  *W = (int)w;
  *tpu = t;
  *slots = (int)((t + w - 1) / w + 1);
}

int rope_mma_slots(int batch, int n_kv_heads, int n_tokens) {
  const int t = (n_tokens + kPT - 1) / kPT;
  const long long total = (long long)batch * n_kv_heads * t;
  const long long warps_max = (long long)kNumSMs * kPWarps;
  const long long w = (total + warps_max - 1) / warps_max;
  return (int)((t + w - 1) / w + 1);
}

cudaError_t launch_rope_mma(const Params& p, cudaStream_t s) {
  int grid, W, tpu, slots;
  rope_mma_plan(p, &grid, &W, &tpu, &slots);
  const PWork wk{W, tpu, p.B * p.Hkv * tpu};
  switch (p.rv) {
    case 32: return launch_p<32>(p, wk, grid, s);
    case 48: return launch_p<48>(p, wk, grid, s);
    default: return launch_p<64>(p, wk, grid, s);
  }
}

}  // namespace kvc
