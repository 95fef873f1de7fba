// Split-T decode on a dense bf16 K/V cache (the baseline the compressed layouts
// are compared with: the same decode step on the uncompressed cache, on the
// same library and GPU).
//
// Every warp streams its own contiguous range of 16-token tiles (the ranges of
// all warps of the grid are equal, so every SM moves the same bytes; a range may
// cross from one (batch row, KV head) unit to the next, with one partial per
// unit part).  A warp keeps a 4-deep ring of K and V tiles in shared memory,
// filled with 16-byte cp.async copies into rows padded to 272 bytes (ldmatrix
// reads them without bank conflicts), and for each tile
//   - scores S = K q^T with mma.sync m16n8k16 (bf16 operands, fp32 accumulate;
//     the GQA group of query heads is the N dimension, padded to 8),
//   - keeps an online softmax with a lazily raised reference maximum,
//   - accumulates acc^T += V^T P with P split into a bf16 high and low part so
//     that the probabilities keep ~16 bits.
// The combine kernel merges the partials (o = acc / l).
#include <math.h>

#include "kvc_device.cuh"
#include "tc_util.cuh"

namespace kvc {
namespace {

using namespace tc;

constexpr int kDT = 16;                  // tokens per tile
constexpr int kWarps = 4;
constexpr int kDThreads = 32 * kWarps;
constexpr int kDStages = 4;
constexpr int kHd = 128;                 // head dim handled
constexpr int kRowB = 272;               // smem bytes per token row (256 + 16 pad)
constexpr int kTileB = kDT * kRowB;      // one K or V tile
constexpr int kStageB = 2 * kTileB;      // K then V
constexpr int kWarpB = kDStages * kStageB;
constexpr int kSmem = kWarps * kWarpB;
constexpr int kMaxG = 8;                 // query heads per KV head (N of the MMA)

struct DWork {
  int W, tpu, total;                     // tiles per warp, tiles per unit, all tiles
};

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(row_addr)));
}

__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__global__ void __launch_bounds__(kDThreads, 1) dense_tc_kernel(Params p, DWork wk) {
  extern __shared__ __align__(128) uint8_t dsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * kWarps + warp;           // global warp = partial slot owner
  const int t_first = gw * wk.W;
  const int n_tiles = min(wk.W, wk.total - t_first);
  if (n_tiles <= 0) return;
  uint8_t* ring = dsm + warp * kWarpB;
  const int G = p.G;
  const int g = lane >> 2, c4 = lane & 3;
  const size_t rows_q = (size_t)p.B * p.Hq;
  const int pst = p.vdim + 2;

  // copy tile jj of the range into its ring stage (zero-filled past the end)
  auto issue = [&](int jj) {
    const int t = t_first + jj;
    const int u = t / wk.tpu, jt = t % wk.tpu;
    const int nt = min(kDT, p.n_tokens - jt * kDT);
    const size_t row0 = (size_t)u * p.tmax + (size_t)jt * kDT;
    const uint8_t* ks = reinterpret_cast<const uint8_t*>(p.kd) + row0 * (kHd * 2);
    const uint8_t* vs = reinterpret_cast<const uint8_t*>(p.vd) + row0 * (kHd * 2);
    uint8_t* st = ring + (jj % kDStages) * kStageB;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = lane + 32 * i, r = c >> 4, col = c & 15;
      const int nb = r < nt ? 16 : 0;
      const size_t go = (size_t)(r < nt ? r : 0) * (kHd * 2) + col * 16;
      cp_async16(st + r * kRowB + col * 16, ks + go, nb);
      cp_async16(st + kTileB + r * kRowB + col * 16, vs + go, nb);
    }
  };

  // prologue: the first kDStages - 1 tiles in flight
#pragma unroll
  for (int i = 0; i < kDStages - 1; ++i) {
    if (i < n_tiles) issue(i);
    cp_async_commit();
  }

  uint32_t qb[8][2];                     // q of head g as B fragments (bf16x2), 0 for g >= G
  float m_ref[2] = {-INFINITY, -INFINITY}, m_thr[2] = {-INFINITY, -INFINITY};
  float l_sum[2] = {0.f, 0.f}, acc[8][4] = {};
  int cur_u = -1, cur_slot = 0;
  auto write_partial = [&]() {
    float l0 = l_sum[0], l1 = l_sum[1];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    const int b = cur_u / p.Hkv, kvh = cur_u % p.Hkv;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = 2 * c4 + e;
      if (h < G) {
        const size_t qr = (size_t)b * p.Hq + kvh * G + h;
        float* dst = p.part + ((size_t)cur_slot * rows_q + qr) * pst;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          dst[16 * mt + g] = acc[mt][e];
          dst[16 * mt + g + 8] = acc[mt][2 + e];
        }
        if (g == 0) {
          dst[p.vdim] = m_ref[e];
          dst[p.vdim + 1] = e ? l1 : l0;
        }
      }
    }
  };

  for (int jj = 0; jj < n_tiles; ++jj) {
    const int t = t_first + jj;
    const int u = t / wk.tpu, jt = t % wk.tpu;
    const int nt = min(kDT, p.n_tokens - jt * kDT);
    if (u != cur_u) {
      if (cur_u >= 0) write_partial();
      cur_u = u;
      cur_slot = gw - (int)(((long long)u * wk.tpu) / wk.W);
      const int b = u / p.Hkv, kvh = u % p.Hkv;
      // padding heads g >= G read head G - 1 and are zeroed
      const __nv_bfloat16* qq = p.q + ((size_t)b * p.Hq + kvh * G + min(g, G - 1)) * kHd;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        qb[kk][0] = g < G ? *reinterpret_cast<const uint32_t*>(qq + 16 * kk + 2 * c4) : 0u;
        qb[kk][1] = g < G ? *reinterpret_cast<const uint32_t*>(qq + 16 * kk + 8 + 2 * c4) : 0u;
      }
      m_ref[0] = m_ref[1] = m_thr[0] = m_thr[1] = -INFINITY;
      l_sum[0] = l_sum[1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
    }
    // keep kDStages - 1 tiles in flight, then wait for tile jj
    if (jj + kDStages - 1 < n_tiles) issue(jj + kDStages - 1);
    cp_async_commit();
    cp_async_wait<kDStages - 1>();
    __syncwarp();
    const uint8_t* kt = ring + (jj % kDStages) * kStageB;
    const uint8_t* vt = kt + kTileB;
    // ---- scores (rows g, g + 8 = tokens; columns 2c4, 2c4 + 1 = heads)
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t a[4];
      ldmatrix_x4(a, kt + (lane & 15) * kRowB + (2 * kk + (lane >> 4)) * 16);
      if (kk & 1) mma_bf16(sb, a, qb[kk][0], qb[kk][1]);
      else mma_bf16(sa, a, qb[kk][0], qb[kk][1]);
    }
    const bool v0 = g < nt, v1 = g + 8 < nt;
    const float s0 = v0 ? (sa[0] + sb[0]) * p.scale_log2 : -INFINITY;
    const float s1 = v0 ? (sa[1] + sb[1]) * p.scale_log2 : -INFINITY;
    const float s2 = v1 ? (sa[2] + sb[2]) * p.scale_log2 : -INFINITY;
    const float s3 = v1 ? (sa[3] + sb[3]) * p.scale_log2 : -INFINITY;
    // ---- online softmax of this warp (lazy maximum, raised by more than 2^8)
    const bool need = s0 > m_thr[0] || s2 > m_thr[0] || s1 > m_thr[1] || s3 > m_thr[1];
    if (__any_sync(0xffffffffu, need)) {
      float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      const float n0 = fmaxf(m_ref[0], mx0), n1 = fmaxf(m_ref[1], mx1);
      const float a0 = ex2_approx(m_ref[0] - n0), a1 = ex2_approx(m_ref[1] - n1);
      l_sum[0] *= a0;
      l_sum[1] *= a1;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        acc[mt][0] *= a0;
        acc[mt][2] *= a0;
        acc[mt][1] *= a1;
        acc[mt][3] *= a1;
      }
      m_ref[0] = n0;
      m_ref[1] = n1;
      m_thr[0] = n0 + 8.f;
      m_thr[1] = n1 + 8.f;
    }
    float pv[4];
    pv[0] = v0 ? ex2_approx(s0 - m_ref[0]) : 0.f;
    pv[1] = v0 ? ex2_approx(s1 - m_ref[1]) : 0.f;
    pv[2] = v1 ? ex2_approx(s2 - m_ref[0]) : 0.f;
    pv[3] = v1 ? ex2_approx(s3 - m_ref[1]) : 0.f;
    l_sum[0] += pv[0] + pv[2];
    l_sum[1] += pv[1] + pv[3];
    // P (token x head) as B fragments, high and low bf16 parts
    const uint32_t h01 = pack_bf2(pv[0], pv[1]), h23 = pack_bf2(pv[2], pv[3]);
    const __nv_bfloat162 hb01 = *reinterpret_cast<const __nv_bfloat162*>(&h01);
    const __nv_bfloat162 hb23 = *reinterpret_cast<const __nv_bfloat162*>(&h23);
    const uint32_t l01 = pack_bf2(pv[0] - __low2float(hb01), pv[1] - __high2float(hb01));
    const uint32_t l23 = pack_bf2(pv[2] - __low2float(hb23), pv[3] - __high2float(hb23));
    const uint32_t ph0 = movmatrix_trans(h01), ph1 = movmatrix_trans(h23);
    const uint32_t pl0 = movmatrix_trans(l01), pl1 = movmatrix_trans(l23);
    // ---- acc^T (dim x head) += V^T (dim x token) P (token x head)
    const int tok = (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      uint32_t a[4];
      ldmatrix_x4_trans(a, vt + tok * kRowB + (2 * mt + ((lane >> 3) & 1)) * 16);
      mma_bf16(acc[mt], a, ph0, ph1);
      mma_bf16(acc[mt], a, pl0, pl1);
    }
    __syncwarp();                        // this stage is refilled next iteration
  }
  cp_async_wait<0>();
  write_partial();
}

}  // namespace

bool dense_tc_supported(const Params& p) {
  return p.kind == KVC_DENSE_BF16 && p.d == kHd && p.G >= 1 && p.G <= kMaxG && p.L == 1 &&
         !p.seq_lens && p.n_tokens > 0 && p.vdim == kHd;
}

// Equal contiguous tile ranges per warp: a unit of tpu tiles spans at most
// ceil(tpu / W) + 1 warps, each writing one partial.
void dense_tc_plan(const Params& p, int* grid, int* W, int* tpu, int* slots) {
  const int t = (p.n_tokens + kDT - 1) / kDT;
  const long long total = (long long)p.B * p.Hkv * t;
  const long long warps_max = (long long)kNumSMs * kWarps;
  const long long w = (total + warps_max - 1) / warps_max;
  const long long n_warps = (total + w - 1) / w;
  *grid = (int)((n_warps + kWarps - 1) / kWarps);
  *W = (int)w;
  *tpu = t;
  *slots = (int)((t + w - 1) / w + 1);
}

int dense_tc_slots(int batch, int n_kv_heads, int n_tokens) {
  const int t = (n_tokens + kDT - 1) / kDT;
  const long long total = (long long)batch * n_kv_heads * t;
  const long long warps_max = (long long)kNumSMs * kWarps;
  const long long w = (total + warps_max - 1) / warps_max;
  return (int)((t + w - 1) / w + 1);
}

cudaError_t launch_dense_tc(const Params& p, cudaStream_t s) {
  int grid, W, tpu, slots;
  dense_tc_plan(p, &grid, &W, &tpu, &slots);
  DWork wk{W, tpu, p.B * p.Hkv * tpu};
  cudaError_t e =
      cudaFuncSetAttribute(dense_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  dense_tc_kernel<<<grid, kDThreads, kSmem, s>>>(p, wk);
  return cudaGetLastError();
}

}  // namespace kvc
