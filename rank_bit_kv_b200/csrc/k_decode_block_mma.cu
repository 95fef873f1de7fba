// Split-T decode on the block-shared latent (one INT4 latent row of width 512
// per token, shared by the KV heads of several layers; BellowsKV "Share the
// Input, Not the Cache"), for the absorbed queries q~ = W_k^l[:, head] q of all
// layers at once.
//
// One CTA per (token range, batch row, group of 32 absorbed queries); 8 warps.
// Per tile of 32 tokens:
//   1. the tile's codes and group scales arrive by 16-byte cp.async (double
//      buffered) and are dequantised once, x = (c - 8) s, into an f16 tile in
//      shared memory that every warp reads;
//   2. scores S = X Q~^T on mma.sync m16n8k16 (warp w: tokens 16 (w & 1).., queries
//      8 (w >> 1)..; K = 512), operands by ldmatrix;
//   3. the per-query tile maxima meet in shared memory; every warp keeps the
//      same lazily raised reference maxima (raised when a score exceeds them by
//      more than 8 in log2 units) and writes its probabilities P (f16);
//   4. O (32 queries x 512) += P X on mma.sync, warp w owning latent columns
//      64 w .. 64 w + 63 (64 fp32 accumulators per thread).
// The partials (O, m, l) per query go to the combine, which applies W_v^l.
// Inside each 8-column block of the latent, shared-memory position p holds
// latent index perm(p) = (p >> 1) | ((p & 1) << 2) (the order in which one
// 32-bit word of codes unpacks into f16 pairs); the queries are stored in the
// same order and the partials are written back in latent order.
#include <math.h>

#include "kvc_device.cuh"
#include "tc_util.cuh"

namespace kvc {
namespace {

using namespace tc;

constexpr int kXT = 32;                  // tokens per tile
constexpr int kXQ = 32;                  // absorbed queries per CTA
constexpr int kXD = 512;                 // latent width
constexpr int kXG = 64;                  // latent columns per scale group
constexpr int kXWarps = 8;
constexpr int kXThreads = 32 * kXWarps;
constexpr int kXRow = kXD * 2 + 16;      // bytes per f16 row of Q~ / X (padded: ldmatrix conflict-free)
constexpr int kPRowB = kXT * 2 + 16;     // bytes per row of P (queries x tokens)
constexpr int kRawCodes = kXT * kXD / 2; // 8 KB of codes per tile
constexpr int kRawScales = kXT * (kXD / kXG) * 2;
constexpr int kRawStage = kRawCodes + kRawScales;
constexpr int OFF_Q = 0;
constexpr int OFF_X = OFF_Q + kXQ * kXRow;
constexpr int OFF_P = OFF_X + kXT * kXRow;
constexpr int OFF_RAW = OFF_P + kXQ * kPRowB;
constexpr int OFF_RED = OFF_RAW + 2 * kRawStage;
constexpr int kXSmem = OFF_RED + 2 * kXQ * 4 + 2 * kXQ * 4;

__device__ __forceinline__ void cp16(uint32_t dst, const void* src, int n) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ uint32_t h2u(__half2 x) { return *reinterpret_cast<uint32_t*>(&x); }
__device__ __forceinline__ __half2 u2h(uint32_t x) { return *reinterpret_cast<__half2*>(&x); }

// latent index held by shared-memory position p (within an 8-column block)
__host__ __device__ constexpr int xperm(int p) { return (p >> 1) | ((p & 1) << 2); }

__global__ void __launch_bounds__(kXThreads, 2) block_mma_kernel(Params p) {
  extern __shared__ __align__(128) uint8_t xsm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c4 = lane & 3;
  const int chunks = p.L * p.Hq / kXQ;
  const int b = blockIdx.y / chunks, chunk = blockIdx.y % chunks;
  const int T = p.n_tokens;
  const int t_a = blockIdx.x * p.split_len, t_b = min(T, t_a + p.split_len);
  const uint32_t sm = smem_u32(xsm);
  float* red = reinterpret_cast<float*>(xsm + OFF_RED);       // [2][32] tile maxima
  float* lsh = red + 2 * kXQ;                                  // [2][32] row sums at the end
  auto qrow = [&](int i) -> size_t {                           // global query row of local query i
    const int qi = chunk * kXQ + i, ll = qi / p.Hq, hh = qi % p.Hq;
    return ((size_t)ll * p.B + b) * p.Hq + hh;
  };

  // ---- the CTA's absorbed queries as f16 rows (softmax scale and log2 e folded)
  for (int e = tid; e < kXQ * kXD / 2; e += kXThreads) {
    const int i = e / (kXD / 2), pp = 2 * (e % (kXD / 2));    // positions pp, pp + 1
    const float* qt = p.qt + qrow(i) * p.qdim;
    const int base = pp & ~7;
    const float a = qt[base + xperm(pp & 7)] * p.scale_log2;
    const float c = qt[base + xperm((pp + 1) & 7)] * p.scale_log2;
    *reinterpret_cast<__half2*>(xsm + OFF_Q + i * kXRow + pp * 2) = __floats2half2_rn(a, c);
  }

  // ---- tile staging: codes [32][256 B] and scales [32][16 B], zero past the end
  const uint8_t* codes = p.lk + (size_t)b * p.tmax * (kXD / 2);
  const uint8_t* scales = reinterpret_cast<const uint8_t*>(p.lksz) + (size_t)b * p.tmax * 16;
  auto stage = [&](int t0, int buf) {
    const uint32_t dst = sm + OFF_RAW + buf * kRawStage;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int c = tid + kXThreads * k;                     // chunk: token c / 16, part c % 16
      const int tok = t0 + (c >> 4);
      const bool ok = tok < t_b;
      cp16(dst + 16 * c, codes + (size_t)(ok ? tok : t_a) * (kXD / 2) + 16 * (c & 15), ok ? 16 : 0);
    }
    if (tid < kXT) {
      const int tok = t0 + tid;
      const bool ok = tok < t_b;
      cp16(dst + kRawCodes + 16 * tid, scales + (size_t)(ok ? tok : t_a) * 16, ok ? 16 : 0);
    }
  };

  // ---- per-thread state
  float o[2][8][4];                      // O: query m-tile, column n-tile (cols 64 warp + 8 n)
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int n = 0; n < 8; ++n) o[a][n][0] = o[a][n][1] = o[a][n][2] = o[a][n][3] = 0.f;
  float m_lane = -INFINITY;              // reference maximum of query `lane` (same in every warp)
  float l_part[2] = {0.f, 0.f};          // row sums of queries 8 (w >> 1) + 2 c4 + e, this warp's tokens
  const int mt = warp & 1, nq = warp >> 1;

  int buf = 0;
  if (t_a < t_b) stage(t_a, 0);
  cp_commit();
  for (int t0 = t_a; t0 < t_b; t0 += kXT) {
    const int nt = min(kXT, t_b - t0);
    if (t0 + kXT < t_b) stage(t0 + kXT, buf ^ 1);
    cp_commit();
    cp_wait<1>();
    __syncthreads();                     // S1: raw tile landed; the previous tile's V is done

    // ---- 1. dequantise: thread -> token tid / 8, scale group tid % 8 (64 columns)
    {
      const int tk = tid >> 3, gr = tid & 7;
      const uint8_t* raw = xsm + OFF_RAW + buf * kRawStage;
      const uint4 w0 = *reinterpret_cast<const uint4*>(raw + tk * 256 + gr * 32);
      const uint4 w1 = *reinterpret_cast<const uint4*>(raw + tk * 256 + gr * 32 + 16);
      const __half s = *reinterpret_cast<const __half*>(raw + kRawCodes + tk * 16 + gr * 2);
      const __half2 s2 = __half2half2(s), k1032 = __float2half2_rn(1032.f);
      const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      uint8_t* dst = xsm + OFF_X + tk * kXRow + gr * kXG * 2;
#pragma unroll
      for (int wi = 0; wi < 8; ++wi) {
        const uint32_t w = ws[wi];
        uint32_t h[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          // nibbles j and j + 4 (latent 8 wi + j, 8 wi + j + 4) -> positions 2j, 2j + 1
          const uint32_t x = ((w >> (4 * j)) & 0x000F000Fu) | 0x64006400u;
          h[j] = h2u(__hmul2(__hsub2(u2h(x), k1032), s2));
        }
        *reinterpret_cast<uint4*>(dst + wi * 16) = make_uint4(h[0], h[1], h[2], h[3]);
      }
    }
    __syncthreads();                     // S2: the f16 tile is complete

    // ---- 2. scores: tokens 16 mt + {g, g + 8}, queries 8 nq + 2 c4 + {0, 1}
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const uint32_t xa = sm + OFF_X + (16 * mt + (lane & 15)) * kXRow + 16 * (lane >> 4);
      const uint32_t qa = sm + OFF_Q + (8 * nq + (lane & 7)) * kXRow + 16 * (lane >> 3);
#pragma unroll 4
      for (int kk = 0; kk < kXD / 32; ++kk) {              // two k-steps of 16 per round
        uint32_t bq[4];
        ldsm_x4(bq, qa + kk * 64);                         // k-steps 2kk, 2kk + 1: (b0, b1) each
        uint32_t a0[4], a1[4];
        ldsm_x4(a0, xa + kk * 64);
        ldsm_x4(a1, xa + kk * 64 + 32);
        mma16816(sa, a0, bq[0], bq[1]);
        mma16816(sb, a1, bq[2], bq[3]);
      }
    }
    float s[4] = {sa[0] + sb[0], sa[1] + sb[1], sa[2] + sb[2], sa[3] + sb[3]};
    if (g >= nt - 16 * mt) s[0] = s[1] = -INFINITY;
    if (g + 8 >= nt - 16 * mt) s[2] = s[3] = -INFINITY;

    // ---- 3. tile maxima per query -> shared memory
    {
      float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
#pragma unroll
      for (int o2 = 4; o2 < 32; o2 <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o2));
      }
      if (g == 0) {
        red[mt * kXQ + 8 * nq + 2 * c4] = mx0;
        red[mt * kXQ + 8 * nq + 2 * c4 + 1] = mx1;
      }
    }
    __syncthreads();                     // S3: every tile maximum is in
    // every warp updates the same reference maxima: lane q owns query q
    const float tmax = fmaxf(red[lane], red[kXQ + lane]);
    const bool raise = tmax > m_lane + 8.f;
    float alpha = 1.f;
    if (raise) {
      alpha = ex2_approx(m_lane - tmax);   // 0 on the first tile
      m_lane = tmax;
    }
    if (__any_sync(0xffffffffu, raise)) {
      // rescale O rows (queries 16 a + g, 16 a + g + 8) and the row sums
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const float f0 = __shfl_sync(0xffffffffu, alpha, 16 * a + g);
        const float f1 = __shfl_sync(0xffffffffu, alpha, 16 * a + g + 8);
#pragma unroll
        for (int n = 0; n < 8; ++n) {
          o[a][n][0] *= f0;
          o[a][n][1] *= f0;
          o[a][n][2] *= f1;
          o[a][n][3] *= f1;
        }
      }
      l_part[0] *= __shfl_sync(0xffffffffu, alpha, 8 * nq + 2 * c4);
      l_part[1] *= __shfl_sync(0xffffffffu, alpha, 8 * nq + 2 * c4 + 1);
    }
    {
      const float m0 = __shfl_sync(0xffffffffu, m_lane, 8 * nq + 2 * c4);
      const float m1 = __shfl_sync(0xffffffffu, m_lane, 8 * nq + 2 * c4 + 1);
      const float p0 = ex2_approx(s[0] - m0), p1 = ex2_approx(s[1] - m1);
      const float p2 = ex2_approx(s[2] - m0), p3 = ex2_approx(s[3] - m1);
      l_part[0] += p0 + p2;
      l_part[1] += p1 + p3;
      // P [query][token], f16
      __half* pr = reinterpret_cast<__half*>(xsm + OFF_P);
      const int q0 = 8 * nq + 2 * c4, tk = 16 * mt + g;
      pr[q0 * (kPRowB / 2) + tk] = __float2half_rn(p0);
      pr[(q0 + 1) * (kPRowB / 2) + tk] = __float2half_rn(p1);
      pr[q0 * (kPRowB / 2) + tk + 8] = __float2half_rn(p2);
      pr[(q0 + 1) * (kPRowB / 2) + tk + 8] = __float2half_rn(p3);
    }
    __syncthreads();                     // S4: P is complete

    // ---- 4. O (queries x columns 64 w ..) += P X
    {
      uint32_t pa[2][2][4];              // [query m-tile][token k-step]
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int kt = 0; kt < 2; ++kt)
          ldsm_x4(pa[a][kt], sm + OFF_P + (16 * a + (lane & 15)) * kPRowB + 32 * kt + 16 * (lane >> 4));
#pragma unroll
      for (int kt = 0; kt < 2; ++kt) {
#pragma unroll
        for (int n2 = 0; n2 < 4; ++n2) {                   // column n-tiles 2 n2, 2 n2 + 1
          uint32_t bx[4];
          ldsm_x4_t(bx, sm + OFF_X + (16 * kt + (lane & 7) + 8 * ((lane >> 3) & 1)) * kXRow +
                            (64 * warp + 16 * n2 + 8 * (lane >> 4)) * 2);
#pragma unroll
          for (int a = 0; a < 2; ++a) {
            mma16816(o[a][2 * n2], pa[a][kt], bx[0], bx[1]);
            mma16816(o[a][2 * n2 + 1], pa[a][kt], bx[2], bx[3]);
          }
        }
      }
    }
    buf ^= 1;
  }
  cp_wait<0>();

  // ---- partials: row sums of both token halves, then O, m, l per query
#pragma unroll
  for (int e = 0; e < 2; ++e) {
#pragma unroll
    for (int o2 = 4; o2 < 32; o2 <<= 1) l_part[e] += __shfl_xor_sync(0xffffffffu, l_part[e], o2);
  }
  __syncthreads();
  if (g == 0) {
    lsh[mt * kXQ + 8 * nq + 2 * c4] = l_part[0];
    lsh[mt * kXQ + 8 * nq + 2 * c4 + 1] = l_part[1];
  }
  __syncthreads();
  const size_t rows = (size_t)p.L * p.B * p.Hq;
  const int pst = p.vdim + 2;
#pragma unroll
  for (int a = 0; a < 2; ++a) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int q = 16 * a + g + 8 * r;
      float* dst = p.part + ((size_t)blockIdx.x * rows + qrow(q)) * pst;
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const int pos = 64 * warp + 8 * n + 2 * c4;       // positions pos, pos + 1
        dst[(pos & ~7) + xperm(pos & 7)] = o[a][n][2 * r];
        dst[(pos & ~7) + xperm((pos + 1) & 7)] = o[a][n][2 * r + 1];
      }
    }
  }
  if (warp == 0) {
    float* dst = p.part + ((size_t)blockIdx.x * rows + qrow(lane)) * pst;
    dst[p.vdim] = m_lane;
    dst[p.vdim + 1] = lsh[lane] + lsh[kXQ + lane];
  }
}

}  // namespace

bool block_mma_supported(const Params& p) {
  return p.kind == KVC_BLOCK_SHARED && p.bits == 4 && p.vbits == 0 && p.D == kXD &&
         p.g == kXG && p.d == 128 &&
         (p.L * p.Hq) % kXQ == 0 && !p.seq_lens && p.n_tokens > 0 && p.qdim == kXD &&
         p.vdim == kXD;
}

// splits of the token range per (batch row, query group), a whole number of tiles
void block_mma_plan(const Params& p, int* splits, int* split_len) {
  const int units = p.B * (p.L * p.Hq / kXQ);
  const int tiles = (p.n_tokens + kXT - 1) / kXT;
  int s = (2 * kNumSMs + units - 1) / units;
  if (s > tiles) s = tiles;
  if (s < 1) s = 1;
  const int per = (tiles + s - 1) / s;
  *split_len = per * kXT;
  *splits = (tiles + per - 1) / per;
}

int block_mma_slots(int batch, int n_layers, int n_q_heads, int n_tokens) {
  const int units = batch * (n_layers * n_q_heads / kXQ);
  const int tiles = (n_tokens + kXT - 1) / kXT;
  int s = (2 * kNumSMs + (units > 0 ? units : 1) - 1) / (units > 0 ? units : 1);
  if (s > tiles) s = tiles;
  return s < 1 ? 1 : s;
}

cudaError_t launch_block_mma(const Params& p, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(block_mma_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kXSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.S, p.B * (p.L * p.Hq / kXQ));
  block_mma_kernel<<<grid, kXThreads, kXSmem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace kvc
