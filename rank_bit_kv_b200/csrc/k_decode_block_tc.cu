// Split-T decode on the block-shared latent with tcgen05 (BellowsKV "Share
// the Input, Not the Cache": one INT4 latent row of width 512 per token serves
// the KV heads of every layer of the block).  For the 128 absorbed queries
// q~ = W_k^l[:, head] q of a batch row (4 layers x 32 heads) the step is a
// dense contraction with M = 128:
//   S = Q~ X^T (K = 512),  online softmax over the tokens,  O += P X (N = 512).
// O is 128 x 512 fp32 -- all of an SM's tensor memory -- so the two halves of
// the latent columns go to two CTAs; each CTA forms the whole S tile (the
// scores need every latent column) and accumulates its own 256 columns of O.
//
// One CTA per (token range, batch row, half); 9 warps:
//   warps 0-3  softmax: thread = query row = TMEM lane; reads its 64 scores
//              with tcgen05.ld, keeps (m, l) with a lazily raised maximum,
//              writes its probabilities as f16 into TMEM (the A operand of the
//              O MMA) and rescales its O row in TMEM when the maximum rises;
//   warps 4-7  producers: load the tiles' codes and scales from global memory
//              into registers two tiles ahead and dequantise x = (c - 8) s into
//              f16 core matrices in shared memory, the other half (read only
//              by the score MMAs) into one buffer, this CTA's half (read by
//              both MMAs) into two;
//   warp 8     allocates TMEM and issues the MMAs from one thread: S(i) over the
//              other half, then over this half, then O(i - 1).
// Every wait is bounded; a wait that gives up sets the workspace error word
// and the CTA winds down.
//
// Shared memory (all f16, no swizzle, core matrix = 8 rows x 16 bytes):
//   Q~  [128 queries x 512]   K-major A operand, LBO 128, SBO 8192
//   X   [64 tokens x 256] per half buffer; core matrix = 8 tokens x 8 latent
//       columns, latent groups 128 B apart, token groups 4096 B apart.  The
//       score MMA reads it K-major (N = tokens), the value MMA MN-major
//       (N = latent columns, K = tokens) -- the same bytes.
// Inside each group of 8 latent columns, position p holds column
// (p >> 1) | ((p & 1) << 2) (the order in which a word of INT4 codes unpacks
// into f16 pairs); Q~ uses the same order and the partials are written back in
// latent order.
//
// TMEM columns: S[2] 0..127 (64 each), P[2] 128..191 (32 each), O 256..511.
#include <math.h>

#include "kvc_device.cuh"
#include "tc_util.cuh"

namespace kvc {
namespace {

using namespace tc;

constexpr int kBT = 64;                  // tokens per tile (N of the score MMA)
constexpr int kBQ = 128;                 // absorbed queries (M)
constexpr int kBD = 512;                 // latent width
constexpr int kBH = 256;                 // latent columns per half
constexpr int kBG = 64;                  // latent columns per scale group
constexpr int kThreads = 288;
constexpr int kWarpProd = 4;             // first producer warp
constexpr int kWarpMma = 8;

constexpr int kHalfBytes = kBT * kBH * 2;          // 32 KB
constexpr int OFF_Q = 0;
constexpr int OFF_OWN = OFF_Q + kBQ * kBD * 2;     // 2 buffers
constexpr int OFF_OTH = OFF_OWN + 2 * kHalfBytes;
constexpr int OFF_BAR = OFF_OTH + kHalfBytes;
constexpr int kSmem = OFF_BAR + 256;

constexpr uint32_t kColS = 0;
constexpr uint32_t kColP = 128;
constexpr uint32_t kColO = 256;
constexpr uint32_t kTmemCols = 512;

struct Bars {
  uint64_t own_full[2], own_free[2], oth_full, oth_free;
  uint64_t s_full[2], s_free[2], p_full[2], o_done[2], drain;
  uint32_t tmem;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier area");
static_assert(kSmem <= 232448, "shared memory");

__device__ __forceinline__ uint32_t h2u(__half2 x) { return *reinterpret_cast<uint32_t*>(&x); }
__device__ __forceinline__ __half2 u2h(uint32_t x) { return *reinterpret_cast<__half2*>(&x); }
__device__ __forceinline__ float u2f(uint32_t x) { return __uint_as_float(x); }

// latent column held by position p of an 8-column group
__host__ __device__ constexpr int xperm(int p) { return (p >> 1) | ((p & 1) << 2); }

// A wait that every lane of the warp takes and whose outcome every lane shares
// (the tcgen05 loads and stores that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint32_t* err) {
  bool ok = mbar_wait(bar, parity, abort, err);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) *abort = 1;
  return ok;
}

// Codes and scales of one half of a token row for one producer thread:
// 128 latent columns = 64 bytes of codes + 2 fp16 scales.
struct HalfRegs {
  uint4 c[4];
  uint32_t s;
};

__device__ __forceinline__ void load_half(HalfRegs& r, const uint8_t* codes_row,
                                          const __half* scales_row, int half, int qh, bool ok) {
  if (ok) {
    const uint4* src = reinterpret_cast<const uint4*>(codes_row + half * (kBH / 2) + qh * 64);
#pragma unroll
    for (int u = 0; u < 4; ++u) r.c[u] = __ldg(src + u);
    r.s = __ldg(reinterpret_cast<const unsigned int*>(scales_row + half * 4 + qh * 2));
  } else {
#pragma unroll
    for (int u = 0; u < 4; ++u) r.c[u] = make_uint4(0u, 0u, 0u, 0u);
    r.s = 0u;                            // scale 0: the row dequantises to zeros
  }
}

// Dequantise one producer thread's 128 columns of token n into the half buffer.
__device__ __forceinline__ void store_half(uint8_t* buf, const HalfRegs& r, int n, int qh) {
  const __half2 k1032 = __float2half2_rn(1032.f);
  uint8_t* row = buf + (n >> 3) * 4096 + (n & 7) * 16;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint32_t sw = (u < 2) ? (r.s & 0xFFFFu) : (r.s >> 16);
    const __half2 s2 = u2h(sw | (sw << 16));
    const uint32_t ws[4] = {r.c[u].x, r.c[u].y, r.c[u].z, r.c[u].w};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      uint32_t h[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        // nibbles j and j + 4 (columns 8 g + j, 8 g + j + 4) -> positions 2 j, 2 j + 1
        const uint32_t x = ((ws[wi] >> (4 * j)) & 0x000F000Fu) | 0x64006400u;
        h[j] = h2u(__hmul2(__hsub2(u2h(x), k1032), s2));
      }
      const int lg = qh * 16 + u * 4 + wi;            // latent group within the half
      *reinterpret_cast<uint4*>(row + lg * 128) = make_uint4(h[0], h[1], h[2], h[3]);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) block_tc_kernel(Params p) {
  // the combine may launch now: its blocks take SMs as this grid's CTAs exit and
  // wait (griddepcontrol.wait) for the whole grid before reading the partials
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ __align__(1024) uint8_t sm[];
  Bars& bars = *reinterpret_cast<Bars*>(sm + OFF_BAR);
  volatile int* abort = &bars.abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int h = blockIdx.x & 1;
  const int b = (blockIdx.x >> 1) % p.B;
  const int split = (blockIdx.x >> 1) / p.B;
  const int T = p.n_tokens;
  const int t_a = split * p.split_len;
  const int t_b = min(T, t_a + p.split_len);
  const int n_tiles = t_a < t_b ? (t_b - t_a + kBT - 1) / kBT : 0;

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.own_full[i], 128);
      mbar_init(&bars.own_free[i], 1);
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.s_free[i], 4);
      mbar_init(&bars.p_full[i], 4);
      mbar_init(&bars.o_done[i], 1);
    }
    mbar_init(&bars.oth_full, 128);
    mbar_init(&bars.oth_free, 1);
    mbar_init(&bars.drain, 1);
    bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&bars.tmem, kTmemCols);
    tmem_relinquish();
  }

  // ---- absorbed queries -> f16 core matrices (softmax scale and log2 e folded)
  auto qrow = [&](int qi) -> size_t {
    const int ll = qi / p.Hq, hh = qi % p.Hq;
    return ((size_t)ll * p.B + b) * p.Hq + hh;
  };
  for (int e = tid; e < kBQ * (kBD / 8); e += kThreads) {
    const int qi = e >> 6, lg = e & 63;
    const float4* src = reinterpret_cast<const float4*>(p.qt + qrow(qi) * p.qdim + lg * 8);
    const float4 a = src[0], c = src[1];
    const float v[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
    uint32_t w[4];
#pragma unroll
    for (int pp = 0; pp < 4; ++pp)
      w[pp] = pack_h2(v[xperm(2 * pp)] * p.scale_log2, v[xperm(2 * pp + 1)] * p.scale_log2);
    *reinterpret_cast<uint4*>(sm + OFF_Q + (qi >> 3) * 8192 + lg * 128 + (qi & 7) * 16) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem;
  uint32_t* err = p.err;

  auto own_buf = [&](int bi) { return sm + OFF_OWN + bi * kHalfBytes; };
  uint8_t* oth_buf = sm + OFF_OTH;

  if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t id_s = idesc_f16(kBQ, kBT, 0, 0);
      const uint32_t id_o = idesc_f16(kBQ, kBH, 0, 1);
      // S(i) k-steps: the other half's 16, then this half's 16 (Q~ columns follow)
      const int other = 1 - h;
      for (int i = 0; i <= n_tiles; ++i) {
        if (i < n_tiles) {
          const int bi = i & 1;
          if (!mbar_wait(&bars.oth_full, i & 1, abort, err)) break;
          if (i >= 2 && !mbar_wait(&bars.s_free[bi], ((i - 2) >> 1) & 1, abort, err)) break;
          tc_fence_after();
          const uint32_t dS = tmem + kColS + 64 * bi;
#pragma unroll 1
          for (int k = 0; k < 16; ++k)
            mma_ss(dS, smem_desc(sm + OFF_Q + (other * 16 + k) * 256, 128, 8192),
                   smem_desc(oth_buf + k * 256, 128, 4096), id_s, k > 0);
          tc_commit(&bars.oth_free);
          if (!mbar_wait(&bars.own_full[bi], (i >> 1) & 1, abort, err)) break;
          tc_fence_after();
#pragma unroll 1
          for (int k = 0; k < 16; ++k)
            mma_ss(dS, smem_desc(sm + OFF_Q + (h * 16 + k) * 256, 128, 8192),
                   smem_desc(own_buf(bi) + k * 256, 128, 4096), id_s, 1);
          tc_commit(&bars.s_full[bi]);
        }
        if (i >= 1) {
          // O += P(i - 1) X_own(i - 1): A = P from TMEM, B = X MN-major
          const int j = i - 1, bj = j & 1;
          if (!mbar_wait(&bars.p_full[bj], (j >> 1) & 1, abort, err)) break;
          tc_fence_after();
#pragma unroll
          for (int kt = 0; kt < kBT / 16; ++kt)
            mma_ts(tmem + kColO, tmem + kColP + 32 * bj + 8 * kt,
                   smem_desc(own_buf(bj) + kt * 2 * 4096, 4096, 128), id_o, (j > 0 || kt > 0));
          tc_commit(&bars.o_done[bj]);
          tc_commit(&bars.own_free[bj]);
        }
      }
      // every MMA issued must complete before TMEM is released
      tc_commit(&bars.drain);
      volatile int no_abort = 0;
      mbar_wait(&bars.drain, 0, &no_abort, nullptr);
    }
    __syncwarp();
  } else if (warp >= kWarpProd) {
    // ------------------------------------------------------------ producers
    const int pt = tid - 32 * kWarpProd;           // 0..127
    // token of the tile and quarter of a half: the 8 lanes of each quarter-warp
    // take 8 consecutive tokens of one quarter, so every 16-byte shared store
    // of a quarter-warp fills one 128-byte row of banks
    const int pl = pt & 31;
    const int n = (pt >> 5) * 16 + (pl & 7) + ((pl >> 4) << 3);
    const int qh = (pl >> 3) & 1;
    const uint8_t* codes = p.lk + (size_t)b * p.tmax * (kBD / 2);
    const __half* scales = p.lksz + (size_t)b * p.tmax * (kBD / kBG);
    auto load_tile = [&](int i, HalfRegs& ro, HalfRegs& rw) {
      const int tok = t_a + i * kBT + n;
      const bool ok = tok < t_b;
      const int t = ok ? tok : t_a;
      const uint8_t* cr = codes + (size_t)t * (kBD / 2);
      const __half* sr = scales + (size_t)t * (kBD / kBG);
      load_half(ro, cr, sr, 1 - h, qh, ok);
      load_half(rw, cr, sr, h, qh, ok);
    };
    // codes stay in registers two tiles ahead of the dequantisation
    auto produce = [&](int i, HalfRegs& ro, HalfRegs& rw) -> bool {
      const bool ahead = i + 2 < n_tiles;
      const int tok = t_a + (i + 2) * kBT + n;
      const bool ok2 = ahead && tok < t_b;
      const int t2 = ok2 ? tok : t_a;
      const uint8_t* cr = codes + (size_t)t2 * (kBD / 2);
      const __half* sr = scales + (size_t)t2 * (kBD / kBG);
      // other half: free once S(i - 1) has read it
      if (i >= 1 && !mbar_wait(&bars.oth_free, (i - 1) & 1, abort, err)) return false;
      store_half(oth_buf, ro, n, qh);
      fence_proxy_async_smem();
      mbar_arrive(&bars.oth_full);
      if (ahead) load_half(ro, cr, sr, 1 - h, qh, ok2);
      // own half: buffer i & 1 is free once O(i - 2) has read it
      if (i >= 2 && !mbar_wait(&bars.own_free[i & 1], ((i - 2) >> 1) & 1, abort, err)) return false;
      store_half(own_buf(i & 1), rw, n, qh);
      fence_proxy_async_smem();
      mbar_arrive(&bars.own_full[i & 1]);
      if (ahead) load_half(rw, cr, sr, h, qh, ok2);
      return true;
    };
    HalfRegs roA, rwA, roB, rwB;                   // tiles i (even) and i + 1
    if (n_tiles > 0) load_tile(0, roA, rwA);
    if (n_tiles > 1) load_tile(1, roB, rwB);
    // test switch: no tile is produced, so the other roles' bounded waits run out
    const int n_prod = p.test_no_copies ? 0 : n_tiles;
    for (int i = 0; i < n_prod; i += 2) {
      if (!produce(i, roA, rwA)) break;
      if (i + 1 < n_prod && !produce(i + 1, roB, rwB)) break;
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-3)
    const int q = tid;                             // query row = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int bi = i & 1;
      if (!(ok = warp_wait(&bars.s_full[bi], (i >> 1) & 1, abort, err))) break;
      tc_fence_after();
      uint32_t s[kBT];
      {
        uint32_t r0[16], r1[16], r2[16], r3[16];
        tmem_ld16(lane_base + kColS + 64 * bi + 0, r0);
        tmem_ld16(lane_base + kColS + 64 * bi + 16, r1);
        tmem_ld16(lane_base + kColS + 64 * bi + 32, r2);
        tmem_ld16(lane_base + kColS + 64 * bi + 48, r3);
        tmem_wait_ld();
        reg_fence(r0);
        reg_fence(r1);
        reg_fence(r2);
        reg_fence(r3);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          s[k] = r0[k];
          s[16 + k] = r1[k];
          s[32 + k] = r2[k];
          s[48 + k] = r3[k];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.s_free[bi]);
      // tokens past the end of the range score -inf
      const int valid = min(kBT, t_b - (t_a + i * kBT));
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < kBT; ++k)
        if (k < valid) mx = fmaxf(mx, u2f(s[k]));
      const bool raise = mx > m + 8.f;
      float alpha = 1.f;
      if (raise) {
        alpha = ex2_approx(m - mx);                // 0 on the first tile
        m = mx;
        l *= alpha;
      }
      if (i > 0 && __any_sync(0xffffffffu, raise)) {
        // O(i - 1) must have landed before its rows are rescaled
        const int j = i - 1;
        if (!(ok = warp_wait(&bars.o_done[j & 1], (j >> 1) & 1, abort, err))) break;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < kBH; c += 16) {
          uint32_t r[16];
          tmem_ld16(lane_base + kColO + c, r);
          tmem_wait_ld();
          reg_fence(r);
#pragma unroll
          for (int k = 0; k < 16; ++k) r[k] = __float_as_uint(u2f(r[k]) * alpha);
          tmem_st16(lane_base + kColO + c, r);
        }
        tmem_wait_st();
      }
      // P buffer bi was last read by O(i - 2)
      if (i >= 2 && !(ok = warp_wait(&bars.o_done[bi], ((i - 2) >> 1) & 1, abort, err))) break;
      tc_fence_after();
      uint32_t pk[kBT / 2];
      float ls = 0.f;
#pragma unroll
      for (int k = 0; k < kBT; k += 2) {
        const float p0 = k < valid ? ex2_approx(u2f(s[k]) - m) : 0.f;
        const float p1 = k + 1 < valid ? ex2_approx(u2f(s[k + 1]) - m) : 0.f;
        ls += p0 + p1;
        pk[k >> 1] = pack_h2(p0, p1);
      }
      l += ls;
      {
        uint32_t r0[16], r1[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          r0[k] = pk[k];
          r1[k] = pk[16 + k];
        }
        tmem_st16(lane_base + kColP + 32 * bi, r0);
        tmem_st16(lane_base + kColP + 32 * bi + 16, r1);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full[bi]);
    }
    // ---- partials: this half's 256 columns of O, and (m, l) from half 0
    if (ok && n_tiles > 0) {
      const int j = n_tiles - 1;
      ok = warp_wait(&bars.o_done[j & 1], (j >> 1) & 1, abort, err);
    }
    if (ok && n_tiles > 0) {
      tc_fence_after();
      const size_t rows = (size_t)p.L * p.B * p.Hq;
      float* dst = p.part + ((size_t)split * rows + qrow(q)) * (p.vdim + 2);
#pragma unroll 1
      for (int c = 0; c < kBH; c += 16) {
        uint32_t r[16];
        tmem_ld16(lane_base + kColO + c, r);
        tmem_wait_ld();
        reg_fence(r);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int pos = c + k;                   // position within the half
          dst[h * kBH + (pos & ~7) + xperm(pos & 7)] = u2f(r[k]);
        }
      }
      if (h == 0) {
        dst[p.vdim] = m;
        dst[p.vdim + 1] = l;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool block_tc_supported(const Params& p) {
  return p.kind == KVC_BLOCK_SHARED && p.bits == 4 && p.vbits == 0 && p.D == kBD &&
         p.g == kBG && p.d == 128 && p.L * p.Hq == kBQ && !p.seq_lens && p.n_tokens > 0 &&
         p.qdim == kBD && p.vdim == kBD;
}

// token ranges per batch row: about one CTA pair per two SMs over the rows, a
// whole number of tiles each, none empty
void block_tc_plan(const Params& p, int* splits, int* split_len) {
  const int tiles = (p.n_tokens + kBT - 1) / kBT;
  int s = kNumSMs / (2 * p.B);
  if (s > tiles) s = tiles;
  if (s < 1) s = 1;
  const int per = (tiles + s - 1) / s;
  *split_len = per * kBT;
  *splits = (tiles + per - 1) / per;
}

int block_tc_slots(int batch, int n_tokens) {
  const int tiles = (n_tokens + kBT - 1) / kBT;
  int s = kNumSMs / (2 * (batch > 0 ? batch : 1));
  if (s > tiles) s = tiles;
  return s < 1 ? 1 : s;
}

cudaError_t launch_block_tc(const Params& p, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(block_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  block_tc_kernel<<<2 * p.B * p.S, kThreads, kSmem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace kvc
