// Split-T decode on the variable-rate layout (per-token ranks, ragged records),
// one lane per (KV head, query head) pair.
//
// A token's rank is shared by all KV heads, so every lane of a warp takes the
// same rank branch for the same token.  The 8 KV heads x 4 query heads of a
// batch row fill the 32 lanes; each lane keeps its own online softmax (no
// shuffles) and its own latent-space accumulator acc[64] in registers; the
// projected queries q~ = Bk q are formed by the CTA itself (one thread per
// (KV head, rank) row of Bk, all four query heads of the group) into shared
// memory, where each lane reads its own row:
//   s_t = sum_{i < r_k(t)} q~_i (c_i s_g + z_g),
//   acc_i += p_t (c_i s_g + z_g) for i < r_v(t).
// Keeping q~ out of the registers lets 16 warps share an SM (4 per scheduler)
// to hide the per-token dependency chain.
// Every warp streams a contiguous token range in chunks of 8 tokens: the byte
// range of the chunk's K records and of its V records (contiguous in the
// per-row streams) is copied with 16-byte cp.async into a double-buffered
// per-warp area while the previous chunk is processed.  The warps of a CTA
// merge their (m, l, acc) in shared memory and write one partial per row; the
// combine kernel maps acc through Bv.
#include <math.h>

#include "kvc_device.cuh"
#include "tc_util.cuh"

namespace kvc {
namespace {

using namespace tc;

constexpr int kVWarps = 16;
constexpr int kVThreads = 32 * kVWarps;
constexpr int kVChunk = 8;                          // tokens per staged chunk
constexpr int kVHkv = 8, kVG = 4;                   // lanes = KV heads x query heads
constexpr int kVRmax = 64;
constexpr int kVRecMax = kVHkv * (kVRmax / 2 + 8);  // token record bytes at rank 64
constexpr int kVBuf = kVChunk * kVRecMax + 32;      // one staged stream chunk (+ alignment slack)
constexpr int kVWarpBytes = 4 * kVBuf;              // K and V, two buffers each
constexpr int kVStage = kVWarps * kVWarpBytes;
constexpr int kVQRow = kVRmax + 4;                  // floats per q~ row (16-byte loads conflict-free)
constexpr int kVOffQ = kVStage;                     // q~ [32][kVQRow] (softmax scale, log2 e folded)
constexpr int kVOffX = kVOffQ + 32 * kVQRow * 4;    // the group's queries [32][128] fp32
constexpr int kVSmem = kVOffX + 32 * 128 * 4;
constexpr int kVPst = kVRmax + 2;                   // merge slot: acc[64], m, l

static_assert(kVWarps * 32 * kVPst * 4 <= kVStage, "merge area fits in the staging area");
static_assert(kVThreads == kVHkv * kVRmax, "one thread per (KV head, rank) row of Bk");

__host__ __device__ constexpr int head_bytes(int r) { return r / 2 + 4 * ((r + 31) / 32); }

__device__ __forceinline__ void cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
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

// the 8 nibbles of w as floats (exact): each nibble is moved into the low byte
// of the bit pattern 0x4B0000xx = 2^23 + c, and 2^23 is subtracted
__device__ __forceinline__ void nib8(uint32_t w, float (&c)[8]) {
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    c[2 * j] = __int_as_float(prmt(lo, 0x4B000000u, 0x7650u + j)) - 8388608.f;
    c[2 * j + 1] = __int_as_float(prmt(hi, 0x4B000000u, 0x7650u + j)) - 8388608.f;
  }
}

__device__ __forceinline__ float2 h2f2(uint32_t x) {
  return __half22float2(*reinterpret_cast<const __half2*>(&x));
}

// sum_{i < R} q_i (c_i s_g + z_g) over the record at rec (R/2 code bytes, then
// the groups' (scale, zero) pairs); pre = prefix sums of q
// (q = this lane's row of q~ in shared memory)
template <int R>
__device__ __forceinline__ float score_r(const uint8_t* rec, const float* q,
                                         const float (&pre)[5]) {
  if constexpr (R == 4) {
    const uint32_t w = *reinterpret_cast<const uint16_t*>(rec);
    const float s = __half2float(*reinterpret_cast<const __half*>(rec + 2));
    const float z = __half2float(*reinterpret_cast<const __half*>(rec + 4));
    const float4 q0 = *reinterpret_cast<const float4*>(q);
    float c[8];
    nib8(w, c);
    float d = c[0] * q0.x;
    d = fmaf(c[1], q0.y, d);
    d = fmaf(c[2], q0.z, d);
    d = fmaf(c[3], q0.w, d);
    return fmaf(s, d, z * pre[0]);
  } else {
    constexpr int NW = R / 8;
    float dw[NW];                       // one chain per code word (short dependency chains)
#pragma unroll
    for (int wi = 0; wi < NW; ++wi) {
      const float4 qa = *reinterpret_cast<const float4*>(q + 8 * wi);
      const float4 qb = *reinterpret_cast<const float4*>(q + 8 * wi + 4);
      const float qq[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
      float c[8];
      nib8(*reinterpret_cast<const uint32_t*>(rec + 4 * wi), c);
      float a = c[0] * qq[0];
#pragma unroll
      for (int k = 1; k < 8; ++k) a = fmaf(c[k], qq[k], a);
      dw[wi] = a;
    }
    float d[2] = {0.f, 0.f};
#pragma unroll
    for (int wi = 0; wi < NW; ++wi) d[wi / 4] += dw[wi];
    const float2 sz0 = h2f2(*reinterpret_cast<const uint32_t*>(rec + R / 2));
    constexpr int P = R == 8 ? 1 : R == 16 ? 2 : 3;     // prefix of group 0 up to min(R, 32)
    float s = fmaf(sz0.x, d[0], sz0.y * pre[P]);
    if constexpr (R == 64) {
      const float2 sz1 = h2f2(*reinterpret_cast<const uint32_t*>(rec + R / 2 + 4));
      s += fmaf(sz1.x, d[1], sz1.y * pre[4]);
    }
    return s;
  }
}

// acc_i += p (c_i s_g + z_g) for i < R
template <int R>
__device__ __forceinline__ void value_r(const uint8_t* rec, float p, float (&acc)[kVRmax]) {
  if constexpr (R == 4) {
    const uint32_t w = *reinterpret_cast<const uint16_t*>(rec);
    const float ps = p * __half2float(*reinterpret_cast<const __half*>(rec + 2));
    const float pz = p * __half2float(*reinterpret_cast<const __half*>(rec + 4));
    float c[8];
    nib8(w, c);
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] = fmaf(ps, c[k], acc[k] + pz);
  } else {
    constexpr int NW = R / 8;
    float ps[2], pz[2];
    {
      const float2 sz0 = h2f2(*reinterpret_cast<const uint32_t*>(rec + R / 2));
      ps[0] = p * sz0.x;
      pz[0] = p * sz0.y;
      if constexpr (R == 64) {
        const float2 sz1 = h2f2(*reinterpret_cast<const uint32_t*>(rec + R / 2 + 4));
        ps[1] = p * sz1.x;
        pz[1] = p * sz1.y;
      } else {
        ps[1] = pz[1] = 0.f;
      }
    }
#pragma unroll
    for (int wi = 0; wi < NW; ++wi) {
      float c[8];
      nib8(*reinterpret_cast<const uint32_t*>(rec + 4 * wi), c);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int i = 8 * wi + k;
        acc[i] = fmaf(ps[wi / 4], c[k], acc[i] + pz[wi / 4]);
      }
    }
  }
}

__global__ void __launch_bounds__(kVThreads, 1) varrate_warp_kernel(Params p, int split_len) {
  extern __shared__ __align__(128) uint8_t vsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s_idx = blockIdx.x, b = blockIdx.y;
  const int T = p.n_tokens;
  const int cta_a = s_idx * split_len, cta_b = min(T, cta_a + split_len);
  const int per_warp = (split_len + kVWarps - 1) / kVWarps;
  const int t_a = min(cta_b, cta_a + warp * per_warp), t_b = min(cta_b, t_a + per_warp);
  const int h = lane >> 2;

  uint8_t* const area = vsm + warp * kVWarpBytes;
  const uint32_t area_s = smem_u32(area);
  const uint8_t* const kstream = p.lk + (size_t)b * p.stream_bytes;
  const uint8_t* const vstream = p.lv + (size_t)b * p.stream_bytes;
  const int* const offk = p.off_k + (size_t)b * (p.tmax + 1);
  const int* const offv = p.off_v + (size_t)b * (p.tmax + 1);
  const uint8_t* const rk = p.rank_k + (size_t)b * p.tmax;
  const uint8_t* const rv = p.rank_v + (size_t)b * p.tmax;
  const long long sbytes = (long long)p.stream_bytes;

  // ---- q~ = Bk q for the row's 32 query heads (softmax scale and log2 e
  // folded in): thread (kvh, j) dots row j of head kvh's Bk with its 4 queries
  float* const qsm = reinterpret_cast<float*>(vsm + kVOffQ);
  {
    float* const xs = reinterpret_cast<float*>(vsm + kVOffX);
    for (int e = threadIdx.x; e < 32 * 128; e += kVThreads)
      xs[e] = bf2f(p.q[(size_t)b * p.Hq * 128 + e]);
    __syncthreads();
    const int kvh = threadIdx.x / kVRmax, j = threadIdx.x % kVRmax;
    const uint4* br = reinterpret_cast<const uint4*>(p.bk + ((size_t)kvh * kVRmax + j) * 128);
    float a4[kVG] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int c = 0; c < 16; ++c) {
      const uint4 w = __ldg(br + c);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = h2f2(ws[k]);
#pragma unroll
        for (int g = 0; g < kVG; ++g) {
          const float* xg = xs + (kvh * kVG + g) * 128 + 8 * c + 2 * k;
          a4[g] = fmaf(f.x, xg[0], a4[g]);
          a4[g] = fmaf(f.y, xg[1], a4[g]);
        }
      }
    }
#pragma unroll
    for (int g = 0; g < kVG; ++g) qsm[(kvh * kVG + g) * kVQRow + j] = a4[g] * p.scale_log2;
    __syncthreads();
  }
  const float* const q = qsm + lane * kVQRow;       // lane = h * 4 + qi
  float pre[5];
  {
    float run = 0.f;
#pragma unroll 8
    for (int i = 0; i < kVRmax; ++i) {
      if (i == 32) run = 0.f;
      run += q[i];
      if (i == 3) pre[0] = run;
      if (i == 7) pre[1] = run;
      if (i == 15) pre[2] = run;
      if (i == 31) pre[3] = run;
      if (i == 63) pre[4] = run;
    }
  }
  float acc[kVRmax];
#pragma unroll
  for (int i = 0; i < kVRmax; ++i) acc[i] = 0.f;
  float m = -INFINITY, m_thr = -INFINITY, l = 0.f;

  // ---- chunk staging: the byte ranges [off[t0], off[t0 + n]) of both streams,
  // from the 16-byte boundary below, clamped to the stream and the buffer
  struct Meta {
    int ok, ov, rkv;                    // lane j < n: offsets and ranks (rk | rv << 8) of token t0 + j
    int base_k, base_v;                 // stream offsets of the staged areas' first byte
  };
  auto stage = [&](int t0, int buf) -> Meta {
    const int n = min(kVChunk, t_b - t0);
    Meta mt;
    mt.ok = lane <= n ? __ldg(offk + t0 + lane) : 0;
    mt.ov = lane <= n ? __ldg(offv + t0 + lane) : 0;
    mt.rkv = lane < n ? (int)__ldg(rk + t0 + lane) | ((int)__ldg(rv + t0 + lane) << 8) : 0;
    const int k0 = __shfl_sync(0xffffffffu, mt.ok, 0), k1 = __shfl_sync(0xffffffffu, mt.ok, n);
    const int v0 = __shfl_sync(0xffffffffu, mt.ov, 0), v1 = __shfl_sync(0xffffffffu, mt.ov, n);
    mt.base_k = k0 & ~15;
    mt.base_v = v0 & ~15;
    const uint32_t dk = area_s + (2 * buf) * kVBuf, dv = area_s + (2 * buf + 1) * kVBuf;
    const long long ek = min((long long)k1, sbytes), ev = min((long long)v1, sbytes);
    const int nk = (int)min((ek - mt.base_k + 15) / 16, (long long)(kVBuf / 16));
    const int nv = (int)min((ev - mt.base_v + 15) / 16, (long long)(kVBuf / 16));
    for (int c = lane; c < nk; c += 32) cp16(dk + 16 * c, kstream + mt.base_k + 16 * c);
    for (int c = lane; c < nv; c += 32) cp16(dv + 16 * c, vstream + mt.base_v + 16 * c);
    return mt;
  };

  Meta cur{}, nxt{};
  int t0 = t_a, buf = 0;
  if (t0 < t_b) cur = stage(t0, 0);
  cp_commit();
  while (t0 < t_b) {
    const int n = min(kVChunk, t_b - t0);
    const int t1 = t0 + n;
    if (t1 < t_b) nxt = stage(t1, buf ^ 1);
    cp_commit();
    cp_wait<1>();
    __syncwarp();
    const uint8_t* kb = area + (2 * buf) * kVBuf;
    const uint8_t* vb = area + (2 * buf + 1) * kVBuf;
    for (int j = 0; j < n; ++j) {
      const int ok = __shfl_sync(0xffffffffu, cur.ok, j) - cur.base_k;
      const int ov = __shfl_sync(0xffffffffu, cur.ov, j) - cur.base_v;
      const int rkv = __shfl_sync(0xffffffffu, cur.rkv, j);
      const int r_k = rkv & 255, r_v = rkv >> 8;
      // records outside the staged area or off their 16-byte grid (offsets
      // inconsistent with the ranks) are skipped
      if (ok < 0 || (ok & 15) || ok + kVHkv * head_bytes(r_k) > kVBuf || ov < 0 || (ov & 15) ||
          ov + kVHkv * head_bytes(r_v) > kVBuf)
        continue;
      float s;
      const uint8_t* krec = kb + ok + h * head_bytes(r_k);
      switch (r_k) {
        case 4: s = score_r<4>(krec, q, pre); break;
        case 8: s = score_r<8>(krec, q, pre); break;
        case 16: s = score_r<16>(krec, q, pre); break;
        case 32: s = score_r<32>(krec, q, pre); break;
        case 64: s = score_r<64>(krec, q, pre); break;
        default: continue;
      }
      if (s > m_thr) {                  // lazily raised maximum (by more than 2^8)
        const float a = ex2_approx(m - s);
        l *= a;
#pragma unroll
        for (int i = 0; i < kVRmax; ++i) acc[i] *= a;
        m = s;
        m_thr = s + 8.f;
      }
      const float pr = ex2_approx(s - m);
      l += pr;
      const uint8_t* vrec = vb + ov + h * head_bytes(r_v);
      switch (r_v) {
        case 4: value_r<4>(vrec, pr, acc); break;
        case 8: value_r<8>(vrec, pr, acc); break;
        case 16: value_r<16>(vrec, pr, acc); break;
        case 32: value_r<32>(vrec, pr, acc); break;
        case 64: value_r<64>(vrec, pr, acc); break;
        default: break;
      }
    }
    __syncwarp();                       // this buffer is refilled by the next stage
    cur = nxt;
    t0 = t1;
    buf ^= 1;
  }
  cp_wait<0>();
  __syncthreads();

  // ---- merge the warps of this CTA, one partial per row
  float* mg = reinterpret_cast<float*>(vsm);
  {
    float* slot = mg + (warp * 32 + lane) * kVPst;
#pragma unroll
    for (int i = 0; i < kVRmax; ++i) slot[i] = acc[i];
    slot[kVRmax] = m;
    slot[kVRmax + 1] = l;
  }
  __syncthreads();
  const size_t rows = (size_t)p.L * p.B * p.Hq;
  const int pst = p.vdim + 2;
  const int ls = threadIdx.x >> 4, pp = threadIdx.x & 15;   // lane slot, part of its values
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kVWarps; ++w) M = fmaxf(M, mg[(w * 32 + ls) * kVPst + kVRmax]);
  float wt[kVWarps], L = 0.f;
#pragma unroll
  for (int w = 0; w < kVWarps; ++w) {
    const float mw = mg[(w * 32 + ls) * kVPst + kVRmax];
    wt[w] = (M == -INFINITY || mw == -INFINITY) ? 0.f : ex2_approx(mw - M);
    L = fmaf(wt[w], mg[(w * 32 + ls) * kVPst + kVRmax + 1], L);
  }
  const size_t orow = (size_t)b * p.Hq + (ls >> 2) * kVG + (ls & 3);
  float* dst = p.part + ((size_t)s_idx * rows + orow) * pst;
  for (int i = pp; i < kVRmax; i += 16) {
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < kVWarps; ++w) a = fmaf(wt[w], mg[(w * 32 + ls) * kVPst + i], a);
    dst[i] = a;
  }
  if (pp == 0) {
    dst[p.vdim] = M;
    dst[p.vdim + 1] = L;
  }
}

}  // namespace

bool varrate_warp_supported(const Params& p) {
  return p.kind == KVC_VARRATE && p.Hkv == kVHkv && p.G == kVG && p.L == 1 && !p.seq_lens &&
         p.n_tokens > 0 && p.qdim == kVRmax && p.vdim == kVRmax && p.g == 32 &&
         p.stream_bytes % 16 == 0;
}

// CTAs per batch row (one partial each) and tokens per CTA
void varrate_warp_plan(const Params& p, int* splits, int* split_len) {
  int s = kNumSMs / (p.B > 0 ? p.B : 1);
  if (s < 1) s = 1;
  const int max_s = (p.n_tokens + kVWarps * kVChunk - 1) / (kVWarps * kVChunk);
  if (s > max_s) s = max_s;
  if (s < 1) s = 1;
  *split_len = (p.n_tokens + s - 1) / s;
  *splits = (p.n_tokens + *split_len - 1) / *split_len;
}

int varrate_warp_slots(int batch, int n_tokens) {
  int s = kNumSMs / (batch > 0 ? batch : 1);
  if (s < 1) s = 1;
  return s;
}

cudaError_t launch_varrate_warp(const Params& p, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(varrate_warp_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kVSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.S, p.B);
  varrate_warp_kernel<<<grid, kVThreads, kVSmem, s>>>(p, p.split_len);
  return cudaGetLastError();
}

}  // namespace kvc
