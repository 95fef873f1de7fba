// Split combine and up-projection, once per query head.
//
// Merges the S split partials of a query row with the log-sum-exp rule
// (w_s = 2^(m_s - m*), acc = sum w_s acc_s, l = sum w_s l_s), then maps the
// value-space accumulator to the head dimension:
//   LOWRANK / VARRATE : o = acc[:r] Bv (+ Q^T acc_res) / l
//   BLOCK_SHARED      : o = acc W_v^l[:, head slice] / l
//   DENSE             : o = acc / l
// A row with no tokens (l = 0) produces zeros.
#include <math.h>

#include "kvc_device.cuh"
#include "tc_util.cuh"

namespace kvc {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxS = 1024;

__global__ void __launch_bounds__(kThreads) combine_kernel(Params p) {
  extern __shared__ float sm[];
  float* acc = sm;                       // [vdim]
  float* ws = sm + p.vdim;               // [S] weights
  float* red = ws + p.S;                 // [kThreads] partial sums of the merge
  __shared__ float lsum;
  const int row = blockIdx.x;            // (l * B + b) * Hq + h
  const int h = row % p.Hq;
  const int l = row / (p.B * p.Hq);
  const int kvh = h / p.G;
  const int tid = threadIdx.x;
  const size_t rows = (size_t)p.L * p.B * p.Hq;
  const int pst = p.vdim + 2;
  const float* part = p.part + (size_t)row * pst;
  // launched as a programmatic dependent of the split kernel: wait for its
  // partials here (the launch itself overlaps the split kernel's tail)
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // partial slots of this row: all S splits, or -- on the persistent
  // tensor-core path -- one partial for every CTA whose tile range covers
  // this row's unit (seg_parts partials per CTA)
  int nS = p.S;
  if (p.seg_W > 0) {
    const int u = (row / p.Hq) * p.Hkv + kvh;   // L == 1 on this path
    const long long a = (long long)u * p.seg_tpu, e = (long long)(u + 1) * p.seg_tpu - 1;
    nS = (int)(e / p.seg_W - a / p.seg_W + 1) * p.seg_parts;
  }
  if (tid < 32) {
    float mx = -INFINITY;
    for (int s = tid; s < nS; s += 32) mx = fmaxf(mx, part[(size_t)s * rows * pst + p.vdim]);
    mx = warp_max(mx);
    float lt = 0.f;
    for (int s = tid; s < nS; s += 32) {
      const float* ps = part + (size_t)s * rows * pst;
      const float w = (mx == -INFINITY) ? 0.f : exp2f(ps[p.vdim] - mx);
      ws[s] = w;
      if (w != 0.f) lt += w * ps[p.vdim + 1];
    }
    lt = warp_sum(lt);
    if (tid == 0) lsum = lt;
  }
  __syncthreads();
  // merge: thread (j, k) sums the partials s = k, k + K, ... of value j, so
  // that small value widths still keep every thread busy; then the K partial
  // sums of each j are added
  const int K = p.vdim < kThreads ? kThreads / p.vdim : 1;
  for (int j0 = 0; j0 < p.vdim; j0 += kThreads / K) {
    const int j = j0 + tid % (kThreads / K), k = tid / (kThreads / K);
    float a = 0.f;
    if (j < p.vdim && k < K) {
      for (int s = k; s < nS; s += K)
        if (ws[s] != 0.f) a = fmaf(ws[s], part[(size_t)s * rows * pst + j], a);
    }
    red[tid] = a;
    __syncthreads();
    if (tid < kThreads / K && j0 + tid < p.vdim) {
      float t = 0.f;
      for (int kk = 0; kk < K; ++kk) t += red[kk * (kThreads / K) + tid];
      acc[j0 + tid] = t;
    }
    __syncthreads();
  }
  const float L = lsum;
  const float inv_l = L > 0.f ? 1.f / L : 0.f;
  const int d = p.d;
  float* outf = reinterpret_cast<float*>(p.out);
  __nv_bfloat16* outb = reinterpret_cast<__nv_bfloat16*>(p.out);

  if (p.kind == KVC_LOWRANK && p.resid) {
    // Q^T acc_res = diag(signs_v) H acc_res / sqrt(128)
    fwht_smem(acc + p.rv, kResidDim, tid, kThreads);
  }
  // up-projection: P threads per output dim i, each summing every P-th row of
  // the factor (rows unrolled so that their loads are in flight together),
  // then the P partial sums are added
  const int P = d < kThreads ? kThreads / d : 1;
  for (int i0 = 0; i0 < d; i0 += kThreads / P) {
    const int i = i0 + tid % (kThreads / P), part_id = tid / (kThreads / P);
    float o = 0.f;
    if (i < d && part_id < P) {
      if (p.kind == KVC_LOWRANK || p.kind == KVC_VARRATE) {
        const int r = p.kind == KVC_VARRATE ? 64 : p.rv;
        const __half* bv = p.bv + (int64_t)kvh * r * d + i;
#pragma unroll 8
        for (int j = part_id; j < r; j += P) o = fmaf(acc[j], h2f(bv[(int64_t)j * d]), o);
        if (p.kind == KVC_LOWRANK && p.resid && part_id == 0)
          o = fmaf((float)p.signs_v[i] * rsqrtf((float)kResidDim), acc[p.rv + i], o);
      } else if (p.kind == KVC_BLOCK_SHARED) {
        const __half* w = p.bv + (int64_t)l * p.D * p.Hkv * d + kvh * d + i;
#pragma unroll 8
        for (int c = part_id; c < p.D; c += P) o = fmaf(acc[c], h2f(w[(int64_t)c * p.Hkv * d]), o);
      } else if (part_id == 0) {
        o = acc[i];
      }
    }
    red[tid] = o;
    __syncthreads();
    if (tid < kThreads / P && i0 + tid < d) {
      float t = 0.f;
      for (int k = 0; k < P; ++k) t += red[k * (kThreads / P) + tid];
      t *= inv_l;
      if (p.out_bf16) outb[(int64_t)row * d + i0 + tid] = __float2bfloat16_rn(t);
      else outf[(int64_t)row * d + i0 + tid] = t;
    }
    __syncthreads();
  }
}


// Low-rank layouts, head dim 128, value rank <= 64 (plus the 128 rotated
// residual values, if any) and few partials per row: every global load of the
// row (the partials' maxima and sums, their accumulators, the Bv column slice,
// the signs) is issued before any arithmetic, so the row costs one round trip
// to memory instead of one per step.  The residual accumulator is mapped back
// with the in-register Hadamard transform of one warp.
constexpr int kFastS = 160;

// NV partial values per thread, NM maxima per lane of warp 0: a small instance
// for few partials (low register use, several blocks per SM) and a large one
template <int NV, int NM>
__global__ void __launch_bounds__(kThreads) combine_lowrank_kernel(Params p) {
  constexpr int kFastVals = NV, kFastM = NM;
  __shared__ float ws[kFastS];
  __shared__ float red[kThreads];
  __shared__ float acc[256];
  __shared__ float lsum;
  const int row = blockIdx.x;            // b * Hq + h
  const int h = row % p.Hq;
  const int kvh = h / p.G;
  const int tid = threadIdx.x, lane = tid & 31;
  const size_t rows = (size_t)p.B * p.Hq;
  const int pst = p.vdim + 2, rv = p.rv, vdim = p.vdim;
  const float* part = p.part + (size_t)row * pst;
  // the Bv column slice and the signs are not written by the split kernel:
  // loaded before waiting for it (this block may start during its last CTAs)
  const int oi = tid & 127, half = tid >> 7;          // output dim, half of the ranks
  const __half* bv = p.bv + (size_t)kvh * rv * 128 + oi;
  float bw[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int r = half + 2 * i;
    bw[i] = r < rv ? h2f(bv[(size_t)r * 128]) : 0.f;
  }
  const float sgn = p.resid ? (float)p.signs_v[oi] * rsqrtf((float)kResidDim) : 0.f;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  int nS = p.S;
  if (p.seg_W > 0) {
    const int u = (row / p.Hq) * p.Hkv + kvh;
    const long long a = (long long)u * p.seg_tpu, e = (long long)(u + 1) * p.seg_tpu - 1;
    nS = (int)(e / p.seg_W - a / p.seg_W + 1) * p.seg_parts;
  }
  // ---- issue every load
  float mm[kFastM], ll[kFastM];
#pragma unroll
  for (int k = 0; k < kFastM; ++k) {
    mm[k] = -INFINITY;
    ll[k] = 0.f;
    if (tid < 32 && lane + 32 * k < nS) {
      mm[k] = part[(size_t)(lane + 32 * k) * rows * pst + vdim];
      ll[k] = part[(size_t)(lane + 32 * k) * rows * pst + vdim + 1];
    }
  }
  const int K = kThreads / vdim;         // partial groups per value index
  const int j = tid % vdim, k = tid / vdim;
  float pv[kFastVals];
#pragma unroll
  for (int i = 0; i < kFastVals; ++i) {
    const int sidx = k + i * K;
    pv[i] = (k < K && sidx < nS) ? part[(size_t)sidx * rows * pst + j] : 0.f;
  }
  // ---- weights
  if (tid < 32) {
    float mx = -INFINITY;
#pragma unroll
    for (int k = 0; k < kFastM; ++k) mx = fmaxf(mx, mm[k]);
    mx = warp_max(mx);
    float lt = 0.f;
#pragma unroll
    for (int k = 0; k < kFastM; ++k) {
      const float w = (mx == -INFINITY || mm[k] == -INFINITY) ? 0.f : exp2f(mm[k] - mx);
      if (lane + 32 * k < nS) ws[lane + 32 * k] = w;
      if (w != 0.f) lt = fmaf(w, ll[k], lt);
    }
    lt = warp_sum(lt);
    if (lane == 0) lsum = lt;
  }
  __syncthreads();
  // ---- merge
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < kFastVals; ++i) {
    const int sidx = k + i * K;
    if (k < K && sidx < nS) {
      const float w = ws[sidx];
      if (w != 0.f) a = fmaf(w, pv[i], a);
    }
  }
  red[tid] = a;
  __syncthreads();
  if (tid < vdim) {
    float t = 0.f;
    for (int kk = 0; kk < K; ++kk) t += red[kk * vdim + tid];
    acc[tid] = t;
  }
  __syncthreads();
  if (p.resid) {
    // Q^T acc_res = diag(signs_v) H acc_res / sqrt(128); H here, the rest below
    if (tid < 32) {
      float x[4];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) x[kk] = acc[rv + 4 * lane + kk];
      fwht128_warp(x, lane);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) acc[rv + 4 * lane + kk] = x[kk];
    }
    __syncthreads();
  }
  // ---- up-projection o = acc Bv / l (two halves of the ranks per output)
  float o = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int r = half + 2 * i;
    if (r < rv) o = fmaf(acc[r], bw[i], o);
  }
  if (p.resid && half) o = fmaf(sgn, acc[rv + oi], o);
  red[tid] = o;
  __syncthreads();
  if (tid < 128) {
    const float L = lsum;
    const float t = (red[tid] + red[tid + 128]) * (L > 0.f ? 1.f / L : 0.f);
    if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)row * 128 + tid] = __float2bfloat16_rn(t);
    else reinterpret_cast<float*>(p.out)[(size_t)row * 128 + tid] = t;
  }
}

}  // namespace

// Block-shared latent: one block per (layer, batch row, KV head) merges the
// G query heads' partials together and applies the layer's W_v slice to all
// of them, so each W_v element is read once per block rather than once per
// query head.  The slice (D rows x head dim) streams through shared memory in
// chunks of 64 rows (16-byte cp.async, double-buffered); thread (i, g0) forms
// output dim i of heads g0, g0 + 2, ... .
constexpr int kBGroup = 8;               // query heads per KV head handled (G <= 8)
constexpr int kBRows = 64;               // W_v rows per staged chunk

__global__ void __launch_bounds__(kThreads) combine_block_kernel(Params p) {
  extern __shared__ __align__(16) float bsm[];
  const int D = p.D, d = p.d, G = p.G;
  float* acc = bsm;                      // [G][D]
  float* ws = acc + G * D;               // [G][S]
  __half* wv = reinterpret_cast<__half*>(ws + ((G * p.S + 3) & ~3));   // [2][kBRows][d], 16-B aligned
  __shared__ float linv[kBGroup];
  const int blk = blockIdx.x;            // (l * B + b) * Hkv + kvh
  const int kvh = blk % p.Hkv, lb = blk / p.Hkv;   // lb = l * B + b
  const int l = lb / p.B;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t rows = (size_t)p.L * p.B * p.Hq;
  const int pst = p.vdim + 2;
  const int nS = p.S;
  const __half* w = p.bv + (int64_t)l * D * p.Hkv * d + kvh * d;
  const int n_chunks = (D + kBRows - 1) / kBRows;
  const int cpr = d / 8;                 // 16-byte chunks per W_v row
  auto stage = [&](int c, int buf) {
    for (int e = tid; e < kBRows * cpr; e += kThreads) {
      const int r = e / cpr, part = e % cpr, row = c * kBRows + r;
      if (row < D) {
        const uint32_t dst = (uint32_t)__cvta_generic_to_shared(wv + ((size_t)buf * kBRows + r) * d + part * 8);
        const __half* src = w + (int64_t)row * p.Hkv * d + part * 8;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  asm volatile("griddepcontrol.wait;" ::: "memory");
  stage(0, 0);
  // split weights and softmax sums of the G rows (warp g: row g)
  for (int g = warp; g < G; g += kThreads / 32) {
    const float* part = p.part + ((size_t)lb * p.Hq + kvh * G + g) * pst;
    float mx = -INFINITY;
    for (int s = lane; s < nS; s += 32) mx = fmaxf(mx, part[(size_t)s * rows * pst + D]);
    mx = warp_max(mx);
    float lt = 0.f;
    for (int s = lane; s < nS; s += 32) {
      const float* ps = part + (size_t)s * rows * pst;
      const float wt = (mx == -INFINITY) ? 0.f : exp2f(ps[D] - mx);
      ws[g * nS + s] = wt;
      if (wt != 0.f) lt += wt * ps[D + 1];
    }
    lt = warp_sum(lt);
    if (lane == 0) linv[g] = lt > 0.f ? 1.f / lt : 0.f;
  }
  __syncthreads();
  // merged accumulators of the G rows
  for (int e = tid; e < G * D; e += kThreads) {
    const int g = e / D, c = e % D;
    const float* part = p.part + ((size_t)lb * p.Hq + kvh * G + g) * pst + c;
    float a = 0.f;
#pragma unroll 8
    for (int s = 0; s < nS; ++s) a = fmaf(ws[g * nS + s], part[(size_t)s * rows * pst], a);
    acc[e] = a;
  }
  // up-projection o_g = acc_g W_v^l[:, kvh slice] / l_g
  const int gstep = kThreads / d;        // heads handled in parallel (2 for d = 128)
  const int i = tid % d, g0 = tid / d;
  float o[kBGroup];
#pragma unroll
  for (int g = 0; g < kBGroup; ++g) o[g] = 0.f;
  for (int c = 0; c < n_chunks; ++c) {
    if (c + 1 < n_chunks) {
      stage(c + 1, (c + 1) & 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const __half* wc = wv + (size_t)(c & 1) * kBRows * d;
    const int nr = min(kBRows, D - c * kBRows);
    if (g0 < gstep) {
      for (int r = 0; r < nr; ++r) {
        const float wvv = __half2float(wc[r * d + i]);
#pragma unroll
        for (int gg = 0; gg < kBGroup; ++gg) {
          const int g = g0 + gstep * gg;
          if (g < G) o[gg] = fmaf(acc[g * D + c * kBRows + r], wvv, o[gg]);
        }
      }
    }
    __syncthreads();                     // buffer c & 1 is restaged for chunk c + 2
  }
  if (g0 < gstep) {
#pragma unroll
    for (int gg = 0; gg < kBGroup; ++gg) {
      const int g = g0 + gstep * gg;
      if (g < G) {
        const float t = o[gg] * linv[g];
        const int64_t orow = (int64_t)lb * p.Hq + kvh * G + g;
        if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[orow * d + i] = __float2bfloat16_rn(t);
        else reinterpret_cast<float*>(p.out)[orow * d + i] = t;
      }
    }
  }
}

// Block-shared latent, head dim 128, all of a block's partials in shared
// memory at once (the usual case: few splits per row, an even group): one
// block per (layer, batch row, KV head).  The first rows of the layer's W_v
// slice are copied
// before the block waits for the split kernel (they do not depend on it); then
// the G query heads' partials (every split, accumulators and (m, l); the G
// rows of a split are one span) arrive by 1-D bulk copies counted on an
// mbarrier (bounded wait), are weighted and merged from shared memory,
// and the rest of the W_v slice lands where the partials were.  The
// up-projection runs on warp-level MMAs: M = 16 output dims (warp w: dims
// 16 w ..), N = 8 heads, K = 16 latent rows; the fp32 accumulators enter as
// the sum of two f16 parts (hi = f16(x), lo = f16(x - hi), after scaling the
// head by a power of two that puts its largest value below 2^14), so the two
// MMAs per k-step carry ~22 significant bits of every accumulator; W_v is
// fp16, products are exact and the sums fp32.
constexpr int kCbThreads = 256;
constexpr int kCbRow = 272;             // bytes per staged W_v row (conflict-free ldmatrix)

struct BlockCombinePlan {
  int rows_a;                           // W_v rows staged before the wait
  size_t off_acc, off_wts, off_wa, bytes;
};

__host__ __device__ inline BlockCombinePlan block_combine_plan(int G, int S, int D, int vdim) {
  BlockCombinePlan pl;
  const size_t pbytes = (size_t)G * S * (vdim + 2) * sizeof(float);
  pl.off_acc = (pbytes + 15) & ~(size_t)15;
  pl.off_wts = pl.off_acc + (size_t)G * D * sizeof(float);
  pl.off_wa = (pl.off_wts + ((size_t)G * S + 24) * sizeof(float) + 15) & ~(size_t)15;
  const size_t budget = 227 * 1024 - 256;   // the kernel's static barriers and flag
  long long ra = pl.off_wa < budget ? (long long)((budget - pl.off_wa) / kCbRow) : 0;
  ra &= ~15ll;
  if (ra > D) ra = D;
  pl.rows_a = (int)ra;
  pl.bytes = pl.off_wa + (size_t)pl.rows_a * kCbRow;
  return pl;
}

__global__ void __launch_bounds__(kCbThreads) combine_block_staged_kernel(Params p) {
  extern __shared__ __align__(16) uint8_t cbs[];
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ int abort_flag;
  const int D = p.D, G = p.G, nS = p.S, pst = p.vdim + 2;
  const BlockCombinePlan pl = block_combine_plan(G, nS, D, p.vdim);
  float* const P = reinterpret_cast<float*>(cbs);                  // [nS][G][pst]
  float* const acc = reinterpret_cast<float*>(cbs + pl.off_acc);  // [G][D]
  float* const wts = reinterpret_cast<float*>(cbs + pl.off_wts);  // [G][nS], then 1/l [G]
  float* const linv = wts + G * nS;
  const int blk = blockIdx.x;            // (l * B + b) * Hkv + kvh
  const int kvh = blk % p.Hkv, lb = blk / p.Hkv;
  const int l = lb / p.B;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t rows = (size_t)p.L * p.B * p.Hq;
  const __half* w = p.bv + (int64_t)l * D * p.Hkv * 128 + kvh * 128;
  const int span = G * pst;              // floats: the G heads' partials of one split
  if (tid == 0) {
    tc::mbar_init(&bars[0], 1);
    tc::mbar_init(&bars[1], 1);
    tc::fence_mbar_init();
    abort_flag = 0;
    // the first W_v rows and every split's span on barrier 0, the other rows on 1
    tc::mbar_arrive_expect_tx(&bars[0], (uint32_t)(pl.rows_a * 256 + nS * span * 4));
    tc::mbar_arrive_expect_tx(&bars[1], (uint32_t)((D - pl.rows_a) * 256));
  }
  __syncthreads();
  // 1-D bulk copies: W_v rows (256 bytes) into rows of kCbRow bytes
  auto copy_w = [&](int r0, int r1, uint8_t* dst, uint64_t* bar) {
    for (int r = r0 + tid; r < r1; r += kCbThreads)
      tc::bulk_g2s(dst + (r - r0) * kCbRow, w + (int64_t)r * p.Hkv * 128, 256, bar);
  };
  copy_w(0, pl.rows_a, cbs + pl.off_wa, &bars[0]);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  {
    // the G heads' partials of split sp are G consecutive rows of (vdim + 2)
    // floats; with G even the span starts on a 16-byte boundary and is a whole
    // number of 16-byte pieces (the launch requires G even)
    const float* const src0 = p.part + ((size_t)lb * p.Hq + kvh * G) * pst;
    for (int sp = tid; sp < nS; sp += kCbThreads)
      tc::bulk_g2s(P + (size_t)sp * span, src0 + (size_t)sp * rows * pst, (uint32_t)span * 4,
                   &bars[0]);
  }
  if (!tc::mbar_wait(&bars[0], 0, &abort_flag, p.err)) return;
  __syncthreads();
  // split weights and softmax sums (warp g: head g)
  for (int g = warp; g < G; g += kCbThreads / 32) {
    const float* pg = P + (size_t)g * pst;
    const size_t sstr = (size_t)G * pst;  // between the splits of one head
    float mx = -INFINITY;
    for (int sp = lane; sp < nS; sp += 32) mx = fmaxf(mx, pg[sp * sstr + D]);
    mx = warp_max(mx);
    float lt = 0.f;
    for (int sp = lane; sp < nS; sp += 32) {
      const float m = pg[sp * sstr + D];
      const float wt = (mx == -INFINITY || m == -INFINITY) ? 0.f : exp2f(m - mx);
      wts[g * nS + sp] = wt;
      lt = fmaf(wt, pg[sp * sstr + D + 1], lt);
    }
    lt = warp_sum(lt);
    if (lane == 0) linv[g] = lt > 0.f ? 1.f / lt : 0.f;
  }
  __syncthreads();
  // merged accumulators: thread t forms dims 2 t, 2 t + 1 (+ 512 k) of every
  // head, one independent chain per (head, dim)
  for (int c2 = 2 * tid; c2 < D; c2 += 2 * kCbThreads) {
    float2 a[kBGroup];
#pragma unroll
    for (int g = 0; g < kBGroup; ++g) a[g] = make_float2(0.f, 0.f);
#pragma unroll 2
    for (int sp = 0; sp < nS; ++sp) {
      const float* ps = P + (size_t)sp * G * pst + c2;
#pragma unroll
      for (int g = 0; g < kBGroup; ++g) {
        if (g < G) {
          const float wgt = wts[g * nS + sp];
          const float2 v = *reinterpret_cast<const float2*>(ps + (size_t)g * pst);
          a[g].x = fmaf(wgt, v.x, a[g].x);
          a[g].y = fmaf(wgt, v.y, a[g].y);
        }
      }
    }
#pragma unroll
    for (int g = 0; g < kBGroup; ++g)
      if (g < G) *reinterpret_cast<float2*>(acc + g * D + c2) = a[g];
  }
  __syncthreads();
  // per-head scale of the merged accumulators (warp g: head g)
  float* const down = linv + 8;         // 2^-e_g
  float* const up = linv + 16;          // 2^e_g / l_g
  for (int g = warp; g < 8; g += kCbThreads / 32) {
    float mx = 0.f;
    if (g < G)
      for (int c = lane; c < D; c += 32) mx = fmaxf(mx, fabsf(acc[g * D + c]));
    mx = warp_max(mx);
    int ex = 0;
    if (mx > 0.f && mx <= 3.0e38f) {
      frexpf(mx, &ex);
      ex = ex > 14 ? ex - 14 : (ex < -100 ? -100 : ex - 14);
    }
    if (lane == 0) {
      down[g] = ldexpf(1.f, -ex);
      up[g] = g < G ? ldexpf(1.f, ex) * linv[g] : 0.f;
    }
  }
  __syncthreads();                      // the partials are dead: W_v's other rows land there
  uint8_t* const wb = cbs;
  copy_w(pl.rows_a, D, wb, &bars[1]);
  // up-projection: warp w forms output dims 16 w .. 16 w + 15 of the 8 heads
  const int n = lane >> 2, kq = 2 * (lane & 3);
  const bool live = n < G;
  const float* const an = acc + (live ? n : 0) * D + kq;
  const float sn = down[n];
  const int lj = lane >> 3, lr = lane & 7;
  const int i_off = 16 * warp + 8 * (lj & 1);
  float c4[4] = {0.f, 0.f, 0.f, 0.f};
  auto ksteps = [&](const uint8_t* wr, int k0, int k1, int r_base) {
    for (int ks = k0; ks < k1; ++ks) {
      const int row = 16 * ks + lr + 8 * (lj >> 1);
      uint32_t a[4];
      tc::ldmatrix_x4_trans(a, wr + (row - r_base) * kCbRow + 2 * i_off);
      float x[4] = {0.f, 0.f, 0.f, 0.f};
      if (live) {
        const float2 v0 = *reinterpret_cast<const float2*>(an + 16 * ks);
        const float2 v8 = *reinterpret_cast<const float2*>(an + 16 * ks + 8);
        x[0] = v0.x * sn; x[1] = v0.y * sn; x[2] = v8.x * sn; x[3] = v8.y * sn;
      }
      const __half2 h0 = __floats2half2_rn(x[0], x[1]), h8 = __floats2half2_rn(x[2], x[3]);
      const float2 f0 = __half22float2(h0), f8 = __half22float2(h8);
      const __half2 l0 = __floats2half2_rn(x[0] - f0.x, x[1] - f0.y);
      const __half2 l8 = __floats2half2_rn(x[2] - f8.x, x[3] - f8.y);
      tc::mma16816(c4, a, *reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h8));
      tc::mma16816(c4, a, *reinterpret_cast<const uint32_t*>(&l0), *reinterpret_cast<const uint32_t*>(&l8));
    }
  };
  ksteps(cbs + pl.off_wa, 0, pl.rows_a / 16, 0);
  if (!tc::mbar_wait(&bars[1], 0, &abort_flag, p.err)) return;
  if (pl.rows_a < D) ksteps(wb, pl.rows_a / 16, D / 16, pl.rows_a);
  // C fragment: dims 16 w + lane / 4 (+ 8), heads 2 (lane % 4) (+ 1)
  const int i0 = 16 * warp + (lane >> 2);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int g = kq + (e & 1), i = i0 + 8 * (e >> 1);
    if (g < G) {
      const int64_t orow = (int64_t)lb * p.Hq + kvh * G + g;
      const float t = c4[e] * up[g];
      if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[orow * 128 + i] = __float2bfloat16_rn(t);
      else reinterpret_cast<float*>(p.out)[orow * 128 + i] = t;
    }
  }
}

cudaError_t launch_combine(const Params& p, cudaStream_t s) {
  if (p.S > kMaxS) return cudaErrorInvalidValue;
  const int rows = p.L * p.B * p.Hq;
  const bool lowrank = p.kind == KVC_LOWRANK && p.vdim == p.rv + (p.resid ? kResidDim : 0) &&
                       p.rv >= 16 && p.rv <= 64;
  const bool varrate = p.kind == KVC_VARRATE && p.vdim == 64 && p.rv == 64 && !p.resid;
  const int per_thread = (lowrank || varrate) ? (p.S + kThreads / p.vdim - 1) / (kThreads / p.vdim) : 0;
  const bool fast = (lowrank || varrate) && p.d == 128 && p.L == 1 && p.S <= kFastS &&
                    per_thread <= 40;
  const bool small = fast && p.S <= 64 && per_thread <= 16;
  const size_t bytes = ((size_t)p.vdim + p.S + kThreads) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(combine_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = fast ? 0 : bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (p.kind == KVC_BLOCK_SHARED && p.G <= kBGroup && p.seg_W == 0 && p.d == 128 &&
      p.vdim == p.D && p.D % 8 == 0) {
    const BlockCombinePlan pl = block_combine_plan(p.G, p.S, p.D, p.vdim);
    if (p.G % 2 == 0 && pl.rows_a >= 16 && (size_t)(p.D - pl.rows_a) * kCbRow <= pl.off_acc) {
      e = cudaFuncSetAttribute(combine_block_staged_kernel,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.bytes);
      if (e != cudaSuccess) return e;
      cfg.gridDim = dim3(p.L * p.B * p.Hkv);
      cfg.blockDim = dim3(kCbThreads);
      cfg.dynamicSmemBytes = pl.bytes;
      return cudaLaunchKernelEx(&cfg, combine_block_staged_kernel, p);
    }
  }
  if (p.kind == KVC_BLOCK_SHARED && p.G <= kBGroup && p.seg_W == 0 && p.d % 8 == 0 &&
      p.d <= kThreads) {
    const size_t bb = ((size_t)p.G * p.D + (size_t)p.G * p.S + 4) * sizeof(float) +
                      (size_t)2 * kBRows * p.d * sizeof(__half);
    e = cudaFuncSetAttribute(combine_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)bb);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(p.L * p.B * p.Hkv);
    cfg.dynamicSmemBytes = bb;
    return cudaLaunchKernelEx(&cfg, combine_block_kernel, p);
  }
  if (small) return cudaLaunchKernelEx(&cfg, combine_lowrank_kernel<16, 2>, p);
  if (fast) return cudaLaunchKernelEx(&cfg, combine_lowrank_kernel<40, 5>, p);
  return cudaLaunchKernelEx(&cfg, combine_kernel, p);
}

}  // namespace kvc
