// Query projection into the latent space: q~ = Bk q (the score against a
// latent row l is q . (l Bk) = l . (Bk q)), plus q^ = Q q for the rotated
// residual (q . Q^T y = (Q q) . y), and the absorbed block-shared query
// q~_l = W_k^l[:, head slice] q_l.
#include "kvc_device.cuh"
#include "tc_util.cuh"

namespace kvc {
namespace {

constexpr int kThreads = 128;

__global__ void __launch_bounds__(kThreads) qproj_kernel(Params p) {
  __shared__ float qs[128];
  __shared__ float ys[128];
  const int row = blockIdx.x;              // (l * B + b) * Hq + h
  const int h = row % p.Hq;
  const int l = row / (p.B * p.Hq);
  const int kvh = h / p.G;
  const int tid = threadIdx.x;
  const int d = p.d;
  for (int i = tid; i < d; i += kThreads) qs[i] = bf2f(p.q[(int64_t)row * d + i]);
  __syncthreads();
  float* out = p.qt + (int64_t)row * p.qdim;

  if (p.kind == KVC_BLOCK_SHARED) {
    const __half* w = p.bk + (int64_t)l * p.D * p.Hkv * d + kvh * d;
    for (int c = tid; c < p.D; c += kThreads) {
      const __half* wr = w + (int64_t)c * p.Hkv * d;
      float acc = 0.f;
      for (int i = 0; i < d; ++i) acc = fmaf(h2f(wr[i]), qs[i], acc);
      out[c] = acc;
    }
    return;
  }
  const int r = p.kind == KVC_VARRATE ? 64 : p.rk;
  const __half* bk = p.bk + (int64_t)kvh * r * d;
  for (int j = tid; j < r; j += kThreads) {
    const __half* br = bk + (int64_t)j * d;
    float acc = 0.f;
    for (int i = 0; i < d; ++i) acc = fmaf(h2f(br[i]), qs[i], acc);
    out[j] = acc;
  }
  if (p.kind == KVC_LOWRANK && p.resid) {
    // q^ = H (D q) / sqrt(128)
    for (int i = tid; i < kResidDim; i += kThreads) ys[i] = (float)p.signs_k[i] * qs[i];
    fwht_smem(ys, kResidDim, tid, kThreads);
    const float inv = rsqrtf((float)kResidDim);
    for (int i = tid; i < kResidDim; i += kThreads) out[r + i] = ys[i] * inv;
  }
}

// Low-rank and variable-rate layouts, head dim 128: one block per (layer,
// batch row, KV head) computes the projections of the whole query group.
// Thread o < G r forms q~[o / r][o % r] from 16-byte loads of its Bk row; warp
// h < G forms q^ of query h with the in-register Hadamard transform.
__global__ void __launch_bounds__(kThreads) qproj_group_kernel(Params p) {
  __shared__ __align__(16) float qs[8][128];
  // the decode kernel that follows may start its copies now; it waits for
  // this grid's writes before reading them
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int unit = blockIdx.x;             // (l * B + b) * Hkv + kvh
  const int kvh = unit % p.Hkv;
  const int row0 = (unit / p.Hkv) * p.Hq + kvh * p.G;   // first query row of the group
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G;
  for (int e = tid; e < G * 128; e += kThreads)
    qs[e >> 7][e & 127] = bf2f(p.q[(int64_t)(row0 + (e >> 7)) * 128 + (e & 127)]);
  __syncthreads();
  const int r = p.kind == KVC_VARRATE ? 64 : p.rk;
  const __half* bk = p.bk + (int64_t)kvh * r * 128;
  for (int o = tid; o < G * r; o += kThreads) {
    const int h = o / r, j = o % r;
    const uint4* br = reinterpret_cast<const uint4*>(bk + (int64_t)j * 128);
    const float4* qq = reinterpret_cast<const float4*>(qs[h]);
    float acc = 0.f;
#pragma unroll 4
    for (int c = 0; c < 16; ++c) {
      const uint4 w = __ldg(br + c);
      const float4 q0 = qq[2 * c], q1 = qq[2 * c + 1];
      const float2 b0 = __half22float2(*reinterpret_cast<const __half2*>(&w.x));
      const float2 b1 = __half22float2(*reinterpret_cast<const __half2*>(&w.y));
      const float2 b2 = __half22float2(*reinterpret_cast<const __half2*>(&w.z));
      const float2 b3 = __half22float2(*reinterpret_cast<const __half2*>(&w.w));
      acc = fmaf(b0.x, q0.x, acc);
      acc = fmaf(b0.y, q0.y, acc);
      acc = fmaf(b1.x, q0.z, acc);
      acc = fmaf(b1.y, q0.w, acc);
      acc = fmaf(b2.x, q1.x, acc);
      acc = fmaf(b2.y, q1.y, acc);
      acc = fmaf(b3.x, q1.z, acc);
      acc = fmaf(b3.y, q1.w, acc);
    }
    p.qt[(int64_t)(row0 + h) * p.qdim + j] = acc;
  }
  if (p.kind == KVC_LOWRANK && p.resid) {
    // q^ = H (D q) / sqrt(128)
    for (int h = warp; h < G; h += kThreads / 32) {
      float x[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) x[k] = (float)p.signs_k[4 * lane + k] * qs[h][4 * lane + k];
      fwht128_warp(x, lane);
      const float inv = rsqrtf((float)kResidDim);
      float* out = p.qt + (int64_t)(row0 + h) * p.qdim + r + 4 * lane;
#pragma unroll
      for (int k = 0; k < 4; ++k) out[k] = x[k] * inv;
    }
  }
}

// Block-shared latent, head dim 128: one block per (layer, batch row, KV head)
// forms the absorbed queries of the whole query group from the layer's W_k
// slice (D rows x 128, staged in shared memory with rows padded to 272 bytes
// so that ldmatrix reads are conflict-free).
constexpr int kQbRow = 272;

// The projection runs on warp-level MMAs, with the whole W_k slice in flight
// at once (D <= 768): M = 16 rows of the slice, N = 8 query heads (G of them
// real), K = 16 head dims.  The group's queries are scaled by a power of two,
// 2^-e, so that the largest lies below 2^14, and rounded to f16: exact for
// bf16 inputs (8 significant bits) down to the f16 subnormals, whose spacing
// is 2^-38 of the largest; W_k is fp16, the products are exact and the sums
// fp32, and the results are scaled back by 2^e.  The rows of the first and of
// the second half of the slice are two copy groups, so the MMAs of the first
// half run while the second lands.
constexpr int kQsMaxRows = 768;
constexpr int kQhRow = 136;              // f16 per staged query row (272 bytes)

__global__ void __launch_bounds__(256) qproj_block_mma_kernel(Params p) {
  extern __shared__ __align__(16) uint8_t qsb[];
  __half* const qh = reinterpret_cast<__half*>(qsb);              // [8][kQhRow]
  float* const red = reinterpret_cast<float*>(qsb + 8 * kQhRow * 2);   // [8] warp maxima
  uint8_t* const wsm = qsb + 8 * kQhRow * 2 + 64;                 // [D][kQbRow]
  const int unit = blockIdx.x;             // (l * B + b) * Hkv + kvh
  const int kvh = unit % p.Hkv;
  const int l = unit / (p.B * p.Hkv);
  const int row0 = (unit / p.Hkv) * p.Hq + kvh * p.G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, G = p.G, D = p.D;
  const __half* w = p.bk + (int64_t)l * D * p.Hkv * 128 + kvh * 128;
  const int mid = min(D, ((D / 16 + 1) / 2) * 16);
  auto stage = [&](int r0, int r1) {
    for (int e = tid; e < (r1 - r0) * 16; e += 256) {
      const int r = r0 + (e >> 4), part = e & 15;
      const uint32_t dst = (uint32_t)__cvta_generic_to_shared(wsm + r * kQbRow + part * 16);
      const __half* src = w + (int64_t)r * p.Hkv * 128 + part * 8;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  stage(0, mid);
  stage(mid, D);
  // the group's queries (4 per thread) and their largest magnitude
  float qv[4], mx = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int e = tid + 256 * k, g = e >> 7;
    qv[k] = g < G ? bf2f(p.q[(int64_t)(row0 + g) * 128 + (e & 127)]) : 0.f;
    mx = fmaxf(mx, fabsf(qv[k]));
  }
  mx = warp_max(mx);
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  mx = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) mx = fmaxf(mx, red[k]);
  int ex = 0;
  if (mx > 0.f && mx <= 3.0e38f) {
    frexpf(mx, &ex);                       // mx < 2^ex
    ex = ex > 14 ? ex - 14 : 0;
  }
  const float down = ldexpf(1.f, -ex), up = ldexpf(1.f, ex);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int e = tid + 256 * k;
    qh[(e >> 7) * kQhRow + (e & 127)] = __float2half_rn(qv[k] * down);
  }
  __syncthreads();
  // B fragments of the 8 k-steps: column n = lane / 4, rows 2 (lane % 4) (+1, +8, +9)
  uint32_t bf[8][2];
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const __half* qr = qh + (lane >> 2) * kQhRow + 16 * ks + 2 * (lane & 3);
    bf[ks][0] = *reinterpret_cast<const uint32_t*>(qr);
    bf[ks][1] = *reinterpret_cast<const uint32_t*>(qr + 8);
  }
  const int lrow = (lane & 7) + 8 * ((lane >> 3) & 1), lk = 8 * (lane >> 4);
  const int n0 = 2 * (lane & 3);
  auto tiles = [&](int t0, int t1) {
    for (int mt = t0 + warp; mt < t1; mt += 8) {
      float c[4] = {0.f, 0.f, 0.f, 0.f};
      const uint8_t* ar = wsm + (16 * mt + lrow) * kQbRow + lk * 2;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t a[4];
        tc::ldmatrix_x4(a, ar + 32 * ks);
        tc::mma16816(c, a, bf[ks][0], bf[ks][1]);
      }
      const int ra = 16 * mt + (lane >> 2);
      if (n0 < G) {
        p.qt[(int64_t)(row0 + n0) * p.qdim + ra] = c[0] * up;
        p.qt[(int64_t)(row0 + n0) * p.qdim + ra + 8] = c[2] * up;
      }
      if (n0 + 1 < G) {
        p.qt[(int64_t)(row0 + n0 + 1) * p.qdim + ra] = c[1] * up;
        p.qt[(int64_t)(row0 + n0 + 1) * p.qdim + ra + 8] = c[3] * up;
      }
    }
  };
  asm volatile("cp.async.wait_group 1;" ::: "memory");
  __syncthreads();
  tiles(0, mid / 16);
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  tiles(mid / 16, D / 16);
}

}  // namespace

cudaError_t launch_qproj(const Params& p, cudaStream_t s) {
  if ((p.kind == KVC_LOWRANK || p.kind == KVC_VARRATE) && p.d == 128 && p.G <= 8) {
    qproj_group_kernel<<<p.L * p.B * p.Hkv, kThreads, 0, s>>>(p);
    return cudaGetLastError();
  }
  if (p.kind == KVC_BLOCK_SHARED && p.d == 128 && p.G <= 8 && p.D <= kQsMaxRows &&
      p.D % 16 == 0) {
    const int bytes = 8 * kQhRow * 2 + 64 + p.D * kQbRow;
    cudaError_t e = cudaFuncSetAttribute(qproj_block_mma_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    qproj_block_mma_kernel<<<p.L * p.B * p.Hkv, 256, bytes, s>>>(p);
    return cudaGetLastError();
  }
  const int rows = p.L * p.B * p.Hq;
  qproj_kernel<<<rows, kThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace kvc
