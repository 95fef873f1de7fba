// Query projection into the latent space: q~ = Bk q (the score against a
// latent row l is q . (l Bk) = l . (Bk q)), plus q^ = Q q for the rotated
// residual (q . Q^T y = (Q q) . y), and the absorbed block-shared query
// q~_l = W_k^l[:, head slice] q_l.
#include "kvc_device.cuh"

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
// forms the absorbed queries of the whole query group, reading each row of the
// layer's W_k slice once (thread c: latent columns c, c + 256, ...).
__global__ void __launch_bounds__(256) qproj_block_kernel(Params p) {
  __shared__ __align__(16) float qs[8][128];
  const int unit = blockIdx.x;             // (l * B + b) * Hkv + kvh
  const int kvh = unit % p.Hkv;
  const int l = unit / (p.B * p.Hkv);
  const int row0 = (unit / p.Hkv) * p.Hq + kvh * p.G;   // first query row of the group
  const int tid = threadIdx.x, G = p.G;
  for (int e = tid; e < G * 128; e += 256)
    qs[e >> 7][e & 127] = bf2f(p.q[(int64_t)(row0 + (e >> 7)) * 128 + (e & 127)]);
  __syncthreads();
  const __half* w = p.bk + (int64_t)l * p.D * p.Hkv * 128 + kvh * 128;
  for (int c = tid; c < p.D; c += 256) {
    const uint4* wr = reinterpret_cast<const uint4*>(w + (int64_t)c * p.Hkv * 128);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
    for (int k = 0; k < 16; ++k) {
      const uint4 u = __ldg(wr + k);
      const uint32_t ws[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ws[j]));
#pragma unroll
        for (int g = 0; g < 8; ++g)
          if (g < G) {
            acc[g] = fmaf(f.x, qs[g][8 * k + 2 * j], acc[g]);
            acc[g] = fmaf(f.y, qs[g][8 * k + 2 * j + 1], acc[g]);
          }
      }
    }
#pragma unroll
    for (int g = 0; g < 8; ++g)
      if (g < G) p.qt[(int64_t)(row0 + g) * p.qdim + c] = acc[g];
  }
}

}  // namespace

cudaError_t launch_qproj(const Params& p, cudaStream_t s) {
  if ((p.kind == KVC_LOWRANK || p.kind == KVC_VARRATE) && p.d == 128 && p.G <= 8) {
    qproj_group_kernel<<<p.L * p.B * p.Hkv, kThreads, 0, s>>>(p);
    return cudaGetLastError();
  }
  if (p.kind == KVC_BLOCK_SHARED && p.d == 128 && p.G <= 8) {
    qproj_block_kernel<<<p.L * p.B * p.Hkv, 256, 0, s>>>(p);
    return cudaGetLastError();
  }
  const int rows = p.L * p.B * p.Hq;
  qproj_kernel<<<rows, kThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace kvc
