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

}  // namespace

cudaError_t launch_qproj(const Params& p, cudaStream_t s) {
  const int rows = p.L * p.B * p.Hq;
  qproj_kernel<<<rows, kThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace kvc
