// Split-T decode, generic CUDA-core version covering every layout kind.
//
// One CTA owns one unit (a (layer, batch row, KV head) for per-head layouts,
// or (batch row, 32 absorbed queries) for the block-shared latent) and one
// contiguous token range of it.  For each tile of tokens it dequantizes the
// compressed rows into fp32 shared memory, scores every query of the unit
// against the tile, updates an online softmax and accumulates p . V in the
// value space the combine kernel up-projects from.  Per split it writes the
// partial (acc, m, l) with m in log2 units.
//
// Score spaces:  LOWRANK without RoPE and VARRATE score in latent space
// (q~ . l_hat (+ q^ . y_hat)); LOWRANK with RoPE reconstructs K = l_hat Bk
// (+ Q^T y_hat), rotates it and scores with q; BLOCK_SHARED scores the
// absorbed queries against the latent; DENSE reads bf16 K/V.
#include <math.h>

#include "kvc_device.cuh"

namespace kvc {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxAcc = 64;     // accumulators per thread

struct Geo {
  int nq, kd, vd, tt;           // queries, score width, value width, tile
  bool alias_v;                 // value tile == key tile (block-shared latent)
  bool recon;                   // RoPE reconstruction path
  int lat_k;                    // latent K width staged before reconstruction
};

__host__ __device__ inline Geo geometry(const Params& p) {
  Geo g;
  g.tt = split_tile(p.kind, p.rope);
  g.alias_v = false;
  g.recon = false;
  g.lat_k = 0;
  const int res = p.resid ? kResidDim : 0;
  switch (p.kind) {
    case KVC_LOWRANK:
      g.nq = p.G;
      g.recon = p.rope != 0;
      g.kd = g.recon ? p.d : p.rk + res;
      g.lat_k = g.recon ? p.rk : 0;
      g.vd = p.rv + res;
      break;
    case KVC_VARRATE:
      g.nq = p.G;
      g.kd = 64;
      g.vd = 64;
      break;
    case KVC_BLOCK_SHARED:
      g.nq = kBlockQueries;
      g.kd = p.D;
      g.vd = p.D;
      g.alias_v = p.vbits == 0;     // one latent feeds keys and values
      break;
    default:
      g.nq = p.G;
      g.kd = p.d;
      g.vd = p.d;
      break;
  }
  return g;
}

// Shared-memory carve-up (floats).
struct Smem {
  int qs, kt, vt, lt, bk, rt, sc, al, total;
};

__host__ __device__ inline Smem carve(const Params& p, const Geo& g) {
  Smem s;
  int o = 0;
  s.qs = o; o += g.nq * g.kd;
  s.kt = o; o += g.tt * (g.kd + 1);
  s.vt = o; if (!g.alias_v) o += g.tt * (g.vd + 1);
  s.lt = o; o += g.recon ? g.tt * (g.lat_k + 1) : 0;
  s.bk = o; o += g.recon ? g.lat_k * p.d : 0;
  s.rt = o; o += (g.recon && p.resid) ? g.tt * kResidDim : 0;
  s.sc = o; o += g.nq * g.tt;
  s.al = o; o += g.nq;
  s.total = o;
  return s;
}

__global__ void __launch_bounds__(kThreads) split_generic_kernel(Params p) {
  extern __shared__ float sm[];
  const Geo g = geometry(p);
  const Smem S = carve(p, g);
  float* qs = sm + S.qs;
  float* kt = sm + S.kt;
  float* vt = g.alias_v ? kt : sm + S.vt;
  float* lt = sm + S.lt;
  float* bks = sm + S.bk;
  float* rt = sm + S.rt;
  float* sc = sm + S.sc;
  float* al = sm + S.al;
  const int kstr = g.kd + 1, vstr = g.alias_v ? kstr : g.vd + 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = kThreads / 32;

  // ---- unit -> (layer, batch row, KV head / query chunk)
  int l = 0, b, kvh = 0, chunk = 0;
  const int unit = blockIdx.y;
  if (p.kind == KVC_BLOCK_SHARED) {
    const int chunks = p.L * p.Hq / kBlockQueries;
    b = unit / chunks;
    chunk = unit % chunks;
  } else {
    kvh = unit % p.Hkv;
    b = (unit / p.Hkv) % p.B;
    l = unit / (p.Hkv * p.B);
  }
  // global query row of local query i
  auto qrow = [&](int i) -> int {
    if (p.kind == KVC_BLOCK_SHARED) {
      const int qi = chunk * kBlockQueries + i;   // flattened (layer, head)
      const int ll = qi / p.Hq, hh = qi % p.Hq;
      return (ll * p.B + b) * p.Hq + hh;
    }
    return (l * p.B + b) * p.Hq + kvh * p.G + i;
  };

  const int len = row_len(p, b);
  const int t_begin = blockIdx.x * p.split_len;
  const int t_end = min(t_begin + p.split_len, len);

  // ---- queries
  for (int e = tid; e < g.nq * g.kd; e += kThreads) {
    const int i = e / g.kd, k = e % g.kd;
    const int r = qrow(i);
    qs[e] = p.qdim ? p.qt[(int64_t)r * p.qdim + k] : bf2f(p.q[(int64_t)r * p.d + k]);
  }
  if (g.recon) {
    const __half* bk = p.bk + (int64_t)kvh * p.rk * p.d;
    for (int e = tid; e < p.rk * p.d; e += kThreads) bks[e] = h2f(bk[e]);
  }

  float acc[kMaxAcc];
  const int nacc = (g.nq * g.vd + kThreads - 1) / kThreads;
#pragma unroll
  for (int k = 0; k < kMaxAcc; ++k) acc[k] = 0.f;
  // query i's running (m, l) is kept by warp i % nwarps, replicated across its lanes
  float m_q[4], l_q[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) m_q[k] = -INFINITY, l_q[k] = 0.f;
  __syncthreads();

  for (int t0 = t_begin; t0 < t_end; t0 += g.tt) {
    const int nt = min(g.tt, t_end - t0);
    // ---------------- load + dequantize the tile
    if (p.kind == KVC_LOWRANK) {
      const int rk = p.rk;
      float* ldst = g.recon ? lt : kt;
      const int lstr = g.recon ? g.lat_k + 1 : kstr;
      for (int e = tid; e < g.tt * rk; e += kThreads) {
        const int t = e / rk, r = e % rk;
        float v = 0.f;
        if (t < nt) {
          const int64_t row = lowrank_row(p, b, kvh, t0 + t);
          if (p.bits == 16) {
            v = h2f(reinterpret_cast<const __half*>(p.lk)[row * rk + r]);
          } else {
            const __half* sz = p.lksz + row * p.ngk * 2 + (r / p.g) * 2;
            v = fmaf((float)int4_at(p.lk + row * p.lk_row, r), h2f(sz[0]), h2f(sz[1]));
          }
        }
        ldst[t * lstr + r] = v;
      }
      const int rv = p.rv;
      for (int e = tid; e < g.tt * rv; e += kThreads) {
        const int t = e / rv, r = e % rv;
        float v = 0.f;
        if (t < nt) {
          const int64_t row = lowrank_row(p, b, kvh, t0 + t);
          if (p.bits == 16) {
            v = h2f(reinterpret_cast<const __half*>(p.lv)[row * rv + r]);
          } else {
            const __half* sz = p.lvsz + row * p.ngv * 2 + (r / p.g) * 2;
            v = fmaf((float)int4_at(p.lv + row * p.lv_row, r), h2f(sz[0]), h2f(sz[1]));
          }
        }
        vt[t * vstr + r] = v;
      }
      if (p.resid) {
        for (int e = tid; e < g.tt * kResidDim; e += kThreads) {
          const int t = e / kResidDim, i = e % kResidDim;
          float yk = 0.f, yv = 0.f;
          if (t < nt) {
            const int64_t row = lowrank_row(p, b, kvh, t0 + t);
            yk = ((float)int2_at(p.rkc + row * (kResidDim / 4), i) - 1.5f) * h2f(p.rks[row]);
            yv = ((float)int2_at(p.rvc + row * (kResidDim / 4), i) - 1.5f) * h2f(p.rvs[row]);
          }
          if (g.recon) rt[t * kResidDim + i] = yk;
          else kt[t * kstr + rk + i] = yk;
          vt[t * vstr + rv + i] = yv;
        }
      }
      if (g.recon) {
        __syncthreads();
        if (p.resid) {
          // e_t = Q^T y_t = diag(signs) H y_t / sqrt(128), one transform per token
          for (int t = 0; t < g.tt; ++t) fwht_smem(rt + t * kResidDim, kResidDim, tid, kThreads);
        }
        const int d = p.d, half = d / 2;
        const float inv = rsqrtf((float)kResidDim);
        for (int e = tid; e < g.tt * half; e += kThreads) {
          const int t = e / half, i = e % half;
          float a = 0.f, c = 0.f;
          for (int r = 0; r < rk; ++r) {
            const float lr = lt[t * lstr + r];
            a = fmaf(lr, bks[r * d + i], a);
            c = fmaf(lr, bks[r * d + i + half], c);
          }
          if (p.resid) {
            a = fmaf((float)p.signs_k[i] * inv, rt[t * kResidDim + i], a);
            c = fmaf((float)p.signs_k[i + half] * inv, rt[t * kResidDim + i + half], c);
          }
          // RoPE at position t0 + t: angle in turns reduced to [-1/2, 1/2]
          const double turns = (double)(t0 + t) * p.rope_f[i];
          const float fr = (float)(turns - rint(turns));
          float sn, cs;
          sincospif(2.f * fr, &sn, &cs);
          kt[t * kstr + i] = a * cs - c * sn;
          kt[t * kstr + i + half] = c * cs + a * sn;
        }
      }
    } else if (p.kind == KVC_VARRATE) {
      const uint8_t* ks = p.lk + (size_t)b * p.stream_bytes;
      const uint8_t* vs = p.lv + (size_t)b * p.stream_bytes;
      for (int e = tid; e < g.tt * 64; e += kThreads) {
        const int t = e / 64, r = e % 64;
        float vk = 0.f, vv = 0.f;
        if (t < nt) {
          const int tok = t0 + t;
          const int64_t mi = (int64_t)b * p.tmax + tok;
          const int rkt = p.rank_k[mi], rvt = p.rank_v[mi];
          if (r < rkt) {
            const uint8_t* rec = ks + p.off_k[(int64_t)b * (p.tmax + 1) + tok] +
                                 kvh * varrate_head_bytes(rkt);
            const __half* sz = reinterpret_cast<const __half*>(rec + rkt / 2) + (r / 32) * 2;
            vk = fmaf((float)int4_at(rec, r), h2f(sz[0]), h2f(sz[1]));
          }
          if (r < rvt) {
            const uint8_t* rec = vs + p.off_v[(int64_t)b * (p.tmax + 1) + tok] +
                                 kvh * varrate_head_bytes(rvt);
            const __half* sz = reinterpret_cast<const __half*>(rec + rvt / 2) + (r / 32) * 2;
            vv = fmaf((float)int4_at(rec, r), h2f(sz[0]), h2f(sz[1]));
          }
        }
        kt[t * kstr + r] = vk;
        vt[t * vstr + r] = vv;
      }
    } else if (p.kind == KVC_BLOCK_SHARED) {
      const int D = p.D, ng = D / p.g;
      const int kb = D * p.bits / 8, vb = D * p.vbits / 8;
      for (int e = tid; e < g.tt * D; e += kThreads) {
        const int t = e / D, c = e % D;
        float v = 0.f, w = 0.f;
        if (t < nt) {
          const int64_t mi = (int64_t)b * p.tmax + t0 + t;
          v = (float)sym_level_at(p.lk + mi * kb, c, p.bits) * h2f(p.lksz[mi * ng + c / p.g]);
          if (p.vbits)
            w = (float)sym_level_at(p.lv + mi * vb, c, p.vbits) * h2f(p.lvsz[mi * ng + c / p.g]);
        }
        kt[t * kstr + c] = v;
        if (p.vbits) vt[t * vstr + c] = w;
      }
    } else {  // dense bf16
      const int d = p.d;
      const int64_t base = (((int64_t)l * p.B + b) * p.Hkv + kvh) * p.tmax;
      for (int e = tid; e < g.tt * d; e += kThreads) {
        const int t = e / d, i = e % d;
        float vk = 0.f, vv = 0.f;
        if (t < nt) {
          vk = bf2f(p.kd[(base + t0 + t) * d + i]);
          vv = bf2f(p.vd[(base + t0 + t) * d + i]);
        }
        kt[t * kstr + i] = vk;
        vt[t * vstr + i] = vv;
      }
    }
    __syncthreads();

    // ---------------- scores (log2 units)
    for (int e = tid; e < g.nq * g.tt; e += kThreads) {
      const int i = e / g.tt, t = e % g.tt;
      float s = -INFINITY;
      if (t < nt) {
        const float* qq = qs + i * g.kd;
        const float* kk = kt + t * kstr;
        float a = 0.f;
        for (int k = 0; k < g.kd; ++k) a = fmaf(qq[k], kk[k], a);
        s = a * p.scale_log2;
      }
      sc[e] = s;
    }
    __syncthreads();

    // ---------------- online softmax, one warp per query
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = warp + k * nwarps;
      if (i >= g.nq) break;
      float mx = -INFINITY;
      for (int t = lane; t < g.tt; t += 32) mx = fmaxf(mx, sc[i * g.tt + t]);
      mx = warp_max(mx);
      const float m_new = fmaxf(m_q[k], mx);
      const float alpha = exp2f(m_q[k] - m_new);   // 0 when m_q was -inf
      float sum = 0.f;
      for (int t = lane; t < g.tt; t += 32) {
        const float pv = exp2f(sc[i * g.tt + t] - m_new);
        sc[i * g.tt + t] = pv;
        sum += pv;
      }
      sum = warp_sum(sum);
      l_q[k] = l_q[k] * alpha + sum;
      m_q[k] = m_new;
      if (lane == 0) al[i] = alpha;
    }
    __syncthreads();

    // ---------------- acc = acc * alpha + P V
#pragma unroll
    for (int k = 0; k < kMaxAcc; ++k) {
      const int e = tid + k * kThreads;
      if (k < nacc && e < g.nq * g.vd) {
        const int i = e / g.vd, j = e % g.vd;
        float a = acc[k] * al[i];
        const float* pp = sc + i * g.tt;
        for (int t = 0; t < nt; ++t) a = fmaf(pp[t], vt[t * vstr + j], a);
        acc[k] = a;
      }
    }
    __syncthreads();
  }

  // ---------------- partials
  const size_t rows = (size_t)p.L * p.B * p.Hq;
  const int pst = p.vdim + 2;
#pragma unroll
  for (int k = 0; k < kMaxAcc; ++k) {
    const int e = tid + k * kThreads;
    if (k < nacc && e < g.nq * g.vd) {
      const int i = e / g.vd, j = e % g.vd;
      p.part[((size_t)blockIdx.x * rows + qrow(i)) * pst + j] = acc[k];
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = warp + k * nwarps;
    if (i < g.nq && lane == 0) {
      float* dst = p.part + ((size_t)blockIdx.x * rows + qrow(i)) * pst + p.vdim;
      dst[0] = m_q[k];
      dst[1] = l_q[k];
    }
  }
}

}  // namespace

cudaError_t launch_split(const Params& p, cudaStream_t s) {
  switch (p.path) {
    case 1: return launch_rope_tc(p, p.err, s);
    case 2: return launch_dense_tc(p, s);
    case 3: return launch_latent_tc(p, s);
    case 4: return launch_rope_mma(p, s);
    case 7: return launch_rope_wg(p, s);
    case 5: return launch_varrate_warp(p, s);
    case 6: return launch_block_mma(p, s);
    case 8: return launch_block_tc(p, s);
    case 9: return launch_varrate_mma(p, s);
    default: break;
  }
  const Geo g = geometry(p);
  const Smem S = carve(p, g);
  const size_t bytes = (size_t)S.total * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(split_generic_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  int units;
  if (p.kind == KVC_BLOCK_SHARED) units = p.B * (p.L * p.Hq / kBlockQueries);
  else units = p.L * p.B * p.Hkv;
  dim3 grid(p.S, units);
  split_generic_kernel<<<grid, kThreads, bytes, s>>>(p);
  return cudaGetLastError();
}

}  // namespace kvc
