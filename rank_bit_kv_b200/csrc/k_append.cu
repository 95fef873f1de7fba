// Append: project each new token's pre-RoPE key / value onto the latent and
// quantize it into its slot (contiguous row, page slot or ragged record).
//
//   l = x Bk^T                                     (fp32, summed over d in order)
//   INT4 per group: z = fp16(min), s = fp16((max - min) / 15),
//                   code = clamp(rint((l - z) / s), 0, 15)  (IEEE fp32 divide,
//                   round half to even; code 0 when s == 0)
//   residual:       e = x - l_hat Bk, y = H (diag(signs) e) / sqrt(128),
//                   s = fp16(max|y| / 1.5), code = clamp(floor(y / s) + 2, 0, 3)
//   block-shared:   b-bit symmetric, s = fp16(max|x| / (2^(b-1) - 1)),
//                   code = clamp(rint(x / s), -(2^(b-1) - 1), 2^(b-1) - 1) + 2^(b-1)
// The INT4 rule is the per-group min/max uniform quantizer of the BellowsKV
// page ("Worked Example: Why the Latent Quantizes Flat"): fifteen equal steps
// between the group's extremes, each value coded by its nearest step, here with
// the step and the offset stored in fp16.
//
// A bulk append of INT4 rows without the residual (prefill) stages the factor
// once per block of tokens and gives each token to one warp; the arithmetic is
// the same, term by term.
//
// pos and the VARRATE ranks are device arrays, so the kernels validate them:
// rows with a slot range outside the cache, tokens with a bad rank or page id,
// and records that would run past their stream are skipped (never written out
// of bounds) and reported by KVC_DEV_* bits in the optional status word.
#include <math.h>

#include "kvc_device.cuh"

namespace kvc {
namespace {

constexpr int kThreads = 128;

__device__ __forceinline__ void flag(uint32_t* status, uint32_t bit) {
  if (status) atomicOr(status, bit);
}

// First slot of row b's new tokens, or -1 when pos[b] leaves the cache.
__device__ __forceinline__ int first_slot(const AppendParams& a, int b) {
  const int p0 = a.pos[b];
  return (p0 < 0 || p0 > a.p.tmax - a.n_new) ? -1 : p0;
}

__device__ __forceinline__ bool varrate_rank_ok(int r) {
  return r == 4 || r == 8 || r == 16 || r == 32 || r == 64;
}

// Quantize lat[0..r) in groups of g into packed INT4 codes and (s, z) pairs.
__device__ void quant_int4_asym(const float* lat, int r, int g, uint8_t* codes, __half* sz,
                                float* lhat, int tid) {
  __shared__ float gs[64], gz[64];
  const int ng = (r + g - 1) / g;
  if (tid < ng) {
    const int a = tid * g, e = min(a + g, r);
    float lo = lat[a], hi = lat[a];
    for (int j = a + 1; j < e; ++j) lo = fminf(lo, lat[j]), hi = fmaxf(hi, lat[j]);
    const __half z = __float2half_rn(lo);
    const __half s = __float2half_rn((hi - lo) / 15.f);
    gs[tid] = __half2float(s);
    gz[tid] = __half2float(z);
    sz[2 * tid] = s;
    sz[2 * tid + 1] = z;
  }
  __syncthreads();
  for (int i = tid; i < r / 2; i += kThreads) {
    int c2[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int j = 2 * i + k, gi = j / g;
      const float s = gs[gi], z = gz[gi];
      int c = 0;
      if (s > 0.f) c = (int)fminf(fmaxf(rintf((lat[j] - z) / s), 0.f), 15.f);
      c2[k] = c;
      if (lhat) lhat[j] = fmaf((float)c, s, z);
    }
    codes[i] = (uint8_t)(c2[0] | (c2[1] << 4));
  }
  __syncthreads();
}

// The factor's r rows are staged in shared memory first (coalesced 4-byte
// loads, rows padded to kFsRow halves so that lane j reading row j is
// conflict-free), so the projection and the residual read no global memory in
// their loops.
constexpr int kFsRow = 130;

__global__ void __launch_bounds__(kThreads) append_lowrank_kernel(AppendParams a) {
  const Params& p = a.p;
  __shared__ __align__(16) __half fsm[128 * kFsRow];
  __shared__ float xs[128];
  __shared__ float lat[128];
  __shared__ float lhat[128];
  __shared__ float ys[128];
  __shared__ float red[kThreads / 32];
  // grid: ((b * Hkv + h) * 2 + comp) * n_new + i
  int idx = blockIdx.x;
  const int i = idx % a.n_new;
  idx /= a.n_new;
  const int comp = idx % 2;
  idx /= 2;
  const int h = idx % p.Hkv;
  const int b = idx / p.Hkv;
  const int tid = threadIdx.x;
  const int d = p.d;
  const int p0 = first_slot(a, b);
  if (p0 < 0) {                       // whole block leaves before any barrier
    if (tid == 0 && h == 0 && comp == 0 && i == 0) flag(a.status, KVC_DEV_BAD_POS);
    return;
  }
  const int tok = p0 + i;
  if (p.page) {
    const int pp = p.page_table[(int64_t)b * (p.tmax / p.page) + tok / p.page];
    if (pp < 0 || pp >= p.n_pages) {
      if (tid == 0 && h == 0 && comp == 0) flag(a.status, KVC_DEV_BAD_PAGE);
      return;
    }
  }
  const __nv_bfloat16* src = (comp == 0 ? a.k_new : a.v_new) + (((int64_t)b * p.Hkv + h) * a.n_new + i) * d;
  for (int j = tid; j < d; j += kThreads) xs[j] = bf2f(src[j]);

  int r;
  const __half* fac;
  if (p.kind == KVC_VARRATE) {
    // stored by the offsets kernel: 0 when the token was skipped
    r = (comp == 0 ? a.rank_k_w : a.rank_v_w)[(int64_t)b * p.tmax + tok];
    if (!varrate_rank_ok(r)) return;
    fac = (comp == 0 ? p.bk : p.bv) + (int64_t)h * 64 * d;
  } else {
    r = comp == 0 ? p.rk : p.rv;
    fac = (comp == 0 ? p.bk : p.bv) + (int64_t)h * r * d;
  }
  for (int e = tid; e < r * (d / 2); e += kThreads) {
    const int row = e / (d / 2), c2 = e % (d / 2);
    *reinterpret_cast<uint32_t*>(fsm + row * kFsRow + 2 * c2) =
        __ldg(reinterpret_cast<const unsigned int*>(fac + (int64_t)row * d + 2 * c2));
  }
  __syncthreads();
  for (int j = tid; j < r; j += kThreads) {
    const __half* br = fsm + j * kFsRow;
    float acc = 0.f;
    for (int k = 0; k < d; ++k) acc = fmaf(xs[k], h2f(br[k]), acc);
    lat[j] = acc;
  }
  __syncthreads();

  if (p.kind == KVC_VARRATE) {
    const int* off = comp == 0 ? a.off_k_w : a.off_v_w;
    uint8_t* stream = (comp == 0 ? a.lk_w : a.lv_w) + (size_t)b * p.stream_bytes;
    const int64_t o = (int64_t)off[(int64_t)b * (p.tmax + 1) + tok] + h * varrate_head_bytes(r);
    if (o < 0 || o + varrate_head_bytes(r) > (int64_t)p.stream_bytes) {
      if (tid == 0) flag(a.status, KVC_DEV_BAD_OFFSET);
      return;
    }
    uint8_t* rec = stream + o;
    quant_int4_asym(lat, r, 32, rec, reinterpret_cast<__half*>(rec + r / 2), nullptr, tid);
    return;
  }
  const int64_t row = lowrank_row(p, b, h, tok);
  if (p.bits == 16) {
    __half* dst = reinterpret_cast<__half*>(comp == 0 ? a.lk_w : a.lv_w) + row * r;
    for (int j = tid; j < r; j += kThreads) dst[j] = __float2half_rn(lat[j]);
    return;
  }
  uint8_t* codes = (comp == 0 ? a.lk_w : a.lv_w) + row * (r / 2);
  __half* sz = (comp == 0 ? a.lksz_w : a.lvsz_w) + row * 2 * ((r + p.g - 1) / p.g);
  quant_int4_asym(lat, r, p.g, codes, sz, p.resid ? lhat : nullptr, tid);
  if (!p.resid) return;

  // residual against the dequantized latent, rotated into the Hadamard basis
  const int8_t* sg = comp == 0 ? p.signs_k : p.signs_v;
  for (int j = tid; j < d; j += kThreads) {
    float e = xs[j];
    for (int k = 0; k < r; ++k) e = fmaf(-lhat[k], h2f(fsm[k * kFsRow + j]), e);
    ys[j] = (float)sg[j] * e;
  }
  fwht_smem(ys, kResidDim, tid, kThreads);
  const float inv = rsqrtf((float)kResidDim);
  float amax = 0.f;
  for (int j = tid; j < d; j += kThreads) {
    ys[j] *= inv;
    amax = fmaxf(amax, fabsf(ys[j]));
  }
  amax = warp_max(amax);
  if ((tid & 31) == 0) red[tid >> 5] = amax;
  __syncthreads();
  float m = red[0];
  for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, red[w]);
  const __half sh = __float2half_rn(m / 1.5f);
  const float s = __half2float(sh);
  if (tid == 0) (comp == 0 ? a.rks_w : a.rvs_w)[row] = sh;
  uint8_t* rc = (comp == 0 ? a.rkc_w : a.rvc_w) + row * (kResidDim / 4);
  for (int j = tid; j < kResidDim / 4; j += kThreads) {
    int byte = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      int c = 2;
      if (s > 0.f) c = (int)fminf(fmaxf(floorf(ys[4 * j + k] / s) + 2.f, 0.f), 3.f);
      byte |= c << (2 * k);
    }
    rc[j] = (uint8_t)byte;
  }
}

// VARRATE: ranks and offsets of the new records, offset[pos + i + 1] =
// offset[pos + i] + size.  A token whose K or V rank is outside the set, or
// whose record would run past the stream, is stored as an empty record of
// rank 0 (the append kernel then skips it and decode ignores it).
__global__ void varrate_offsets_kernel(AppendParams a) {
  const Params& p = a.p;
  const int comp = blockIdx.x % 2, b = blockIdx.x / 2;
  if (threadIdx.x != 0) return;
  const int p0 = first_slot(a, b);
  if (p0 < 0) {
    if (comp == 0) flag(a.status, KVC_DEV_BAD_POS);
    return;
  }
  int* off = (comp == 0 ? a.off_k_w : a.off_v_w) + (int64_t)b * (p.tmax + 1);
  uint8_t* rank = (comp == 0 ? a.rank_k_w : a.rank_v_w) + (int64_t)b * p.tmax;
  const uint8_t* nk = a.new_ranks + (int64_t)b * a.n_new;
  const uint8_t* nv = a.new_ranks + ((int64_t)p.B + b) * a.n_new;
  int64_t o = off[p0];
  bool dead = o < 0 || o > (int64_t)p.stream_bytes;
  if (dead) flag(a.status, KVC_DEV_BAD_OFFSET);
  for (int i = 0; i < a.n_new; ++i) {
    const int rk = nk[i], rv = nv[i];
    const bool ok = varrate_rank_ok(rk) && varrate_rank_ok(rv);
    if (!ok && comp == 0) flag(a.status, KVC_DEV_BAD_RANK);
    int size = (ok && !dead) ? p.Hkv * varrate_head_bytes(comp == 0 ? rk : rv) : 0;
    if (size && o + size > (int64_t)p.stream_bytes) {
      dead = true;
      size = 0;
      flag(a.status, KVC_DEV_BAD_OFFSET);
    }
    rank[p0 + i] = size ? (uint8_t)(comp == 0 ? rk : rv) : 0;
    o += size;
    off[p0 + i + 1] = (int)o;
  }
}

__global__ void __launch_bounds__(kThreads) append_block_kernel(AppendParams a) {
  const Params& p = a.p;
  // grid: ((b * n_new + i) * ncomp + comp); comp 1 is the separate value latent
  const int ncomp = p.vbits ? 2 : 1;
  int idx = blockIdx.x;
  const int comp = idx % ncomp;
  idx /= ncomp;
  const int i = idx % a.n_new, b = idx / a.n_new;
  const int p0 = first_slot(a, b);
  if (p0 < 0) {
    if (threadIdx.x == 0 && i == 0 && comp == 0) flag(a.status, KVC_DEV_BAD_POS);
    return;
  }
  const int tok = p0 + i;
  const int D = p.D, g = p.g, ng = D / g;
  const int bits = comp ? p.vbits : p.bits;
  const int qmax = (1 << (bits - 1)) - 1, zero_code = 1 << (bits - 1);
  const __nv_bfloat16* src = (comp ? a.v_new : a.k_new) + ((int64_t)b * a.n_new + i) * D;
  const int64_t mi = (int64_t)b * p.tmax + tok;
  uint8_t* codes = (comp ? a.lv_w : a.lk_w) + mi * (D * bits / 8);
  __half* sc = (comp ? a.lvsz_w : a.lksz_w) + mi * ng;
  __shared__ float gsc[64];
  for (int gi = threadIdx.x; gi < ng; gi += kThreads) {
    float m = 0.f;
    for (int j = gi * g; j < (gi + 1) * g; ++j) m = fmaxf(m, fabsf(bf2f(src[j])));
    const __half sh = __float2half_rn(m / (float)qmax);
    sc[gi] = sh;
    gsc[gi] = __half2float(sh);
  }
  __syncthreads();
  // eight codes per thread: element e in bits [bits e, bits e + bits) of the row
  for (int j = threadIdx.x; j < D / 8; j += kThreads) {
    uint64_t word = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int e = 8 * j + k;
      const float s = gsc[e / g];
      int c = zero_code;
      if (s > 0.f)
        c = (int)fminf(fmaxf(rintf(bf2f(src[e]) / s), (float)-qmax), (float)qmax) + zero_code;
      word |= (uint64_t)c << (bits * k);
    }
    for (int k = 0; k < bits; ++k) codes[(size_t)j * bits + k] = (uint8_t)(word >> (8 * k));
  }
}

__global__ void append_dense_kernel(AppendParams a) {
  const Params& p = a.p;
  // grid: ((l * B + b) * Hkv + h) * n_new + i
  int idx = blockIdx.x;
  const int i = idx % a.n_new;
  idx /= a.n_new;
  const int h = idx % p.Hkv;
  idx /= p.Hkv;
  const int b = idx % p.B;
  const int l = idx / p.B;
  const int d = p.d;
  const int p0 = first_slot(a, b);
  if (p0 < 0) {
    if (threadIdx.x == 0 && i == 0 && h == 0 && l == 0) flag(a.status, KVC_DEV_BAD_POS);
    return;
  }
  const int64_t src = ((((int64_t)l * p.B + b) * p.Hkv + h) * a.n_new + i) * d;
  const int64_t dst = ((((int64_t)l * p.B + b) * p.Hkv + h) * p.tmax + p0 + i) * d;
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    a.kd_w[dst + j] = a.k_new[src + j];
    a.vd_w[dst + j] = a.v_new[src + j];
  }
}

// Bulk append (prefill) of INT4 low-rank rows without the residual: one block
// per (chunk of kBulkTok tokens, batch row, KV head, K or V).  The factor rows
// are staged once in shared memory as fp32 (rows padded to 132 floats, so the
// 16-byte loads of 8 lanes reading 8 rows are conflict-free); each warp takes
// kBulkGroup tokens at a time, lane j forming latent entries j and j + 32 of
// all of them from one read of its factor rows, each entry summed over d in
// the order of append_lowrank_kernel (so the codes are the same); then the
// groups' minimum and maximum by shuffles and the codes, two per byte.
constexpr int kBulkTok = 256;
constexpr int kBulkThreads = 256;
constexpr int kBulkGroup = 8;                    // tokens per warp pass
constexpr int kBulkRow = 132;                    // floats per staged factor row

__global__ void __launch_bounds__(kBulkThreads) append_lowrank_bulk_kernel(AppendParams a) {
  const Params& p = a.p;
  extern __shared__ __align__(16) float fs[];    // [r][132] factor rows, then x [8 warps][8][128]
  const int chunk = blockIdx.x;
  int idx = blockIdx.y;                          // (b * Hkv + h) * 2 + comp
  const int comp = idx & 1;
  idx >>= 1;
  const int h = idx % p.Hkv, b = idx / p.Hkv;
  const int p0 = first_slot(a, b);
  if (p0 < 0) {
    if (threadIdx.x == 0 && h == 0 && comp == 0 && chunk == 0) flag(a.status, KVC_DEV_BAD_POS);
    return;
  }
  const int r = comp == 0 ? p.rk : p.rv;
  const int ng = (r + 31) / 32;
  const __half* fac = (comp == 0 ? p.bk : p.bv) + (int64_t)h * r * 128;
  for (int e = threadIdx.x; e < r * 128; e += kBulkThreads) fs[(e >> 7) * kBulkRow + (e & 127)] = h2f(fac[e]);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rmax = p.rk > p.rv ? p.rk : p.rv;
  float* xs = fs + rmax * kBulkRow + warp * kBulkGroup * 128;
  __syncthreads();
  const int i_end = min(a.n_new, (chunk + 1) * kBulkTok);
  for (int i0 = chunk * kBulkTok + warp * kBulkGroup; i0 < i_end; i0 += (kBulkThreads / 32) * kBulkGroup) {
    // the group's rows of x (zeros past the end)
#pragma unroll
    for (int t = 0; t < kBulkGroup; ++t) {
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i0 + t < i_end) {
        const __nv_bfloat16* src = (comp == 0 ? a.k_new : a.v_new) +
                                   (((int64_t)b * p.Hkv + h) * a.n_new + i0 + t) * 128;
        const uint2 u = *reinterpret_cast<const uint2*>(src + 4 * lane);
        const __nv_bfloat162 x01 = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
        const __nv_bfloat162 x23 = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
        v = make_float4(__low2float(x01), __high2float(x01), __low2float(x23), __high2float(x23));
      }
      *reinterpret_cast<float4*>(xs + t * 128 + 4 * lane) = v;
    }
    __syncwarp();
    float lat[2][kBulkGroup];
#pragma unroll
    for (int t = 0; t < kBulkGroup; ++t) lat[0][t] = lat[1][t] = 0.f;
    const bool two = lane + 32 < r;
    const float* b0 = fs + lane * kBulkRow;
    const float* b1 = fs + (two ? lane + 32 : lane) * kBulkRow;
#pragma unroll 2
    for (int k = 0; k < 128; k += 4) {
      const float4 w0 = *reinterpret_cast<const float4*>(b0 + k);
      const float4 w1 = *reinterpret_cast<const float4*>(b1 + k);
#pragma unroll
      for (int t = 0; t < kBulkGroup; ++t) {
        const float4 x = *reinterpret_cast<const float4*>(xs + t * 128 + k);
        lat[0][t] = fmaf(x.x, w0.x, lat[0][t]);
        lat[0][t] = fmaf(x.y, w0.y, lat[0][t]);
        lat[0][t] = fmaf(x.z, w0.z, lat[0][t]);
        lat[0][t] = fmaf(x.w, w0.w, lat[0][t]);
        lat[1][t] = fmaf(x.x, w1.x, lat[1][t]);
        lat[1][t] = fmaf(x.y, w1.y, lat[1][t]);
        lat[1][t] = fmaf(x.z, w1.z, lat[1][t]);
        lat[1][t] = fmaf(x.w, w1.w, lat[1][t]);
      }
    }
#pragma unroll
    for (int t = 0; t < kBulkGroup; ++t) {
      const int i = i0 + t;
      if (i >= i_end) break;
      const int tok = p0 + i;
      if (p.page) {
        const int pp = p.page_table[(int64_t)b * (p.tmax / p.page) + tok / p.page];
        if (pp < 0 || pp >= p.n_pages) {
          if (lane == 0 && h == 0 && comp == 0) flag(a.status, KVC_DEV_BAD_PAGE);
          continue;
        }
      }
      const int64_t row = lowrank_row(p, b, h, tok);
      uint8_t* codes = (comp == 0 ? a.lk_w : a.lv_w) + row * (r / 2);
      __half* sz = (comp == 0 ? a.lksz_w : a.lvsz_w) + row * 2 * ng;
      for (int gi = 0; gi < ng; ++gi) {
        const int j = lane + 32 * gi;
        const bool in = j < r;
        const float v = gi == 0 ? lat[0][t] : lat[1][t];
        float lo = in ? v : INFINITY, hi = in ? v : -INFINITY;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
          hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        const __half zh = __float2half_rn(lo);
        const __half sh = __float2half_rn((hi - lo) / 15.f);
        const float s = __half2float(sh), z = __half2float(zh);
        int c = 0;
        if (in && s > 0.f) c = (int)fminf(fmaxf(rintf((v - z) / s), 0.f), 15.f);
        const int cn = __shfl_down_sync(0xffffffffu, c, 1);
        if (in && !(lane & 1)) codes[j >> 1] = (uint8_t)(c | (cn << 4));
        if (lane == 0) {
          sz[2 * gi] = sh;
          sz[2 * gi + 1] = zh;
        }
      }
    }
    __syncwarp();                                // xs is rewritten by the next group
  }
}

bool bulk_ok(const AppendParams& a) {
  const Params& p = a.p;
  return p.kind == KVC_LOWRANK && p.bits == 4 && p.g == 32 && !p.resid && p.d == 128 &&
         p.rk <= 64 && p.rv <= 64 && a.n_new >= 64;
}

}  // namespace

cudaError_t launch_append(const AppendParams& a, cudaStream_t s) {
  const Params& p = a.p;
  switch (p.kind) {
    case KVC_LOWRANK:
      if (bulk_ok(a)) {
        const int rmax = p.rk > p.rv ? p.rk : p.rv;
        const size_t smem =
            ((size_t)rmax * kBulkRow + (kBulkThreads / 32) * kBulkGroup * 128) * sizeof(float);
        cudaError_t e = cudaFuncSetAttribute(append_lowrank_bulk_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        dim3 grid((a.n_new + kBulkTok - 1) / kBulkTok, p.B * p.Hkv * 2);
        append_lowrank_bulk_kernel<<<grid, kBulkThreads, smem, s>>>(a);
      } else {
        append_lowrank_kernel<<<p.B * p.Hkv * 2 * a.n_new, kThreads, 0, s>>>(a);
      }
      break;
    case KVC_VARRATE:
      varrate_offsets_kernel<<<p.B * 2, 32, 0, s>>>(a);
      append_lowrank_kernel<<<p.B * p.Hkv * 2 * a.n_new, kThreads, 0, s>>>(a);
      break;
    case KVC_BLOCK_SHARED:
      append_block_kernel<<<p.B * a.n_new * (p.vbits ? 2 : 1), kThreads, 0, s>>>(a);
      break;
    default:
      append_dense_kernel<<<p.L * p.B * p.Hkv * a.n_new, 128, 0, s>>>(a);
      break;
  }
  return cudaGetLastError();
}

}  // namespace kvc
