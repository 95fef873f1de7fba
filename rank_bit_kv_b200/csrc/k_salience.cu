// Token-importance producers: query salience, per-token ranks by salience, and
// one keep decision per block of layers with its compaction.
//
// "VarRate: Training-Free Variable-Rate KV Cache Compression ...", "Summary"
// and "Method": each token gets a low-rank budget chosen by its query
// salience, never zero.  "BellowsKV Architecture ...", "Three Measurements,
// Three Operators": the layers of a block agree on which tokens matter, so one
// importance decision per block, from all n layers' scores, is applied once to
// the shared latent.
//
//   salience_t = sum over query heads h and window queries w of
//                softmax_t(scale * q_{h,w} . k_{kv(h),t})
//
// Two tensor-core passes over the dense prefill keys (bf16, head dim 128): the
// first forms each window row's softmax maximum and sum (online, per token
// split, then merged), the second sums the normalised probabilities over the
// rows of a KV head per token (one partial per KV head, no atomics).  The
// rank / keep selection ranks tokens by (salience descending, position
// ascending) exactly: a radix select on 64-bit keys finds the key at every
// rung boundary, and a token's rung is the number of boundaries at or below
// its key.
#include <math.h>

#include "kvc_device.cuh"
#include "tc_util.cuh"

namespace kvc {
namespace {

using namespace tc;

constexpr int kSD = 128;               // head dim
constexpr int kSRows = 128;            // window rows per CTA (heads x window queries)
constexpr int kSWarps = 8;             // 16 rows each
constexpr int kSTile = 64;             // tokens per key tile
constexpr int kSRowB = 272;            // shared bytes per staged key row (no bank conflicts)
constexpr int kSSplits = 32;           // token splits per (row, KV head) in the first pass

struct SalParams {
  const __nv_bfloat16* q;              // [B, Hq, W, 128]
  const __nv_bfloat16* k;              // [B, Hkv, cap, 128]
  int B, Hq, Hkv, W, cap, T;
  float scale_log2;
  float* part_ml;                      // [kSSplits, B * Hq * W, 2]  (max in log2 units, sum)
  float* ml;                           // [B * Hq * W, 2]
  float* part_sal;                     // [B, Hkv, T]
};

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Rows of a CTA: 128 consecutive (head, window) rows of KV head kvh's group,
// row r <-> query head kvh * G + r / W, window query r % W (rows past G * W
// are padding).  Scores of a 64-token tile, rows 16 w + g (+8), tokens 8 nt +
// 2 c4 (+1), in log2 units.
struct ScoreTile {
  float s[8][4];
};

// Shared: query rows [128][272 B] (bf16), key tile [64][272 B] double-buffered.
template <int PASS>
__global__ void __launch_bounds__(32 * kSWarps) salience_kernel(SalParams p, int rows_per_kv,
                                                                 int ctas_per_kv) {
  extern __shared__ __align__(16) uint8_t ssm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c4 = lane & 3;
  // grid: x = token split (PASS 0) or token tile block (PASS 1), y = (b, kvh, row block)
  const int yb = blockIdx.y;
  const int rb = yb % ctas_per_kv, bk = yb / ctas_per_kv;
  const int kvh = bk % p.Hkv, b = bk / p.Hkv;
  const int G = p.Hq / p.Hkv;
  const int row_base = rb * kSRows;                  // first row of this CTA in the KV head's rows
  uint8_t* qs = ssm;
  uint8_t* ks = ssm + kSRows * kSRowB;
  const uint32_t ks_s = smem_u32(ks), qs_s = smem_u32(qs);
  // ---- query rows (zero past the group's rows)
  for (int c = threadIdx.x; c < kSRows * 16; c += blockDim.x) {
    const int r = c >> 4, col = c & 15;
    const int rr = row_base + r;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (rr < rows_per_kv) {
      const int h = kvh * G + rr / p.W, w = rr % p.W;
      v = *reinterpret_cast<const uint4*>(p.q + ((((size_t)b * p.Hq + h) * p.W + w) * kSD) + col * 8);
    }
    *reinterpret_cast<uint4*>(qs + r * kSRowB + col * 16) = v;
  }
  // token range of this CTA
  const int tiles = (p.T + kSTile - 1) / kSTile;
  const int per = (tiles + gridDim.x - 1) / gridDim.x;
  const int j0 = blockIdx.x * per, j1 = min(tiles, j0 + per);
  auto issue = [&](int j, int buf) {
    if (j < j1) {
      for (int c = threadIdx.x; c < kSTile * 16; c += blockDim.x) {
        const int r = c >> 4, col = c & 15;
        const int t = j * kSTile + r;
        const bool valid = t < p.T;
        const __nv_bfloat16* src =
            p.k + (((size_t)b * p.Hkv + kvh) * p.cap + (valid ? t : 0)) * kSD + col * 8;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                         ks_s + buf * kSTile * kSRowB + r * kSRowB + col * 16),
                     "l"(src), "r"(valid ? 16 : 0)
                     : "memory");
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  __syncthreads();
  // A fragments of this warp's 16 rows (8 k-steps), once
  uint32_t qa[8][4];
  {
    const int mi = lane >> 3, rr = lane & 7;
    const int row = 16 * warp + rr + 8 * (mi & 1), col = 8 * (mi >> 1);
#pragma unroll
    for (int ks8 = 0; ks8 < 8; ++ks8) ldsm_x4(qa[ks8], qs_s + row * kSRowB + (16 * ks8 + col) * 2);
  }
  const size_t nrows = (size_t)p.B * p.Hq * p.W;
  // rows of this thread (global row index, or -1 for padding)
  int grow[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int rr = row_base + 16 * warp + g + 8 * e;
    grow[e] = rr < rows_per_kv ? (int)((((size_t)b * p.Hq + kvh * G + rr / p.W) * p.W) + rr % p.W) : -1;
  }
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};   // PASS 0 state
  float mr[2] = {0.f, 0.f}, il[2] = {0.f, 0.f};             // PASS 1: row max, 1 / sum
  if (PASS == 1) {
#pragma unroll
    for (int e = 0; e < 2; ++e)
      if (grow[e] >= 0) {
        mr[e] = p.ml[2 * grow[e]];
        il[e] = 1.f / p.ml[2 * grow[e] + 1];
      }
  }
  float* red = reinterpret_cast<float*>(ssm + kSRows * kSRowB + 2 * kSTile * kSRowB);   // [8][64]
  issue(j0, 0);
  int it = 0;
  for (int j = j0; j < j1; ++j, ++it) {
    issue(j + 1, (it + 1) & 1);
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncthreads();
    const uint32_t kb = ks_s + (it & 1) * kSTile * kSRowB;
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
    {
      const int mi = lane >> 3, rr = lane & 7;
      // B fragments: tokens (n) = rows of the key tile, dims (k): matrices
      // (n-tile, k half) -> non-transposed ldmatrix of key rows
      const int trow = rr + 8 * (mi >> 1), tcol = 8 * (mi & 1);
#pragma unroll
      for (int ks8 = 0; ks8 < 8; ++ks8) {
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t bb[4];
          ldsm_x4(bb, kb + (16 * np + trow) * kSRowB + (16 * ks8 + tcol) * 2);
          mma_bf16(s[2 * np], qa[ks8], bb[0], bb[1]);
          mma_bf16(s[2 * np + 1], qa[ks8], bb[2], bb[3]);
        }
      }
    }
    const int tbase = j * kSTile;
    if (PASS == 0) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float mx = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int t = tbase + 8 * nt + 2 * c4 + q;
            const float v = t < p.T ? s[nt][2 * e + q] * p.scale_log2 : -INFINITY;
            s[nt][2 * e + q] = v;
            mx = fmaxf(mx, v);
          }
        const float nm = fmaxf(m[e], mx);
        float acc = l[e] * (nm == -INFINITY ? 0.f : exp2f(m[e] - nm));
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int q = 0; q < 2; ++q) acc += nm == -INFINITY ? 0.f : exp2f(s[nt][2 * e + q] - nm);
        m[e] = nm;
        l[e] = acc;
      }
    } else {
      // column sums over this warp's 16 rows, then over the 8 warps
      float col[8][2];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          float v = 0.f;
#pragma unroll
          for (int e = 0; e < 2; ++e)
            if (grow[e] >= 0) v += exp2f(s[nt][2 * e + q] * p.scale_log2 - mr[e]) * il[e];
#pragma unroll
          for (int o = 4; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          col[nt][q] = v;
        }
      if (g == 0) {
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int q = 0; q < 2; ++q) red[warp * kSTile + 8 * nt + 2 * c4 + q] = col[nt][q];
      }
      __syncthreads();
      for (int c = threadIdx.x; c < kSTile; c += blockDim.x) {
        const int t = tbase + c;
        float v = 0.f;
        for (int w = 0; w < kSWarps; ++w) v += red[w * kSTile + c];
        if (t < p.T) {
          p.part_sal[((size_t)b * p.Hkv + kvh) * p.T + t] = v;
        }
      }
    }
    __syncthreads();                 // the key buffer is refilled by the next issue
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  if (PASS == 0) {
    // this thread's rows: reduce (m, l) over the 4 threads of a row (c4)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float mm = m[e], ll = l[e];
#pragma unroll
      for (int o = 1; o < 4; o <<= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, mm, o), l2 = __shfl_xor_sync(0xffffffffu, ll, o);
        const float nm = fmaxf(mm, m2);
        ll = (nm == -INFINITY) ? 0.f : ll * exp2f(mm - nm) + l2 * exp2f(m2 - nm);
        mm = nm;
      }
      if (c4 == 0 && grow[e] >= 0) {
        float* dst = p.part_ml + ((size_t)blockIdx.x * nrows + grow[e]) * 2;
        dst[0] = mm;
        dst[1] = ll;
      }
    }
  }
}

// Merge the splits' (max, sum) of every window row.
__global__ void merge_ml_kernel(SalParams p, int splits) {
  const size_t nrows = (size_t)p.B * p.Hq * p.W;
  for (size_t r = blockIdx.x * blockDim.x + threadIdx.x; r < nrows; r += gridDim.x * blockDim.x) {
    float mm = -INFINITY, ll = 0.f;
    for (int s = 0; s < splits; ++s) {
      const float m2 = p.part_ml[((size_t)s * nrows + r) * 2], l2 = p.part_ml[((size_t)s * nrows + r) * 2 + 1];
      const float nm = fmaxf(mm, m2);
      if (nm == -INFINITY) continue;
      ll = ll * exp2f(mm - nm) + l2 * exp2f(m2 - nm);
      mm = nm;
    }
    p.ml[2 * r] = mm;
    p.ml[2 * r + 1] = ll;
  }
}

// salience = sum over the KV heads' partials, in head order
__global__ void sum_heads_kernel(const float* part_sal, int Hkv, int T, float* sal) {
  const int b = blockIdx.y;
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  float v = 0.f;
  for (int h = 0; h < Hkv; ++h) v += part_sal[((size_t)b * Hkv + h) * T + t];
  sal[(size_t)b * T + t] = v;
}

// ---------------------------------------------------------------- selection

constexpr int kSelThreads = 1024;
constexpr int kMaxRungs = 8;

// 64-bit order key: salience descending, then position ascending.
__device__ __forceinline__ uint64_t order_key(float v, int t) {
  return ((uint64_t)(~__float_as_uint(fmaxf(v, 0.f))) << 32) | (uint32_t)t;
}

// One CTA per batch row: sal[t] = sum over KV heads of the partials (fixed
// order) when part_sal is given, else sal is read as is; find the keys at the
// boundary positions bound[0..nb) by an 8-pass radix select; class_out[t] =
// number of boundaries whose key is <= the token's key.
__device__ void select_classes(float* sal, int T, const int* bound, int nb, uint64_t* kb_out,
                               unsigned* hist) {
  __shared__ uint64_t prefix[kMaxRungs];
  __shared__ int remaining[kMaxRungs];
  if (threadIdx.x < nb) {
    prefix[threadIdx.x] = 0;
    remaining[threadIdx.x] = bound[threadIdx.x];
  }
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = threadIdx.x; i < nb * 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
      const uint64_t key = order_key(sal[t], t);
      for (int k = 0; k < nb; ++k) {
        const uint64_t hi_mask = pass == 0 ? 0ull : (~0ull << (shift + 8));
        if ((key & hi_mask) == prefix[k]) atomicAdd(&hist[k * 256 + ((key >> shift) & 255)], 1u);
      }
    }
    __syncthreads();
    if (threadIdx.x < nb) {
      const int k = threadIdx.x;
      unsigned cum = 0;
      int d = 0;
      for (; d < 256; ++d) {
        if (cum + hist[k * 256 + d] > (unsigned)remaining[k]) break;
        cum += hist[k * 256 + d];
      }
      remaining[k] -= (int)cum;
      prefix[k] |= (uint64_t)d << shift;
    }
    __syncthreads();
  }
  if (threadIdx.x < nb) kb_out[threadIdx.x] = prefix[threadIdx.x];
  __syncthreads();
}

__global__ void __launch_bounds__(kSelThreads) ranks_kernel(const float* part_sal, int Hkv,
                                                            float* sal, int B, int T,
                                                            RankLadder lad, uint8_t* ranks) {
  __shared__ unsigned hist[kMaxRungs * 256];
  __shared__ uint64_t kbound[kMaxRungs];
  const int b = blockIdx.x;
  float* row = sal + (size_t)b * T;
  if (part_sal) {
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
      float v = 0.f;
      for (int h = 0; h < Hkv; ++h) v += part_sal[((size_t)b * Hkv + h) * T + t];
      row[t] = v;
    }
    __syncthreads();
  }
  // boundary positions: cumulative counts of all rungs but the last, clipped to T
  int bound[kMaxRungs];
  int nb = 0, cum = 0;
  for (int i = 0; i + 1 < lad.n; ++i) {
    cum += lad.count[i];
    if (cum >= T) break;
    bound[nb++] = cum;
  }
  select_classes(row, T, bound, nb, kbound, hist);
  for (int t = threadIdx.x; t < T; t += blockDim.x) {
    const uint64_t key = order_key(row[t], t);
    int cls = 0;
    for (int k = 0; k < nb; ++k) cls += key >= kbound[k];
    const uint8_t r = (uint8_t)lad.rank[cls];
    ranks[(size_t)b * T + t] = r;                       // K ranks
    ranks[((size_t)B + b) * T + t] = r;                 // V ranks (same salience)
  }
}

// Keep decision of a block: importance = sum of the layers' saliences (fixed
// order); kept positions are the `keep` first of the order, written ascending.
__global__ void __launch_bounds__(kSelThreads) keep_kernel(const float* sal_layers, int n_layers,
                                                           float* importance, int B, int T,
                                                           int keep, int* kept) {
  __shared__ unsigned hist[256];
  __shared__ uint64_t kbound[1];
  __shared__ int wsum[kSelThreads / 32];
  const int b = blockIdx.x;
  float* row = importance + (size_t)b * T;
  for (int t = threadIdx.x; t < T; t += blockDim.x) {
    float v = 0.f;
    for (int l = 0; l < n_layers; ++l) v += sal_layers[((size_t)l * B + b) * T + t];
    row[t] = v;
  }
  __syncthreads();
  int bound[1] = {keep};
  const int nb = keep < T ? 1 : 0;
  select_classes(row, T, bound, nb, kbound, hist);
  // stable compaction of the kept positions (key below the boundary's key)
  int base = 0;
  for (int t0 = 0; t0 < T; t0 += blockDim.x) {
    const int t = t0 + threadIdx.x;
    const bool k = t < T && (nb == 0 || order_key(row[t], t) < kbound[0]);
    const unsigned m = __ballot_sync(0xffffffffu, k);
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    if (lane == 0) wsum[w] = __popc(m);
    __syncthreads();
    int before = 0, total = 0;
    for (int i = 0; i < (int)(blockDim.x / 32); ++i) {
      if (i < w) before += wsum[i];
      total += wsum[i];
    }
    if (k) kept[(size_t)b * keep + base + before + __popc(m & ((1u << lane) - 1u))] = t;
    base += total;
    __syncthreads();
  }
}

// Copy the kept rows of a block-shared latent (codes + scales) into a compacted
// cache: dst row i of batch row b <- src row kept[b][i].
__global__ void compact_kernel(const uint8_t* src_codes, const __half* src_scales, uint8_t* dst_codes,
                               __half* dst_scales, const int* kept, int B, int cap_src, int cap_dst,
                               int keep, int code_bytes, int n_scales) {
  const int i = blockIdx.x, b = blockIdx.y;
  const int t = kept[(size_t)b * keep + i];
  const uint8_t* sc = src_codes + ((size_t)b * cap_src + t) * code_bytes;
  uint8_t* dc = dst_codes + ((size_t)b * cap_dst + i) * code_bytes;
  for (int c = threadIdx.x; c < code_bytes / 16; c += blockDim.x)
    reinterpret_cast<uint4*>(dc)[c] = reinterpret_cast<const uint4*>(sc)[c];
  const __half* ss = src_scales + ((size_t)b * cap_src + t) * n_scales;
  __half* ds = dst_scales + ((size_t)b * cap_dst + i) * n_scales;
  for (int c = threadIdx.x; c < n_scales; c += blockDim.x) ds[c] = ss[c];
}

size_t sal_smem() { return (size_t)kSRows * kSRowB + 2 * kSTile * kSRowB + kSWarps * kSTile * 4; }

}  // namespace

size_t salience_workspace_bytes(int B, int Hq, int Hkv, int W, int T) {
  const size_t rows = (size_t)B * Hq * W;
  size_t b = (size_t)kSSplits * rows * 2 * 4;
  b = (b + 255) / 256 * 256 + (rows * 2 * 4 + 255) / 256 * 256;
  b += ((size_t)B * Hkv * T * 4 + 255) / 256 * 256;
  return b;
}

cudaError_t launch_salience(const SalienceCall& c, cudaStream_t s) {
  SalParams p;
  p.q = c.q;
  p.k = c.k;
  p.B = c.B;
  p.Hq = c.Hq;
  p.Hkv = c.Hkv;
  p.W = c.W;
  p.cap = c.cap;
  p.T = c.T;
  p.scale_log2 = c.scale * 1.4426950408889634f;
  char* ws = (char*)c.workspace;
  const size_t rows = (size_t)c.B * c.Hq * c.W;
  p.part_ml = (float*)ws;
  size_t off = ((size_t)kSSplits * rows * 2 * 4 + 255) / 256 * 256;
  p.ml = (float*)(ws + off);
  off += (rows * 2 * 4 + 255) / 256 * 256;
  p.part_sal = (float*)(ws + off);
  const int G = c.Hq / c.Hkv;
  const int rows_per_kv = G * c.W;
  const int ctas_per_kv = (rows_per_kv + kSRows - 1) / kSRows;
  const size_t sm = sal_smem();
  cudaError_t e = cudaFuncSetAttribute(salience_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(salience_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const int tiles = (c.T + kSTile - 1) / kSTile;
  const int splits = tiles < kSSplits ? tiles : kSSplits;
  salience_kernel<0><<<dim3(splits, c.B * c.Hkv * ctas_per_kv), 32 * kSWarps, sm, s>>>(p, rows_per_kv, ctas_per_kv);
  merge_ml_kernel<<<(int)((rows + 255) / 256), 256, 0, s>>>(p, splits);
  // second pass: 8 key tiles per CTA; the rows of a KV head fit one CTA, so
  // every (b, KV head, token) partial is written by exactly one thread
  const int blocks = (tiles + 7) / 8;
  salience_kernel<1><<<dim3(blocks, c.B * c.Hkv * ctas_per_kv), 32 * kSWarps, sm, s>>>(p, rows_per_kv, ctas_per_kv);
  sum_heads_kernel<<<dim3((c.T + 255) / 256, c.B), 256, 0, s>>>(p.part_sal, c.Hkv, c.T, c.sal);
  return cudaGetLastError();
}

cudaError_t launch_ranks(const float* part_sal, int Hkv, float* sal, int B, int T,
                         const RankLadder& lad, uint8_t* ranks, cudaStream_t s) {
  ranks_kernel<<<B, kSelThreads, 0, s>>>(part_sal, Hkv, sal, B, T, lad, ranks);
  return cudaGetLastError();
}

cudaError_t launch_keep(const float* sal_layers, int n_layers, float* importance, int B, int T,
                        int keep, int* kept, cudaStream_t s) {
  keep_kernel<<<B, kSelThreads, 0, s>>>(sal_layers, n_layers, importance, B, T, keep, kept);
  return cudaGetLastError();
}

cudaError_t launch_compact(const uint8_t* src_codes, const __half* src_scales, uint8_t* dst_codes,
                           __half* dst_scales, const int* kept, int B, int cap_src, int cap_dst,
                           int keep, int code_bytes, int n_scales, cudaStream_t s) {
  if (keep <= 0) return cudaSuccess;
  compact_kernel<<<dim3(keep, B), 64, 0, s>>>(src_codes, src_scales, dst_codes, dst_scales, kept, B,
                                              cap_src, cap_dst, keep, code_bytes, n_scales);
  return cudaGetLastError();
}

}  // namespace kvc
