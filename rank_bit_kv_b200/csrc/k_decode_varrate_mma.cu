// Split-T decode on the variable-rate layout (per-token ranks, ragged records;
// VarRate "Method") on warp-level tensor cores.
//
// The per-token ranks differ, so the contraction is written at the full rank
// (64) with every code beyond a token's rank masked to zero, and only the
// zero-point terms depend on the rank:
//   s_t = 2^24 sum_g s_{t,g} (c_t . q~)_g + sum_g z_{t,g} sum_{i in g, i < r_t} q~_i
//   acc_i = sum_t p_t s_{t,g(i)} c_{t,i} + sum_{t: r_t > i} p_t z_{t,g(i)}
// Warp (KV head h, half) takes 16 tokens of every 32-token chunk: the scores
// are an MMA with the tokens as M, the rank as K (the 4 query heads of the KV
// head as N), the values an MMA with the latent dims as M, the tokens as K.
// Codes enter the MMAs as f16 subnormals (c 2^-24; value codes centred,
// (c - 8) 2^-24, the zero terms then taking z + 8 s); k-steps and M-tiles that
// no token of the group reaches are skipped; the zero terms are summed per
// rank class.  The CTA projects its batch row's queries itself (q~ = Bk q),
// stages each chunk's byte ranges of the K and V streams with 16-byte
// cp.async (a ring of three chunks, one CTA barrier per chunk), and merges the
// two halves of every head into one partial per row.
//
// Selectable (kvc_select_varrate_kernel(1)); the lane-per-head kernel stays the
// default: with every warp synchronised per 32-token chunk this kernel spends
// ~6 800 cycles per chunk (copy and metadata issue ~1 600, score operands and
// MMAs ~1 400, score arithmetic ~1 100, softmax ~1 800, values ~700) and
// measured 125 us for the C4 step's kernel against 58 us.
#include <math.h>

#include "kvc_device.cuh"
#include "tc_util.cuh"

namespace kvc {
namespace {

using namespace tc;

constexpr int kMHkv = 8, kMG = 4, kMR = 64;
constexpr int kMWarps = 16;                          // (KV head, half of the chunk)
constexpr int kMThreads = 32 * kMWarps;
constexpr int kMChunk = 32;                          // tokens per staged chunk
constexpr int kMRec = kMHkv * (kMR / 2 + 8);         // token record bytes at rank 64
constexpr int kMBuf = kMChunk * kMRec + 32;          // one staged stream chunk (+ slack)
constexpr int kMQRow = kMR + 4;                      // floats per q~ row
constexpr int kMStages = 3;                          // staged chunks (ring)
constexpr int kMSlots = 4;                           // metadata slots (ring)
constexpr int OFF_STAGE = 0;                         // [kMStages buffers][K, V]
constexpr int OFF_META = OFF_STAGE + 2 * kMStages * kMBuf;   // [slots][ok 33, ov 33, rkv 32] ints
constexpr int kMeta = 2 * (kMChunk + 1) + kMChunk;
constexpr int OFF_Q = OFF_META + kMSlots * kMeta * 4;        // q~ [32][68] fp32
constexpr int OFF_X = OFF_Q + 32 * kMQRow * 4;       // the row's queries [32][128] fp32
constexpr int kMSmem = OFF_X + 32 * 128 * 4;
constexpr int kMPst = kMR + 2;                       // merge slot: o[64], m, l

static_assert(kMThreads == kMHkv * kMR, "one thread per (KV head, rank) row of Bk");
static_assert(kMHkv * kMG * kMPst * 4 <= 2 * kMStages * kMBuf, "merge area fits in the staging area");

__host__ __device__ constexpr int head_bytes(int r) { return r / 2 + 4 * ((r + 31) / 32); }

__device__ __forceinline__ bool rank_ok(int r) {
  return r == 4 || r == 8 || r == 16 || r == 32 || r == 64;
}

__device__ __forceinline__ void cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all_groups() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void cp_wait_one_group() {
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}

__device__ __forceinline__ uint32_t h2u(__half2 x) { return *reinterpret_cast<uint32_t*>(&x); }
__device__ __forceinline__ __half2 u2h2(uint32_t x) { return *reinterpret_cast<__half2*>(&x); }

// code byte (two INT4 codes, element 2i in the low nibble) -> f16x2 subnormals
__device__ __forceinline__ uint32_t sub2(uint32_t byte) {
  return (byte & 0xFu) | ((byte & 0xF0u) << 12);
}
constexpr uint32_t kCentre = 0x00080008u;            // 8 * 2^-24 in both halves

// (scale, zero) fp16 pair at a 2-byte aligned address (a head record of rank 4
// is 6 bytes long, so its pair is not always 4-byte aligned)
__device__ __forceinline__ float2 sz_at(const uint8_t* q) {
  const __half* hp = reinterpret_cast<const __half*>(q);
  return make_float2(__half2float(hp[0]), __half2float(hp[1]));
}

__device__ __forceinline__ uint32_t hsub_u32(uint32_t x, uint32_t c) {
  return h2u(__hsub2(u2h2(x), u2h2(c)));
}

__global__ void __launch_bounds__(kMThreads, 1) varrate_mma_kernel(Params p, int split_len) {
  extern __shared__ __align__(128) uint8_t vsm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c4 = lane & 3;
  const int h = warp & 7, half = warp >> 3;
  const int s_idx = blockIdx.x, b = blockIdx.y;
  const int T = p.n_tokens;
  const int cta_a = s_idx * split_len, cta_b = min(T, cta_a + split_len);

  const uint8_t* const kstream = p.lk + (size_t)b * p.stream_bytes;
  const uint8_t* const vstream = p.lv + (size_t)b * p.stream_bytes;
  const int* const offk = p.off_k + (size_t)b * (p.tmax + 1);
  const int* const offv = p.off_v + (size_t)b * (p.tmax + 1);
  const uint8_t* const rkg = p.rank_k + (size_t)b * p.tmax;
  const uint8_t* const rvg = p.rank_v + (size_t)b * p.tmax;
  const long long sbytes = (long long)p.stream_bytes;
  int* const meta = reinterpret_cast<int*>(vsm + OFF_META);

  // ---- staging of chunk c: its metadata (threads 0..32, loaded into
  // registers one iteration before it is stored into slot c % 4), then the
  // byte ranges of both streams into buffer c % 3, from the 16-byte boundary
  // below, clamped to the stream and the buffer; the copies of chunk c are
  // issued while chunk c - 2 is computed
  int m_ok = 0, m_ov = 0, m_rkv = 0;                 // this thread's metadata of the next chunk
  auto meta_load = [&](int c) {
    const int t0 = cta_a + c * kMChunk;
    const int n = min(kMChunk, cta_b - t0);
    if (tid <= n) {
      m_ok = __ldg(offk + t0 + tid);
      m_ov = __ldg(offv + t0 + tid);
    }
    m_rkv = tid < n ? (int)__ldg(rkg + t0 + tid) | ((int)__ldg(rvg + t0 + tid) << 8) : 0;
  };
  auto meta_store = [&](int c) {
    int* mt = meta + (c % kMSlots) * kMeta;
    const int t0 = cta_a + c * kMChunk;
    const int n = min(kMChunk, cta_b - t0);
    if (tid <= n) {
      mt[tid] = m_ok;
      mt[kMChunk + 1 + tid] = m_ov;
    }
    if (tid < kMChunk) mt[2 * (kMChunk + 1) + tid] = m_rkv;
  };
  auto copies = [&](int c) {
    const int* mt = meta + (c % kMSlots) * kMeta;
    const int t0 = cta_a + c * kMChunk;
    const int n = min(kMChunk, cta_b - t0);
    const uint32_t dst = smem_u32(vsm + OFF_STAGE + (c % kMStages) * 2 * kMBuf);
#pragma unroll
    for (int sv = 0; sv < 2; ++sv) {
      const int* o = mt + sv * (kMChunk + 1);
      const long long base = (long long)(o[0] & ~15);
      const long long e = min((long long)o[n], sbytes);
      long long nch = (e - base + 15) / 16;
      if (base < 0 || base >= sbytes) nch = 0;
      nch = min(nch, (long long)(kMBuf / 16));
      const uint8_t* src = (sv ? vstream : kstream) + base;
      for (int k = tid; k < nch; k += kMThreads) cp16(dst + sv * kMBuf + 16 * k, src + 16 * k);
    }
    cp_commit();
  };

  // ---- q~ = Bk q for the row's 32 query heads (softmax scale and log2 e
  // folded in): thread (kvh, j) dots row j of head kvh's Bk with its 4 queries
  float* const qsm = reinterpret_cast<float*>(vsm + OFF_Q);
  {
    float* const xs = reinterpret_cast<float*>(vsm + OFF_X);
    for (int e = tid; e < 32 * 128; e += kMThreads) xs[e] = bf2f(p.q[(size_t)b * p.Hq * 128 + e]);
    __syncthreads();
    const int kvh = tid / kMR, j = tid % kMR;
    const uint4* br = reinterpret_cast<const uint4*>(p.bk + ((size_t)kvh * kMR + j) * 128);
    float a4[kMG] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int c = 0; c < 16; ++c) {
      const uint4 w = __ldg(br + c);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __half22float2(u2h2(ws[k]));
#pragma unroll
        for (int gq = 0; gq < kMG; ++gq) {
          const float* xg = xs + (kvh * kMG + gq) * 128 + 8 * c + 2 * k;
          a4[gq] = fmaf(f.x, xg[0], a4[gq]);
          a4[gq] = fmaf(f.y, xg[1], a4[gq]);
        }
      }
    }
#pragma unroll
    for (int gq = 0; gq < kMG; ++gq) qsm[(kvh * kMG + gq) * kMQRow + j] = a4[gq] * p.scale_log2;
  }
  const int n_chunks = (cta_b - cta_a + kMChunk - 1) / kMChunk;
  __syncthreads();                                   // q~ complete
  if (n_chunks > 0) {
    meta_load(0);
    meta_store(0);
  }
  if (n_chunks > 1) {
    meta_load(1);
    meta_store(1);
  }

  // ---- this warp's query operand (B of the score MMA: k = rank, n = query g)
  // and the prefix sums of q~ for the zero terms (lanes c4 < 2: queries 2c4, 2c4 + 1)
  uint32_t qb[4][2];
  {
    const float* qr = qsm + (h * kMG + (g & 3)) * kMQRow;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const int d0 = 16 * ks + 2 * c4;
      qb[ks][0] = g < kMG ? pack_h2(qr[d0], qr[d0 + 1]) : 0u;
      qb[ks][1] = g < kMG ? pack_h2(qr[d0 + 8], qr[d0 + 9]) : 0u;
    }
  }
  float pre[2][5];                                   // [query e][r = 4, 8, 16, 32 | dims 32..63]
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const float* qr = qsm + (h * kMG + ((2 * c4 + e) & 3)) * kMQRow;
    float run = 0.f;
#pragma unroll 8
    for (int i = 0; i < kMR; ++i) {
      if (i == 32) run = 0.f;
      run += qr[i];
      if (i == 3) pre[e][0] = run;
      if (i == 7) pre[e][1] = run;
      if (i == 15) pre[e][2] = run;
      if (i == 31) pre[e][3] = run;
      if (i == 63) pre[e][4] = run;
    }
  }
  __syncthreads();                                   // metadata of chunks 0, 1 stored
  if (n_chunks > 0) copies(0);
  if (n_chunks > 1) copies(1);
  if (n_chunks > 2) meta_load(2);

  float acc[4][4];                                   // [M-tile][(dim g | g + 8) x (query 2c4 | + 1)]
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
  float zc[6][2];                                    // zero terms per rank class and query
#pragma unroll
  for (int k = 0; k < 6; ++k) zc[k][0] = zc[k][1] = 0.f;
  float m_ref[2] = {-INFINITY, -INFINITY}, m_thr[2] = {-INFINITY, -INFINITY};
  float l_sum[2] = {0.f, 0.f};

  for (int c = 0; c < n_chunks; ++c) {
    // metadata of chunk c + 2 (loaded during the previous iteration) into its
    // slot; that slot last served chunk c - 2, which every warp has finished
    if (c + 2 < n_chunks) meta_store(c + 2);
    // this thread's copies of chunk c have landed (those of chunk c + 1 may
    // still be in flight)
    if (c + 1 < n_chunks) cp_wait_one_group();
    else cp_wait_all_groups();
    __syncthreads();                                 // chunk c visible; chunk c - 1 is done
    if (c + 2 < n_chunks) copies(c + 2);             // into the buffer chunk c - 1 used
    if (c + 3 < n_chunks) meta_load(c + 3);

    const int* mt_ = meta + (c % kMSlots) * kMeta;
    const uint8_t* kb = vsm + OFF_STAGE + (c % kMStages) * 2 * kMBuf;
    const uint8_t* vb = kb + kMBuf;
    const int t0 = cta_a + c * kMChunk;
    const int n = min(kMChunk, cta_b - t0);
    const int base_k = mt_[0] & ~15, base_v = mt_[kMChunk + 1] & ~15;
    // ---- the two rows of this lane: tokens 16 half + g (+ 8) of the chunk
    int rk[2], rv[2], ko[2], vo[2];
    bool ok[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int j = 16 * half + g + 8 * r;
      const int rkv = j < n ? mt_[2 * (kMChunk + 1) + j] : 0;
      rk[r] = rkv & 255;
      rv[r] = rkv >> 8;
      const int okk = j < n ? mt_[j] - base_k : -1;
      const int ovv = j < n ? mt_[kMChunk + 1 + j] - base_v : -1;
      // records outside the staged area or off their 16-byte grid (offsets
      // inconsistent with the ranks) make the token count for nothing
      ok[r] = j < n && rank_ok(rk[r]) && rank_ok(rv[r]) && okk >= 0 && !(okk & 15) &&
              okk + kMHkv * head_bytes(rk[r]) <= kMBuf && ovv >= 0 && !(ovv & 15) &&
              ovv + kMHkv * head_bytes(rv[r]) <= kMBuf;
      if (!ok[r]) rk[r] = rv[r] = 0;
      ko[r] = ok[r] ? okk + h * head_bytes(rk[r]) : 0;
      vo[r] = ok[r] ? ovv + h * head_bytes(rv[r]) : 0;
    }
    int kmax = max(rk[0], rk[1]), vmax = max(rv[0], rv[1]);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
      vmax = max(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    }

    // ---- scores: M = 16 tokens, K = rank (k-steps below the group's largest rank)
    float dg[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      if (16 * ks < kmax) {
        uint32_t a[4];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int d0 = 16 * ks + 2 * c4;
          a[r] = d0 < rk[r] ? sub2(kb[ko[r] + 8 * ks + c4]) : 0u;
          a[2 + r] = d0 + 8 < rk[r] ? sub2(kb[ko[r] + 8 * ks + 4 + c4]) : 0u;
        }
        mma16816(dg[ks >> 1], a, qb[ks][0], qb[ks][1]);
      }
    }
    float s[2][2];                                   // [row][query e]
    float sv_s[2][2], sv_z[2][2];                    // V scale / zero per [row][group]
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float2 k0 = make_float2(0.f, 0.f), k1 = make_float2(0.f, 0.f);
      float2 v0 = make_float2(0.f, 0.f), v1 = make_float2(0.f, 0.f);
      if (ok[r]) {
        k0 = sz_at(kb + ko[r] + rk[r] / 2);
        if (rk[r] == kMR) k1 = sz_at(kb + ko[r] + rk[r] / 2 + 4);
        v0 = sz_at(vb + vo[r] + rv[r] / 2);
        if (rv[r] == kMR) v1 = sz_at(vb + vo[r] + rv[r] / 2 + 4);
      }
      sv_s[r][0] = v0.x;
      sv_z[r][0] = v0.y;
      sv_s[r][1] = v1.x;
      sv_z[r][1] = v1.y;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        // sum of q~ over the token's first min(r, 32) entries
        const float pr = rk[r] == 4 ? pre[e][0] : rk[r] == 8 ? pre[e][1]
                       : rk[r] == 16 ? pre[e][2] : pre[e][3];
        float v = 16777216.f * fmaf(k0.x, dg[0][2 * r + e], k1.x * dg[1][2 * r + e]);
        v = fmaf(k0.y, pr, v);
        if (rk[r] == kMR) v = fmaf(k1.y, pre[e][4], v);
        s[r][e] = (ok[r] && c4 < 2) ? v : -INFINITY;
      }
    }

    // ---- online softmax per query over the group's 16 tokens (lazily raised maximum)
    float mx[2] = {fmaxf(s[0][0], s[1][0]), fmaxf(s[0][1], s[1][1])};
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx[0] = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], o));
      mx[1] = fmaxf(mx[1], __shfl_xor_sync(0xffffffffu, mx[1], o));
    }
    const bool need = mx[0] > m_thr[0] || mx[1] > m_thr[1];
    if (__any_sync(0xffffffffu, need)) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float nm = fmaxf(m_ref[e], mx[e]);
        // 0 while nothing was seen; 1 (no change) while nothing is seen at all
        const float al = nm == -INFINITY ? 1.f : ex2_approx(m_ref[e] - nm);
        l_sum[e] *= al;
#pragma unroll
        for (int k = 0; k < 6; ++k) zc[k][e] *= al;
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) acc[mt][e] *= al, acc[mt][2 + e] *= al;
        m_ref[e] = nm;
        m_thr[e] = nm + 8.f;
      }
    }
    float pv[2][2];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        pv[r][e] = s[r][e] == -INFINITY ? 0.f : ex2_approx(s[r][e] - m_ref[e]);
        l_sum[e] += pv[r][e];
      }
    // zero terms per rank class (class k: rank 4 << k on the first group; 5: the second group)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int cls = rv[r] == 4 ? 0 : rv[r] == 8 ? 1 : rv[r] == 16 ? 2 : rv[r] == 32 ? 3 : 4;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float t0z = pv[r][e] * fmaf(8.f, sv_s[r][0], sv_z[r][0]);
#pragma unroll
        for (int k = 0; k < 5; ++k)
          if (cls == k) zc[k][e] += t0z;
        zc[5][e] = fmaf(pv[r][e], fmaf(8.f, sv_s[r][1], sv_z[r][1]), zc[5][e]);
      }
    }

    // ---- values: M = 16 latent dims per tile, K = the 16 tokens, N = queries
    uint32_t bq[2][2];                               // [group][tokens 0..7 | 8..15]
#pragma unroll
    for (int gr = 0; gr < 2; ++gr)
#pragma unroll
      for (int r = 0; r < 2; ++r)
        bq[gr][r] = movmatrix_trans(pack_h2(pv[r][0] * sv_s[r][gr], pv[r][1] * sv_s[r][gr]));
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      if (16 * mt < vmax) {
        uint32_t x[2][2];                            // [token block][dim block 2mt | 2mt + 1]
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int db = 0; db < 2; ++db) {
            const int bblk = 2 * mt + db;            // dims 8 bblk + 2c4, + 1
            const bool in = 8 * bblk + 2 * c4 < rv[r];
            x[r][db] = in ? hsub_u32(sub2(vb[vo[r] + 4 * bblk + c4]), kCentre) : 0u;
          }
        const uint32_t a[4] = {movmatrix_trans(x[0][0]), movmatrix_trans(x[0][1]),
                               movmatrix_trans(x[1][0]), movmatrix_trans(x[1][1])};
        mma16816(acc[mt], a, bq[mt >> 1][0], bq[mt >> 1][1]);
      }
    }
  }
  cp_wait_all_groups();

  // ---- finish: sums over the g lanes, dims = 2^24 acc + zero terms, then the
  // two halves of each head merge into one partial per row
#pragma unroll
  for (int e = 0; e < 2; ++e) {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l_sum[e] += __shfl_xor_sync(0xffffffffu, l_sum[e], o);
#pragma unroll
      for (int k = 0; k < 6; ++k) zc[k][e] += __shfl_xor_sync(0xffffffffu, zc[k][e], o);
    }
  }
  auto zero_term = [&](int dim, int e) -> float {
    if (dim >= 32) return zc[5][e];
    float z = zc[4][e] + zc[3][e];
    if (dim < 16) z += zc[2][e];
    if (dim < 8) z += zc[1][e];
    if (dim < 4) z += zc[0][e];
    return z;
  };
  __syncthreads();                                   // staging buffers become the merge area
  float* mg = reinterpret_cast<float*>(vsm + OFF_STAGE);
  if (half == 1 && c4 < 2) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float* slot = mg + (h * kMG + 2 * c4 + e) * kMPst;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        slot[16 * mt + g] = fmaf(16777216.f, acc[mt][e], zero_term(16 * mt + g, e));
        slot[16 * mt + g + 8] = fmaf(16777216.f, acc[mt][2 + e], zero_term(16 * mt + g + 8, e));
      }
      if (g == 0) {
        slot[kMR] = m_ref[e];
        slot[kMR + 1] = l_sum[e];
      }
    }
  }
  __syncthreads();
  if (half == 0 && c4 < 2) {
    const size_t rows = (size_t)p.L * p.B * p.Hq;
    const int pst = p.vdim + 2;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float* slot = mg + (h * kMG + 2 * c4 + e) * kMPst;
      const float m1 = slot[kMR], l1 = slot[kMR + 1];
      const float M = fmaxf(m_ref[e], m1);
      const float w0 = (m_ref[e] == -INFINITY) ? 0.f : ex2_approx(m_ref[e] - M);
      const float w1 = (m1 == -INFINITY) ? 0.f : ex2_approx(m1 - M);
      const size_t orow = (size_t)b * p.Hq + h * kMG + 2 * c4 + e;
      float* dst = p.part + ((size_t)s_idx * rows + orow) * pst;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int dim = 16 * mt + g + 8 * rr;
          const float own = fmaf(16777216.f, acc[mt][2 * rr + e], zero_term(dim, e));
          dst[dim] = own * w0 + slot[dim] * w1;
        }
      }
      if (g == 0) {
        dst[p.vdim] = M;
        dst[p.vdim + 1] = l_sum[e] * w0 + l1 * w1;
      }
    }
  }
}

}  // namespace

bool varrate_mma_supported(const Params& p) {
  return p.kind == KVC_VARRATE && p.Hkv == kMHkv && p.G == kMG && p.L == 1 && !p.seq_lens &&
         p.n_tokens > 0 && p.qdim == kMR && p.vdim == kMR && p.g == 32 &&
         p.stream_bytes % 16 == 0 && p.d == 128;
}

// CTAs per batch row (one partial each) and tokens per CTA
void varrate_mma_plan(const Params& p, int* splits, int* split_len) {
  int s = kNumSMs / (p.B > 0 ? p.B : 1);
  if (s < 1) s = 1;
  const int max_s = (p.n_tokens + kMChunk - 1) / kMChunk;
  if (s > max_s) s = max_s;
  if (s < 1) s = 1;
  *split_len = (p.n_tokens + s - 1) / s;
  *splits = (p.n_tokens + *split_len - 1) / *split_len;
}

cudaError_t launch_varrate_mma(const Params& p, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(varrate_mma_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kMSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.S, p.B);
  varrate_mma_kernel<<<grid, kMThreads, kMSmem, s>>>(p, p.split_len);
  return cudaGetLastError();
}

}  // namespace kvc
