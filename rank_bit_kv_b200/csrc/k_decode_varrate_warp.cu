// Split-T decode on the variable-rate layout (per-token ranks, ragged records),
// one lane per (KV head, query head) pair.
//
// A token's rank is shared by all KV heads, so every lane of a warp takes the
// same rank branch for the same token; a staged chunk of up to 16 tokens is
// taken class by class (all its key-rank-4 tokens, then rank 8, ...: one loop
// per class instead of a dispatch per token), with one maximum update and
// independent exp2 for the chunk, the weights kept in per-warp slots, and the
// value updates again class by class.  The 8 KV heads x 4 query heads of a
// batch row fill the 32 lanes; each lane keeps its own online softmax (no
// shuffles) and its own latent-space accumulator acc[64] in registers; the
// projected queries q~ = Bk q are formed by the CTA itself on warp-level MMAs
// (warp w: 32 rows of head w / 2) into shared memory, where each lane reads
// its own row:
//   s_t = sum_{i < r_k(t)} q~_i (c_i s_g + z_g),
//   acc_i += p_t (c_i s_g + z_g) for i < r_v(t).
// Keeping q~ out of the registers lets 16 warps share an SM (4 per scheduler)
// to hide the per-token dependency chain.
// The arithmetic is paired: Blackwell's two-wide fp32 instructions
// (fma/sub/mul .f32x2) take two elements per instruction.  Key codes enter the
// dot product as f = 1 + c/16 (exact: the nibble is placed in the top mantissa
// bits), so sum q_i c_i = 16 (sum q_i f_i - sum q_i) needs no per-code
// subtraction; value codes are centred, c - 8, and the zero terms p (z + 8 s)
// of the tokens are summed per rank class and added to the accumulator once,
// at the end, over the indices each class covers.
// Every warp streams a contiguous token range in chunks of up to 16 tokens
// (as many as fit a buffer sized for 8 tokens of rank 64; ~86 bytes per token
// and stream on average): the byte range of the chunk's K records and of its
// V records (contiguous in the per-row streams) is copied with 16-byte
// cp.async into a double-buffered per-warp area while the previous chunk is
// processed.  The chunk's records are validated once (offsets on their
// 16-byte grid and inside the staged area, ranks in the rank set), by the
// lane that holds the token's metadata, which packs offsets, rank classes and
// the validity bit into one word.  The warps of a CTA merge their (m, l, acc)
// in shared memory and write one partial per row; the combine kernel maps acc
// through Bv.
#include <math.h>

#include "kvc_device.cuh"
#include "tc_util.cuh"

namespace kvc {
namespace {

using namespace tc;

constexpr int kVWarps = 16;
constexpr int kVThreads = 32 * kVWarps;
constexpr int kVChunk = 16;                         // tokens per staged chunk at most
constexpr int kVBufTok = 8;                         // tokens of rank 64 a chunk buffer holds
constexpr int kVHkv = 8, kVG = 4;                   // lanes = KV heads x query heads
constexpr int kVRmax = 64;
constexpr int kVRecMax = kVHkv * (kVRmax / 2 + 8);  // token record bytes at rank 64
constexpr int kVBuf = kVBufTok * kVRecMax + 32;     // one staged stream chunk (+ alignment slack)
constexpr int kVWarpBytes = 4 * kVBuf;              // K and V, two buffers each
constexpr int kVStage = kVWarps * kVWarpBytes;
constexpr int kVQRow = kVRmax + 4;                  // floats per q~ row (16-byte loads conflict-free)
constexpr int kVOffQ = kVStage;                     // q~ [32][kVQRow] (softmax scale, log2 e folded)
constexpr int kVOffX = kVOffQ + 32 * kVQRow * 4;    // the queries [32][kVQhRow] f16, then 16 maxima
constexpr int kVQhRow = 136;                        // f16 per staged query row (272 bytes)
constexpr int kVOffS = kVOffX + 32 * 128 * 4;       // the warps' score slots [kVChunk][32]
constexpr int kVSmem = kVOffS + kVWarps * kVChunk * 32 * 4;
constexpr int kVPst = kVRmax + 2;                   // merge slot: acc[64], m, l

static_assert(kVWarps * 32 * kVPst * 4 <= kVStage, "merge area fits in the staging area");
static_assert(kVThreads * 16 == kVHkv * kVRmax * 16, "16 Bk copy pieces per thread");
static_assert(kVHkv * kVRmax * 256 <= kVStage, "Bk's copy fits in the staging area");
static_assert(kVBuf <= 4096, "record offsets in a staged chunk fit in 12 bits");
static_assert(32 * kVQhRow * 2 + kVWarps * 4 <= 32 * 128 * 4, "f16 queries and maxima fit");
static_assert(kVSmem <= 227 * 1024, "shared memory of a CTA");

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

// ---- two-wide fp32 arithmetic (element 0 in the low word)
__device__ __forceinline__ uint64_t pk2(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ uint64_t pkf(float lo, float hi) {
  return pk2(__float_as_uint(lo), __float_as_uint(hi));
}
__device__ __forceinline__ float2 upk(uint64_t v) {
  uint32_t lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
  return make_float2(__uint_as_float(lo), __uint_as_float(hi));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// key codes of word w (nibble 2j = low nibble of byte j, 2j+1 = high nibble) as
// the pairs (1 + c_2j/16, 1 + c_2j+1/16): each nibble is moved to mantissa bits
// 19..22 of the bit pattern of 1.0 (exact)
__device__ __forceinline__ uint64_t key_pair(uint32_t lo, uint32_t hi, int j) {
  const uint32_t sel = 0x7044u | ((uint32_t)j << 8);
  return pk2(prmt(lo, 0x3F000000u, sel), prmt(hi, 0x3F000000u, sel));
}
__device__ __forceinline__ void key_words(uint32_t w, uint32_t& lo, uint32_t& hi) {
  lo = ((w << 3) & 0x78787878u) | 0x80808080u;
  hi = ((w >> 1) & 0x78787878u) | 0x80808080u;
}

// value codes of word w, centred: the pairs (c_2j - 8, c_2j+1 - 8), formed as
// (2^23 + c) - (2^23 + 8) (exact)
__device__ __forceinline__ uint64_t value_pair(uint32_t lo, uint32_t hi, int j) {
  const uint32_t sel = 0x7650u + (uint32_t)j;
  return sub2(pk2(prmt(lo, 0x4B000000u, sel), prmt(hi, 0x4B000000u, sel)),
              pkf(8388616.f, 8388616.f));
}

__device__ __forceinline__ float2 h2f2(uint32_t x) {
  return __half22float2(*reinterpret_cast<const __half2*>(&x));
}
__device__ __forceinline__ float hsum(uint64_t v) {
  const float2 f = upk(v);
  return f.x + f.y;
}

// sum_{i < R} q_i (c_i s_g + z_g) over the record at rec (R/2 code bytes, then
// the groups' (scale, zero) pairs); q = this lane's row of q~ in shared memory,
// pre = its prefix sums: with f_i = 1 + c_i/16,
//   sum_g [16 s_g sum_{i in g} q_i f_i + (z_g - 16 s_g) sum_{i in g} q_i]
template <int R>
__device__ __forceinline__ float score_r(const uint8_t* rec, const float* q,
                                         const float (&pre)[5]) {
  if constexpr (R == 4) {
    const uint32_t w = *reinterpret_cast<const uint16_t*>(rec);
    const float s = __half2float(*reinterpret_cast<const __half*>(rec + 2));
    const float z = __half2float(*reinterpret_cast<const __half*>(rec + 4));
    const ulonglong2 qv = *reinterpret_cast<const ulonglong2*>(q);
    uint32_t lo, hi;
    key_words(w, lo, hi);
    const float d = hsum(fma2(key_pair(lo, hi, 1), qv.y, mul2(key_pair(lo, hi, 0), qv.x)));
    return fmaf(16.f * s, d, fmaf(-16.f, s, z) * pre[0]);
  } else {
    constexpr int NW = R / 8;
    uint64_t dw[NW];                    // one chain per code word (short dependency chains)
#pragma unroll
    for (int wi = 0; wi < NW; ++wi) {
      const ulonglong2 qa = *reinterpret_cast<const ulonglong2*>(q + 8 * wi);
      const ulonglong2 qb = *reinterpret_cast<const ulonglong2*>(q + 8 * wi + 4);
      uint32_t lo, hi;
      key_words(*reinterpret_cast<const uint32_t*>(rec + 4 * wi), lo, hi);
      uint64_t a = mul2(key_pair(lo, hi, 0), qa.x);
      a = fma2(key_pair(lo, hi, 1), qa.y, a);
      a = fma2(key_pair(lo, hi, 2), qb.x, a);
      dw[wi] = fma2(key_pair(lo, hi, 3), qb.y, a);
    }
    float d[2] = {0.f, 0.f};
#pragma unroll
    for (int wi = 0; wi < NW; ++wi) d[wi / 4] += hsum(dw[wi]);
    const float2 sz0 = h2f2(*reinterpret_cast<const uint32_t*>(rec + R / 2));
    constexpr int P = R == 8 ? 1 : R == 16 ? 2 : 3;     // prefix of group 0 up to min(R, 32)
    float s = fmaf(16.f * sz0.x, d[0], fmaf(-16.f, sz0.x, sz0.y) * pre[P]);
    if constexpr (R == 64) {
      const float2 sz1 = h2f2(*reinterpret_cast<const uint32_t*>(rec + R / 2 + 4));
      s += fmaf(16.f * sz1.x, d[1], fmaf(-16.f, sz1.x, sz1.y) * pre[4]);
    }
    return s;
  }
}

// the per-class sums of p (z_g + 8 s_g): index 0..3 for ranks 4..32 (group 0),
// 4 and 5 for the two groups of rank 64; the accumulator takes
//   acc_i += p s_g (c_i - 8) for i < R
// and the class sums are added at the end over the indices each class covers
template <int R>
__device__ __forceinline__ void value_r(const uint8_t* rec, float p, uint64_t (&acc)[kVRmax / 2],
                                        float (&zc)[6]) {
  if constexpr (R == 4) {
    const uint32_t w = *reinterpret_cast<const uint16_t*>(rec);
    const float s = __half2float(*reinterpret_cast<const __half*>(rec + 2));
    const float z = __half2float(*reinterpret_cast<const __half*>(rec + 4));
    const float ps = p * s;
    zc[0] = fmaf(p, fmaf(8.f, s, z), zc[0]);
    const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
    const uint64_t ps2 = pkf(ps, ps);
    acc[0] = fma2(ps2, value_pair(lo, hi, 0), acc[0]);
    acc[1] = fma2(ps2, value_pair(lo, hi, 1), acc[1]);
  } else {
    constexpr int NW = R / 8;
    constexpr int ZC = R == 8 ? 1 : R == 16 ? 2 : R == 32 ? 3 : 4;
    uint64_t ps2[2];
    {
      const float2 sz0 = h2f2(*reinterpret_cast<const uint32_t*>(rec + R / 2));
      const float ps = p * sz0.x;
      ps2[0] = pkf(ps, ps);
      zc[ZC] = fmaf(p, fmaf(8.f, sz0.x, sz0.y), zc[ZC]);
      if constexpr (R == 64) {
        const float2 sz1 = h2f2(*reinterpret_cast<const uint32_t*>(rec + R / 2 + 4));
        const float ps1 = p * sz1.x;
        ps2[1] = pkf(ps1, ps1);
        zc[5] = fmaf(p, fmaf(8.f, sz1.x, sz1.y), zc[5]);
      } else {
        ps2[1] = ps2[0];
      }
    }
#pragma unroll
    for (int wi = 0; wi < NW; ++wi) {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(rec + 4 * wi);
      const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        acc[4 * wi + j] = fma2(ps2[wi / 4], value_pair(lo, hi, j), acc[4 * wi + j]);
    }
  }
}

// the scores of the chunk's tokens of key rank R (bit j of m: token j), into
// this lane's column of the warp's score slots sc[j][lane]; lane j holds token
// j's metadata word mw
template <int R>
__device__ __forceinline__ void scores_of_class(uint32_t m, uint32_t mw, const uint8_t* kb, int h,
                                                const float* q, const float (&pre)[5], float* sc,
                                                int lane) {
  while (m) {
    const int j = __ffs(m) - 1;
    m &= m - 1;
    const uint32_t w = __shfl_sync(0xffffffffu, mw, j);
    sc[j * 32 + lane] = score_r<R>(kb + (w & 0xFFFu) + h * head_bytes(R), q, pre);
  }
}

// the value updates of the chunk's tokens of value rank R, with the weights p
// in the score slots
template <int R>
__device__ __forceinline__ void values_of_class(uint32_t m, uint32_t mw, const uint8_t* vb, int h,
                                                const float* sc, int lane,
                                                uint64_t (&acc)[kVRmax / 2], float (&zc)[6]) {
  while (m) {
    const int j = __ffs(m) - 1;
    m &= m - 1;
    const uint32_t w = __shfl_sync(0xffffffffu, mw, j);
    value_r<R>(vb + ((w >> 12) & 0xFFFu) + h * head_bytes(R), sc[j * 32 + lane], acc, zc);
  }
}

__device__ __forceinline__ bool rank_in_set(int r) {
  return r == 4 || r == 8 || r == 16 || r == 32 || r == 64;
}

__global__ void __launch_bounds__(kVThreads, 1) varrate_warp_kernel(Params p, int split_len) {
  // the combine may launch now: its blocks take SMs as this grid's CTAs exit and
  // wait (griddepcontrol.wait) for the whole grid before reading the partials
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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

  // ---- chunk staging: the byte ranges [off[t0], off[t0 + n]) of both streams,
  // from the 16-byte boundary below, clamped to the stream and the buffer.
  // A chunk's metadata (lane j <= n: offsets, lane j < n: ranks of token
  // t0 + j) is loaded one chunk before its copies are issued, so the copies of
  // chunk c + 1 never wait for memory; lane j < n then keeps token t0 + j's
  // offsets (relative to the staged areas) and ranks, and the chunk's validity
  // mask is formed once, at issue
  struct Raw {
    int ok, ov, rkv;
  };
  struct Meta {
    // lane j < n: token t0 + j's K and V record offsets in the staged areas
    // (bits 0-11, 12-23), rank classes (log2 r - 2; bits 24-26, 27-29) and
    // bit 30 set when its records lie in the staged areas; one shuffle per token
    uint32_t w;
    int n;                              // tokens in the chunk (the same in every lane)
  };
  auto meta_load = [&](int t0) -> Raw {
    const int n = min(kVChunk, t_b - t0);   // at most; the chunk may end sooner
    Raw r;
    r.ok = lane <= n ? __ldg(offk + t0 + lane) : 0;
    r.ov = lane <= n ? __ldg(offv + t0 + lane) : 0;
    r.rkv = lane < n ? (int)__ldg(rk + t0 + lane) | ((int)__ldg(rv + t0 + lane) << 8) : 0;
    return r;
  };
  auto stage = [&](const Raw& r, int t0, int buf) -> Meta {
    const int nmax = min(kVChunk, t_b - t0);
    Meta mt;
    const int k0 = __shfl_sync(0xffffffffu, r.ok, 0), v0 = __shfl_sync(0xffffffffu, r.ov, 0);
    const int base_k = k0 & ~15, base_v = v0 & ~15;
    // the chunk: the longest run of tokens (at most nmax, at least one) whose
    // K and V records both fit a buffer; lane j holds the end of token j - 1
    const bool over = lane >= 1 && lane <= nmax &&
                      (r.ok - base_k > kVBuf || r.ov - base_v > kVBuf || r.ok < k0 || r.ov < v0);
    const uint32_t ov_mask = __ballot_sync(0xffffffffu, over);
    const int n = ov_mask ? max(__ffs(ov_mask) - 2, 1) : nmax;
    mt.n = n;
    const int k1 = __shfl_sync(0xffffffffu, r.ok, n), v1 = __shfl_sync(0xffffffffu, r.ov, n);
    const uint32_t dk = area_s + (2 * buf) * kVBuf, dv = area_s + (2 * buf + 1) * kVBuf;
    const long long ek = min((long long)k1, sbytes), ev = min((long long)v1, sbytes);
    const int nk = (int)min((ek - base_k + 15) / 16, (long long)(kVBuf / 16));
    const int nv = (int)min((ev - base_v + 15) / 16, (long long)(kVBuf / 16));
    for (int c = lane; c < nk; c += 32) cp16(dk + 16 * c, kstream + base_k + 16 * c);
    for (int c = lane; c < nv; c += 32) cp16(dv + 16 * c, vstream + base_v + 16 * c);
    // records outside the staged areas or off their 16-byte grid (offsets
    // inconsistent with the ranks), or ranks outside the set, are skipped
    const int ok = r.ok - base_k, ov = r.ov - base_v;
    const int r_k = r.rkv & 255, r_v = r.rkv >> 8;
    const bool good = lane < n && rank_in_set(r_k) && rank_in_set(r_v) && ok >= 0 &&
                      !(ok & 15) && ok + kVHkv * head_bytes(r_k) <= 16 * nk &&
                      ov >= 0 && !(ov & 15) && ov + kVHkv * head_bytes(r_v) <= 16 * nv;
    mt.w = good ? (uint32_t)ok | ((uint32_t)ov << 12) | ((uint32_t)(__ffs(r_k) - 3) << 24) |
                      ((uint32_t)(__ffs(r_v) - 3) << 27) | (1u << 30)
                : 0u;
    return mt;
  };

  Meta cur{0u, 0}, nxt{0u, 0};
  Raw raw0{}, raw1{};                   // metadata of the current and of the next chunk
  int t0 = t_a, buf = 0;
  if (t0 < t_b) raw0 = meta_load(t0);   // in flight during the query projection

  // ---- q~ = Bk q for the row's 32 query heads (softmax scale and log2 e
  // folded in), on warp-level MMAs.  Bk (8 heads x 64 rows x 128, fp16) is first
  // copied into the staging area with coalesced 16-byte copies, row r's 16-byte
  // piece c at r * 256 + (c ^ (r & 15)) * 16 (conflict-free ldmatrix rows).  The
  // queries are scaled by a power of two, 2^-e, so that the largest lies below
  // 2^14, and rounded to f16: exact for bf16 values down to the f16
  // subnormals, whose spacing is 2^-38 of the largest.  Warp w forms rows
  // 32 (w % 2) .. + 31 of head w / 2: M = 16 rows, N = the head's 4 queries (of
  // 8), K = 16 dims; products exact, sums fp32, scaled back by 2^e.
  float* const qsm = reinterpret_cast<float*>(vsm + kVOffQ);
  {
    const uint32_t bks = smem_u32(vsm);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int idx = c * kVThreads + threadIdx.x, r = idx >> 4, pc = idx & 15;
      cp16(bks + r * 256 + ((pc ^ (r & 15)) << 4), p.bk + (size_t)idx * 8);
    }
    cp_commit();
    __half* const qh = reinterpret_cast<__half*>(vsm + kVOffX);             // [32][kVQhRow]
    float* const red = reinterpret_cast<float*>(vsm + kVOffX + 32 * kVQhRow * 2);
    // the row's 32 x 128 bf16 queries, 8 per thread (one 16-byte load)
    const uint4 xq = __ldg(reinterpret_cast<const uint4*>(p.q + (size_t)b * p.Hq * 128) +
                           threadIdx.x);
    const uint32_t xw[4] = {xq.x, xq.y, xq.z, xq.w};
    float v[8], mx = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[2 * k] = __uint_as_float(xw[k] << 16);
      v[2 * k + 1] = __uint_as_float(xw[k] & 0xFFFF0000u);
      mx = fmaxf(mx, fmaxf(fabsf(v[2 * k]), fabsf(v[2 * k + 1])));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    mx = 0.f;
#pragma unroll
    for (int k = 0; k < kVWarps; ++k) mx = fmaxf(mx, red[k]);
    int ex = 0;
    if (mx > 0.f && mx <= 3.0e38f) {
      frexpf(mx, &ex);                  // mx < 2^ex
      ex = ex > 14 ? ex - 14 : 0;
    }
    const float down = ldexpf(1.f, -ex), up = ldexpf(1.f, ex) * p.scale_log2;
    {
      uint32_t hw[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __half2 h2 = __floats2half2_rn(v[2 * k] * down, v[2 * k + 1] * down);
        hw[k] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      *reinterpret_cast<uint4*>(qh + (threadIdx.x >> 4) * kVQhRow + 8 * (threadIdx.x & 15)) =
          make_uint4(hw[0], hw[1], hw[2], hw[3]);
    }
    cp_wait<0>();
    __syncthreads();
    const int kvh = warp >> 1, n = lane >> 2, kq = 2 * (lane & 3);
    uint32_t bf[8][2];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const __half* qr = qh + (kvh * kVG + (n & 3)) * kVQhRow + 16 * ks + kq;
      bf[ks][0] = n < kVG ? *reinterpret_cast<const uint32_t*>(qr) : 0u;
      bf[ks][1] = n < kVG ? *reinterpret_cast<const uint32_t*>(qr + 8) : 0u;
    }
    const int lrow = (lane & 7) + 8 * ((lane >> 3) & 1), lpc = lane >> 4;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      const int j0 = 32 * (warp & 1) + 16 * mt;          // first row of the tile in the head
      const int r = kvh * kVRmax + j0 + lrow;             // this lane's ldmatrix row
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t a[4];
        ldmatrix_x4(a, vsm + r * 256 + (((2 * ks + lpc) ^ (r & 15)) << 4));
        mma16816(c, a, bf[ks][0], bf[ks][1]);
      }
      if (kq < kVG) {                   // C: rows lane / 4 (+ 8), queries kq, kq + 1
        const int jr = j0 + (lane >> 2);
        qsm[(kvh * kVG + kq) * kVQRow + jr] = c[0] * up;
        qsm[(kvh * kVG + kq + 1) * kVQRow + jr] = c[1] * up;
        qsm[(kvh * kVG + kq) * kVQRow + jr + 8] = c[2] * up;
        qsm[(kvh * kVG + kq + 1) * kVQRow + jr + 8] = c[3] * up;
      }
    }
    __syncthreads();                    // Bk's copy in the staging area is dead from here
  }
  if (t0 < t_b) {
    cur = stage(raw0, t0, 0);
    if (t0 + cur.n < t_b) raw1 = meta_load(t0 + cur.n);
  }
  cp_commit();
  const float* const q = qsm + lane * kVQRow;       // lane = h * 4 + qi
  // this warp's score slots [kVChunk][32]
  float* const sc = reinterpret_cast<float*>(vsm + kVOffS) + warp * (kVChunk * 32);
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
  uint64_t acc[kVRmax / 2];
#pragma unroll
  for (int i = 0; i < kVRmax / 2; ++i) acc[i] = 0ull;
  float zc[6] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float m = -INFINITY, m_thr = -INFINITY, l = 0.f;

  while (t0 < t_b) {
    const int t1 = t0 + cur.n;
    Raw raw2{};
    if (t1 < t_b) {
      nxt = stage(raw1, t1, buf ^ 1);
      if (t1 + nxt.n < t_b) raw2 = meta_load(t1 + nxt.n);
    }
    cp_commit();
    cp_wait<1>();
    __syncwarp();
    const uint8_t* kb = area + (2 * buf) * kVBuf;
    const uint8_t* vb = area + (2 * buf + 1) * kVBuf;
    // the chunk by rank class: the scores of all its tokens (one loop per key
    // rank class), one maximum update and the weights of all of them, then the
    // value updates (one loop per value rank class); lanes >= n hold word 0
    {
      const uint32_t mw = cur.w;
      const bool live = (mw >> 30) != 0;
      const uint32_t ck = (mw >> 24) & 7u;
      const uint32_t valid = __ballot_sync(0xffffffffu, live);
      scores_of_class<4>(__ballot_sync(0xffffffffu, live && ck == 0u), mw, kb, h, q, pre, sc, lane);
      scores_of_class<8>(__ballot_sync(0xffffffffu, live && ck == 1u), mw, kb, h, q, pre, sc, lane);
      scores_of_class<16>(__ballot_sync(0xffffffffu, live && ck == 2u), mw, kb, h, q, pre, sc, lane);
      scores_of_class<32>(__ballot_sync(0xffffffffu, live && ck == 3u), mw, kb, h, q, pre, sc, lane);
      scores_of_class<64>(__ballot_sync(0xffffffffu, live && ck == 4u), mw, kb, h, q, pre, sc, lane);
      float smax = -INFINITY;
#pragma unroll
      for (int j = 0; j < kVChunk; ++j)
        if ((valid >> j) & 1u) smax = fmaxf(smax, sc[j * 32 + lane]);
      if (smax > m_thr) {               // lazily raised maximum (by more than 2^8)
        const float a = ex2_approx(m - smax);
        l *= a;
        const uint64_t a2 = pkf(a, a);
#pragma unroll
        for (int i = 0; i < kVRmax / 2; ++i) acc[i] = mul2(acc[i], a2);
#pragma unroll
        for (int i = 0; i < 6; ++i) zc[i] *= a;
        m = smax;
        m_thr = smax + 8.f;
      }
#pragma unroll
      for (int j = 0; j < kVChunk; ++j) {
        if ((valid >> j) & 1u) {
          const float pr = ex2_approx(sc[j * 32 + lane] - m);
          l += pr;
          sc[j * 32 + lane] = pr;
        }
      }
      const uint32_t cv = (mw >> 27) & 7u;
      values_of_class<4>(__ballot_sync(0xffffffffu, live && cv == 0u), mw, vb, h, sc, lane, acc, zc);
      values_of_class<8>(__ballot_sync(0xffffffffu, live && cv == 1u), mw, vb, h, sc, lane, acc, zc);
      values_of_class<16>(__ballot_sync(0xffffffffu, live && cv == 2u), mw, vb, h, sc, lane, acc, zc);
      values_of_class<32>(__ballot_sync(0xffffffffu, live && cv == 3u), mw, vb, h, sc, lane, acc, zc);
      values_of_class<64>(__ballot_sync(0xffffffffu, live && cv == 4u), mw, vb, h, sc, lane, acc, zc);
    }
    __syncwarp();                       // this buffer is refilled by the next stage
    cur = nxt;
    raw1 = raw2;
    t0 = t1;
    buf ^= 1;
  }
  cp_wait<0>();
  __syncthreads();

  // ---- merge the warps of this CTA, one partial per row; the class sums of
  // the zero terms join the accumulator first (class of rank R covers i < R)
  float* mg = reinterpret_cast<float*>(vsm);
  {
    float* slot = mg + (warp * 32 + lane) * kVPst;
    const float z3 = zc[3] + zc[4];     // 16 <= i < 32: ranks 32, 64
    const float z2 = zc[2] + z3;        // 8 <= i < 16: and 16
    const float z1 = zc[1] + z2;        // 4 <= i < 8: and 8
    const float z0 = zc[0] + z1;        // i < 4: and 4
#pragma unroll
    for (int i = 0; i < kVRmax / 2; ++i) {
      const float2 v = upk(acc[i]);
      const int e = 2 * i;
      const float z = e < 4 ? z0 : e < 8 ? z1 : e < 16 ? z2 : e < 32 ? z3 : zc[5];
      slot[e] = v.x + z;
      slot[e + 1] = v.y + z;
    }
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
