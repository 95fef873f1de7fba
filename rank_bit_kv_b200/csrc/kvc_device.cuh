// Device helpers shared by the kernels of libkvc.
#pragma once

#include "kvc_internal.h"

namespace kvc {

__device__ __forceinline__ float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float h2f(__half x) { return __half2float(x); }

// Tokens attended by batch row b: seq_lens[b] clamped to [0, n_tokens].
__device__ __forceinline__ int row_len(const Params& p, int b) {
  int n = p.n_tokens;
  if (p.seq_lens) {
    int s = p.seq_lens[b];
    n = s < 0 ? 0 : (s < n ? s : n);
  }
  return n;
}

// Physical page of token t of batch row b, clamped to the pool so that a bad
// page-table entry never sends a read outside the cache.
__device__ __forceinline__ int page_of(const Params& p, int b, int t) {
  const int pp = p.page_table[(int64_t)b * (p.tmax / p.page) + t / p.page];
  return min(max(pp, 0), p.n_pages - 1);
}

// Row index of (batch row b, KV head h, token t) in a low-rank component.
__device__ __forceinline__ int64_t lowrank_row(const Params& p, int b, int h, int t) {
  if (p.page) return ((int64_t)page_of(p, b, t) * p.Hkv + h) * p.page + (t % p.page);
  return ((int64_t)b * p.Hkv + h) * p.tmax + t;
}

// INT4 element r of a row: element 2i in the low nibble of byte i.
__device__ __forceinline__ int int4_at(const uint8_t* row, int r) {
  const int byte = row[r >> 1];
  return (r & 1) ? (byte >> 4) : (byte & 15);
}

// Signed level of the symmetric code of width `bits` at element i of a row:
// element i occupies bits [bits * i, bits * i + bits) of the row's
// little-endian bit stream; level = code - 2^(bits - 1).
__device__ __forceinline__ int sym_level_at(const uint8_t* row, int i, int bits) {
  const int o = i * bits, byte = o >> 3, sh = o & 7;
  int v = row[byte] >> sh;
  if (sh + bits > 8) v |= row[byte + 1] << (8 - sh);
  return (v & ((1 << bits) - 1)) - (1 << (bits - 1));
}

// 2-bit element i of a row: element 4j+k in bits 2k..2k+1 of byte j.
__device__ __forceinline__ int int2_at(const uint8_t* row, int i) {
  return (row[i >> 2] >> (2 * (i & 3))) & 3;
}

// Bytes of one VARRATE record per KV head at rank r.
__device__ __forceinline__ int varrate_head_bytes(int r) { return r / 2 + 4 * ((r + 31) / 32); }

// In-place unnormalised Walsh-Hadamard transform (Sylvester order) of n
// values in shared memory, computed by nthreads cooperating threads.
// Butterflies (a, b) -> (a + b, a - b) over blocks of doubling size give H x.
__device__ __forceinline__ void fwht_smem(float* x, int n, int tid, int nthreads) {
  for (int len = 1; len < n; len <<= 1) {
    __syncthreads();
    for (int k = tid; k < n / 2; k += nthreads) {
      const int blk = k / len, off = k % len;
      const int i = blk * 2 * len + off, j = i + len;
      const float a = x[i], b = x[j];
      x[i] = a + b;
      x[j] = a - b;
    }
  }
  __syncthreads();
}

// Unnormalised Walsh-Hadamard transform (Sylvester order) of 128 values held
// by one warp, lane l holding x[k] = v[4 l + k]: butterflies (a, b) ->
// (a + b, a - b) over blocks of doubling size, the first two inside a lane and
// the rest between lanes l and l ^ m (the lower index keeps a + b).
__device__ __forceinline__ void fwht128_warp(float (&x)[4], int lane) {
  float a = x[0] + x[1], b = x[0] - x[1], c = x[2] + x[3], e = x[2] - x[3];
  x[0] = a + c;
  x[1] = b + e;
  x[2] = a - c;
  x[3] = b - e;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool hi = lane & m;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float o = __shfl_xor_sync(0xffffffffu, x[k], m);
      x[k] = hi ? o - x[k] : x[k] + o;
    }
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace kvc
