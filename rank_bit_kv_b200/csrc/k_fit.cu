// Per-KV-head factor fit by randomized SVD, for bulk prefill compression.
//
// "A JoLT for the KV cache ...", "Abstract (arXiv)": FlashJoLT replaces the
// exact token-mode SVD with a randomized approximation; "JoLT: Near-Lossless
// KV Cache Compression", "How JoLT works" / "Key findings": only the token and
// feature axes are truncated (per-head factors), on keys before RoPE.  The
// factor B of a head (r x d) is the top-r right singular subspace of its
// token-major matrix X (all batch rows' prefill tokens, N x d); a token's
// latent is then x B^T (kvc_append).
//
// The randomized range finder needs X only through products with d x k
// matrices, so one streaming pass forms the Gram matrix G = X^T X (d x d) and
// everything after it is small dense algebra on G (exact in exact arithmetic):
//   W = Omega;  repeat q times: W = orth(G W)       (span of X W = the power
//                                                    iterations' span of Q)
//   P = G W;  W^T P = R^T R (Cholesky);  T = P R^-1  (T = B_s^T for B_s = Q^T X,
//                                                    Q = X W R^-1)
//   T^T T = U L U^T (Jacobi);  V = T U L^-1/2        (B_s = U S V^T)
// and the factor rows are the columns of V with the r largest L.
//
// Kernels: the Gram matrix on tensor cores (bf16 in, fp32 accumulate), one
// partial per CTA; a fixed-order fp64 reduction (deterministic); one CTA per
// head for the small stage in fp64.
#include <math.h>

#include "kvc_device.cuh"
#include "tc_util.cuh"

namespace kvc {
namespace {

using namespace tc;

constexpr int kFD = 128;              // head dim
constexpr int kFRows = 128;           // token rows per staged tile
constexpr int kFRowB = 272;           // shared bytes per staged row (256 + 16 pad: no bank conflicts)
constexpr int kFThreads = 256;        // 8 warps: warp w forms rows 16w .. 16w + 15 of G
constexpr int kFTile = kFRows * kFRowB;
constexpr int kSThreads = 256;        // small-stage threads

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
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

// G partial of CTA (chunk, head): sum over the head's 128-row tiles chunk,
// chunk + n_chunks, ... of X_tile^T X_tile.  Rows past n_rows are zero-filled.
__global__ void __launch_bounds__(kFThreads) gram_kernel(const __nv_bfloat16* __restrict__ x,
                                                         int B, int Hkv, int cap, int n_rows,
                                                         int n_chunks, float* __restrict__ part) {
  extern __shared__ __align__(16) uint8_t gsm[];
  const int chunk = blockIdx.x, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tpr = (n_rows + kFRows - 1) / kFRows;       // tiles per batch row
  const int total = B * tpr;
  const uint32_t sm_s = smem_u32(gsm);
  auto issue = [&](int tile, int buf) {
    if (tile < total) {
      const int b = tile / tpr, t0 = (tile % tpr) * kFRows;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = threadIdx.x + kFThreads * i;       // 16-byte chunk 0..2047
        const int r = c >> 4, col = c & 15;
        const int t = t0 + r;
        const bool valid = t < n_rows;
        const __nv_bfloat16* src =
            x + (((size_t)b * Hkv + h) * cap + (valid ? t : 0)) * kFD + col * 8;
        const uint32_t dst = sm_s + buf * kFTile + r * kFRowB + col * 16;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                     "r"(valid ? 16 : 0)
                     : "memory");
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  float acc[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  // ldmatrix row addresses: lane -> (matrix lane / 8, row lane % 8)
  const int mi = lane >> 3, rr = lane & 7;
  const int a_row = rr + 8 * (mi >> 1), a_col = 16 * warp + 8 * (mi & 1);   // A = X^T
  const int b_row = rr + 8 * (mi & 1), b_col = 8 * (mi >> 1);               // B = X
  issue(chunk, 0);
  int it = 0;
  for (int tile = chunk; tile < total; tile += n_chunks, ++it) {
    issue(tile + n_chunks, (it + 1) & 1);
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncthreads();
    const uint32_t X = sm_s + (it & 1) * kFTile;
#pragma unroll 1
    for (int ks = 0; ks < kFRows / 16; ++ks) {
      uint32_t a[4];
      ldsm_x4_trans(a, X + (16 * ks + a_row) * kFRowB + a_col * 2);
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        uint32_t b[4];
        ldsm_x4_trans(b, X + (16 * ks + b_row) * kFRowB + (16 * np + b_col) * 2);
        mma_bf16(acc[2 * np], a, b[0], b[1]);
        mma_bf16(acc[2 * np + 1], a, b[2], b[3]);
      }
    }
    __syncthreads();                  // the buffer is refilled by the next issue
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  const int g = lane >> 2, c4 = lane & 3;
  float* dst = part + ((size_t)h * n_chunks + chunk) * kFD * kFD;
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    const int i = 16 * warp + g, j = 8 * nt + 2 * c4;
    dst[i * kFD + j] = acc[nt][0];
    dst[i * kFD + j + 1] = acc[nt][1];
    dst[(i + 8) * kFD + j] = acc[nt][2];
    dst[(i + 8) * kFD + j + 1] = acc[nt][3];
  }
}

// G = sum of the partials of a head, in chunk order, in fp64, symmetrised
// (the tensor-core partials accumulate the two triangles in different orders):
// G_ij = (S_ij + S_ji) / 2.  Grid (entry blocks, heads), one entry per thread.
__global__ void gram_reduce_kernel(const float* __restrict__ part, int n_chunks,
                                   double* __restrict__ G) {
  const int h = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= kFD * kFD) return;
  const int i = e / kFD, j = e % kFD;
  const float* src = part + (size_t)h * n_chunks * kFD * kFD;
  double a = 0.0, b = 0.0;
#pragma unroll 16
  for (int c = 0; c < n_chunks; ++c) {
    a += (double)src[(size_t)c * kFD * kFD + e];
    b += (double)src[(size_t)c * kFD * kFD + j * kFD + i];
  }
  G[(size_t)h * kFD * kFD + e] = 0.5 * (a + b);
}

struct SmallWs {          // per-head fp64 scratch in global memory
  double* W;              // d x k (column-major: W[col * d + row])
  double* P;              // d x k
  double* V;              // d x k
};

// Y[:, j] = G X[:, j] for all columns (column-major d x k).  Thread (row,
// block of 8 columns) reads G[l][row] (= G[row][l], G is symmetric; the lanes
// of a warp take consecutive rows, so the loads are coalesced) once for its 8
// accumulators; the X entries are the same for the whole warp (broadcast).
__device__ void gemm_G(const double* __restrict__ G, const double* X, double* Y, int k) {
  constexpr int CB = 8;
  const int nblk = (k + CB - 1) / CB;
  for (int e = threadIdx.x; e < kFD * nblk; e += blockDim.x) {
    const int row = e % kFD, c0 = (e / kFD) * CB;
    double acc[CB];
#pragma unroll
    for (int j = 0; j < CB; ++j) acc[j] = 0.0;
#pragma unroll 4
    for (int l = 0; l < kFD; ++l) {
      const double gv = G[(size_t)l * kFD + row];
#pragma unroll
      for (int j = 0; j < CB; ++j)
        if (c0 + j < k) acc[j] = fma(gv, X[(size_t)(c0 + j) * kFD + l], acc[j]);
    }
#pragma unroll
    for (int j = 0; j < CB; ++j)
      if (c0 + j < k) Y[(size_t)(c0 + j) * kFD + row] = acc[j];
  }
  __syncthreads();
}

// C = A^T B for column-major d x k matrices A, B (k x k, row-major), in 4 x 4
// blocks per thread; lane-rotated summation start keeps the column reads of a
// warp on different banks.
__device__ void gram_small(const double* A, const double* Bm, double* C, int k) {
  const int nb = (k + 3) / 4;
  const int lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < nb * nb; e += blockDim.x) {
    const int i0 = 4 * (e / nb), j0 = 4 * (e % nb);
    // columns past k read column k - 1 (in range) and are not stored
    int ia[4], jb[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      ia[a] = min(i0 + a, k - 1);
      jb[a] = min(j0 + a, k - 1);
    }
    double acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
#pragma unroll 2
    for (int l0 = 0; l0 < kFD; ++l0) {
      const int l = (l0 + lane) & (kFD - 1);
      double x[4], y[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) x[a] = A[(size_t)ia[a] * kFD + l];
#pragma unroll
      for (int b = 0; b < 4; ++b) y[b] = Bm[(size_t)jb[b] * kFD + l];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fma(x[a], y[b], acc[a][b]);
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b)
        if (i0 + a < k && j0 + b < k) C[(i0 + a) * k + j0 + b] = acc[a][b];
  }
}

// Orthonormalise the k columns of W (d x k) by classical Gram-Schmidt applied
// twice per column; red = shared scratch of at least d + 1 doubles.  The dot
// products of a pass are spread over the warps (lanes split the d entries).
__device__ void orthonormalise(double* W, int k, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int j = 0; j < k; ++j) {
    double* wj = W + (size_t)j * kFD;
    for (int pass = 0; pass < 2; ++pass) {
      for (int l = warp; l < j; l += nw) {
        const double* wl = W + (size_t)l * kFD;
        double s = 0.0;
        for (int i = lane; i < kFD; i += 32) s += wl[i] * wj[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) red[l] = s;
      }
      __syncthreads();
      for (int i = threadIdx.x; i < kFD; i += blockDim.x) {
        double v = wj[i];
        for (int l = 0; l < j; ++l) v -= red[l] * W[(size_t)l * kFD + i];
        wj[i] = v;
      }
      __syncthreads();
    }
    if (warp == 0) {
      double s = 0.0;
      for (int i = lane; i < kFD; i += 32) s += wj[i] * wj[i];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) red[kFD] = s > 0.0 ? 1.0 / sqrt(s) : 0.0;
    }
    __syncthreads();
    const double inv = red[kFD];
    for (int i = threadIdx.x; i < kFD; i += blockDim.x) wj[i] *= inv;
    __syncthreads();
  }
}

// shared bytes of the small stage without / with W and P
__host__ __device__ size_t small_smem_base(int k) {
  return (size_t)(2 * k * k + kFD + 1 + k) * sizeof(double) + (size_t)2 * k * sizeof(int) + 64;
}
size_t small_smem_wp(int k) {
  return ((small_smem_base(k) + 15) & ~(size_t)15) + (size_t)2 * kFD * k * sizeof(double);
}

// One CTA per head: the small stage in fp64 (see the file comment).
// Shared: C (k x k), U (k x k), scratch.  k <= kFitMaxK, even.
__global__ void __launch_bounds__(kSThreads) rsvd_small_kernel(
    const double* __restrict__ Gall, const float* __restrict__ omega, int k, int rank,
    int power_iters, SmallWs ws_base, __half* __restrict__ factor, float* __restrict__ sigma2,
    int wp_in_smem) {
  extern __shared__ __align__(16) double ssm[];
  const int h = blockIdx.x;
  const int tid = threadIdx.x, nth = blockDim.x;
  const double* G = Gall + (size_t)h * kFD * kFD;
  const size_t dk = (size_t)kFD * kFitMaxK;
  double* C = ssm;                          // k x k, row-major
  double* U = C + k * k;                    // k x k
  double* red = U + k * k;                  // kFD + 1 + 2k scratch
  double* cs = red + kFD + 1;               // rotation cosines / sines of a round
  double* sn = cs + k / 2;
  int* order = reinterpret_cast<int*>(sn + k / 2);   // k ints
  int* pa = order + k;                      // the pairs of a Jacobi round (k / 2 each)
  int* pb = pa + k / 2;
  // W and P (d x k) live in shared memory when the launch gave room for them
  // (the Gram-Schmidt passes re-read them column by column), else in global
  double* const sm_wp = reinterpret_cast<double*>(
      reinterpret_cast<char*>(ssm) + ((small_smem_base(k) + 15) & ~(size_t)15));
  double* W = wp_in_smem ? sm_wp : ws_base.W + h * dk;
  double* P = wp_in_smem ? sm_wp + (size_t)kFD * k : ws_base.P + h * dk;
  double* V = ws_base.V + h * dk;

  // W = Omega (column-major), power iterations
  for (int e = tid; e < kFD * k; e += nth) {
    const int row = e % kFD, col = e / kFD;
    W[(size_t)col * kFD + row] = (double)omega[((size_t)h * kFD + row) * k + col];
  }
  __syncthreads();
  orthonormalise(W, k, red);
  for (int it = 0; it < power_iters; ++it) {
    gemm_G(G, W, P, k);
    for (int e = tid; e < kFD * k; e += nth) W[e] = P[e];
    __syncthreads();
    orthonormalise(W, k, red);
  }
  // P = G W; C = W^T P (k x k)
  gemm_G(G, W, P, k);
  gram_small(W, P, C, k);
  __syncthreads();
  // Cholesky C = R^T R in place (upper triangle holds R); a pivot that has
  // vanished (rank-deficient sketch) makes its column of R and of T zero
  double trace = 0.0;
  for (int i = 0; i < k; ++i) trace += C[i * k + i];
  for (int j = 0; j < k; ++j) {
    if (tid == 0) {
      double s = C[j * k + j];
      for (int l = 0; l < j; ++l) s -= C[l * k + j] * C[l * k + j];
      C[j * k + j] = s > 1e-26 * trace ? sqrt(s) : 0.0;
    }
    __syncthreads();
    const double rjj = C[j * k + j];
    for (int i = j + 1 + tid; i < k; i += nth) {
      double s = C[j * k + i];
      for (int l = 0; l < j; ++l) s -= C[l * k + j] * C[l * k + i];
      C[j * k + i] = rjj > 0.0 ? s / rjj : 0.0;
    }
    __syncthreads();
  }
  // T = P R^-1, column by column, in place in P
  for (int j = 0; j < k; ++j) {
    const double rjj = C[j * k + j];
    for (int i = tid; i < kFD; i += nth) {
      double v = P[(size_t)j * kFD + i];
      for (int l = 0; l < j; ++l) v -= P[(size_t)l * kFD + i] * C[l * k + j];
      P[(size_t)j * kFD + i] = rjj > 0.0 ? v / rjj : 0.0;
    }
    __syncthreads();
  }
  // C = T^T T; U = I
  gram_small(P, P, C, k);
  for (int e = tid; e < k * k; e += nth) U[e] = (e / k == e % k) ? 1.0 : 0.0;
  __syncthreads();
  // cyclic Jacobi, round-robin pairing (k even): every round rotates k / 2
  // disjoint pairs; at most kFitSweeps sweeps (quadratic convergence), fewer
  // once the off-diagonal mass is negligible against the diagonal
  const int half = k / 2;
  for (int sweep = 0; sweep < kFitSweeps; ++sweep) {
    {
      double off = 0.0, dia = 0.0;
      for (int e = tid; e < k * k; e += nth) {
        const double v = C[e] * C[e];
        if (e / k == e % k) dia += v;
        else off += v;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        off += __shfl_xor_sync(0xffffffffu, off, o);
        dia += __shfl_xor_sync(0xffffffffu, dia, o);
      }
      if ((tid & 31) == 0) {
        red[2 * (tid >> 5)] = off;
        red[2 * (tid >> 5) + 1] = dia;
      }
      __syncthreads();
      double offs = 0.0, dias = 0.0;
      for (int w = 0; w < nth / 32; ++w) {
        offs += red[2 * w];
        dias += red[2 * w + 1];
      }
      __syncthreads();
      if (offs <= 1e-30 * dias) break;
    }
    for (int round = 0; round < k - 1; ++round) {
      auto member = [&](int pos) { return pos == 0 ? 0 : 1 + (pos - 1 + round) % (k - 1); };
      for (int q = tid; q < half; q += nth) {
        const int a = member(q), b = member(k - 1 - q);
        const double app = C[a * k + a], aqq = C[b * k + b], apq = C[a * k + b];
        double c = 1.0, s = 0.0;
        if (fabs(apq) > 1e-300) {
          const double th = (aqq - app) / (2.0 * apq);
          const double t = (th >= 0.0 ? 1.0 : -1.0) / (fabs(th) + sqrt(th * th + 1.0));
          c = 1.0 / sqrt(t * t + 1.0);
          s = t * c;
        }
        cs[q] = c;
        sn[q] = s;
        pa[q] = a;
        pb[q] = b;
      }
      __syncthreads();
      // columns: C <- C J, U <- U J
      for (int e = tid; e < k * half; e += nth) {
        const int i = e / half, q = e % half;
        const int a = pa[q], b = pb[q];
        const double c = cs[q], s = sn[q];
        const double x = C[i * k + a], y = C[i * k + b];
        C[i * k + a] = c * x - s * y;
        C[i * k + b] = s * x + c * y;
        const double u = U[i * k + a], v = U[i * k + b];
        U[i * k + a] = c * u - s * v;
        U[i * k + b] = s * u + c * v;
      }
      __syncthreads();
      // rows: C <- J^T C
      for (int e = tid; e < k * half; e += nth) {
        const int j = e / half, q = e % half;
        const int a = pa[q], b = pb[q];
        const double c = cs[q], s = sn[q];
        const double x = C[a * k + j], y = C[b * k + j];
        C[a * k + j] = c * x - s * y;
        C[b * k + j] = s * x + c * y;
      }
      __syncthreads();
    }
  }
  // order of the eigenvalues, largest first (ties: lower index first)
  for (int i = tid; i < k; i += nth) {
    const double li = C[i * k + i];
    int pos = 0;
    for (int j = 0; j < k; ++j) {
      const double lj = C[j * k + j];
      pos += (lj > li) || (lj == li && j < i);
    }
    order[pos] = i;
  }
  __syncthreads();
  if (sigma2)
    for (int p = tid; p < k; p += nth) sigma2[(size_t)h * k + p] = (float)fmax(C[order[p] * k + order[p]], 0.0);
  // V[:, p] = T U[:, order[p]] / sqrt(L) for the first rank columns
  for (int e = tid; e < kFD * rank; e += nth) {
    const int i = e % kFD, p = e / kFD;
    const int m = order[p];
    const double lam = C[m * k + m];
    double s = 0.0;
    for (int l = 0; l < k; ++l) s += P[(size_t)l * kFD + i] * U[l * k + m];
    V[(size_t)p * kFD + i] = lam > 0.0 ? s / sqrt(lam) : 0.0;
  }
  __syncthreads();
  // factor rows, each with its largest-magnitude entry positive, as fp16
  for (int p = tid; p < rank; p += nth) {
    const double* v = V + (size_t)p * kFD;
    int arg = 0;
    for (int i = 1; i < kFD; ++i)
      if (fabs(v[i]) > fabs(v[arg])) arg = i;
    red[p] = v[arg] < 0.0 ? -1.0 : 1.0;
  }
  __syncthreads();
  for (int e = tid; e < kFD * rank; e += nth) {
    const int i = e % kFD, p = e / kFD;
    factor[((size_t)h * rank + p) * kFD + i] = __double2half(red[p] * V[(size_t)p * kFD + i]);
  }
}


}  // namespace

size_t fit_workspace_bytes(int n_kv_heads) {
  const size_t part = (size_t)n_kv_heads * kFitChunks * kFD * kFD * sizeof(float);
  const size_t G = (size_t)n_kv_heads * kFD * kFD * sizeof(double);
  const size_t small = 3 * (size_t)n_kv_heads * kFD * kFitMaxK * sizeof(double);
  return part + G + small + 3 * 256;
}

cudaError_t launch_fit(const FitParams& f, cudaStream_t s) {
  char* ws = (char*)f.workspace;
  float* part = (float*)ws;
  size_t off = (size_t)f.Hkv * kFitChunks * kFD * kFD * sizeof(float);
  off = (off + 255) / 256 * 256;
  double* G = (double*)(ws + off);
  off += (size_t)f.Hkv * kFD * kFD * sizeof(double);
  off = (off + 255) / 256 * 256;
  SmallWs sw;
  const size_t dk = (size_t)f.Hkv * kFD * kFitMaxK;
  sw.W = (double*)(ws + off);
  sw.P = sw.W + dk;
  sw.V = sw.P + dk;
  const int gsm = 2 * kFTile;
  cudaError_t e = cudaFuncSetAttribute(gram_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, gsm);
  if (e != cudaSuccess) return e;
  gram_kernel<<<dim3(kFitChunks, f.Hkv), kFThreads, gsm, s>>>(f.x, f.B, f.Hkv, f.cap, f.n_rows,
                                                              kFitChunks, part);
  gram_reduce_kernel<<<dim3(kFD * kFD / 256, f.Hkv), 256, 0, s>>>(part, kFitChunks, G);
  const int wp = small_smem_wp(f.k) <= 227 * 1024 ? 1 : 0;
  const size_t ssm = wp ? small_smem_wp(f.k) : small_smem_base(f.k);
  e = cudaFuncSetAttribute(rsvd_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssm);
  if (e != cudaSuccess) return e;
  rsvd_small_kernel<<<f.Hkv, kSThreads, ssm, s>>>(G, f.omega, f.k, f.rank, f.power_iters, sw,
                                                  f.factor, f.sigma2, wp);
  return cudaGetLastError();
}

}  // namespace kvc
