// Joint rank / residual-bit allocation under one byte budget (host code).
//
// "JoLT: Near-Lossless KV Cache Compression", section "How JoLT works": the
// layers are grouped, keys and values of each group are separate cells, and
// one Lagrangian multiplier picks every cell's ranks and residual bit-width
// under a shared byte budget; "A JoLT for the KV cache ...", "Abstract
// (arXiv)": a single Lagrangian dual under a global byte constraint.
//
// For a multiplier lam each cell independently takes the option with the least
// distortion + lam * bytes; the total bytes only change where lam crosses a
// cell's pairwise break point (D_a - D_b) / (B_b - B_a), so the smallest
// feasible multiplier is found exactly by a binary search over the sorted
// break points (bytes are non-increasing in lam).  The allocation at that lam
// has the least total distortion of all allocations that use no more bytes
// (Everett's theorem for Lagrange multipliers).
#include <math.h>

#include <algorithm>
#include <vector>

#include "kvc_internal.h"

namespace {

// Option of cell c minimising D + lam * B; ties go to fewer bytes, then to the
// earlier option.
int best_option(const double* B, const double* D, int n_opt, double lam) {
  int best = 0;
  for (int j = 1; j < n_opt; ++j) {
    const double vj = D[j] + lam * B[j];
    const double vb = D[best] + lam * B[best];
    if (vj < vb || (vj == vb && B[j] < B[best])) best = j;
  }
  return best;
}

double total_bytes(int n_cells, int n_opt, const double* B, const double* D, double lam,
                   int32_t* choice) {
  double t = 0.0;
  for (int c = 0; c < n_cells; ++c) {
    const int j = best_option(B + (size_t)c * n_opt, D + (size_t)c * n_opt, n_opt, lam);
    if (choice) choice[c] = j;
    t += B[(size_t)c * n_opt + j];
  }
  return t;
}

int ceil_div(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

}  // namespace

extern "C" kvc_status kvc_rank_bit_tables(int32_t n_cells, int32_t spec_len,
                                          const double* spectra, const int64_t* rows,
                                          const int32_t* heads, int32_t n_options,
                                          const kvc_rank_bits* options, int32_t head_dim,
                                          int32_t latent_bits, int32_t group, double eta_latent,
                                          const double* eta_resid, double* bytes,
                                          double* distortion) {
  if (n_cells < 1 || spec_len < 1 || n_options < 1 || !spectra || !rows || !heads || !options ||
      !eta_resid || !bytes || !distortion)
    return kvc::report_error(KVC_EINVAL, "kvc_rank_bit_tables: NULL argument or empty size");
  if (head_dim < 1 || group < 1 || (latent_bits != 16 && (latent_bits < 1 || latent_bits > 8)))
    return kvc::report_error(KVC_EINVAL, "kvc_rank_bit_tables: head_dim %d, latent_bits %d, group %d",
                             head_dim, latent_bits, group);
  for (int j = 0; j < n_options; ++j) {
    if (options[j].rank < 1 || options[j].rank > spec_len || options[j].bits < 0 ||
        options[j].bits > KVC_MAX_RESID_BITS || (head_dim * options[j].bits) % 8)
      return kvc::report_error(KVC_EINVAL, "option %d: rank %d / bits %d outside 1..%d / 0..%d",
                               j, options[j].rank, options[j].bits, spec_len,
                               KVC_MAX_RESID_BITS);
  }
  for (int c = 0; c < n_cells; ++c) {
    const double* s = spectra + (size_t)c * spec_len;
    double total = 0.0;
    for (int i = 0; i < spec_len; ++i) total += s[i];
    for (int j = 0; j < n_options; ++j) {
      const int r = options[j].rank, b = options[j].bits;
      double head = 0.0;
      for (int i = 0; i < r; ++i) head += s[i];
      const double tail = total - head;
      const int lat = ceil_div((int64_t)r * latent_bits, 8) +
                      (latent_bits < 16 ? 4 * ceil_div(r, group) : 0);
      const int res = b > 0 ? head_dim * b / 8 + 2 : 0;
      bytes[(size_t)c * n_options + j] =
          (double)rows[c] * (lat + res) + (double)heads[c] * r * head_dim * 2 +
          (b > 0 ? (double)heads[c] * head_dim : 0.0);
      distortion[(size_t)c * n_options + j] = eta_latent * head + eta_resid[b] * tail;
    }
  }
  return KVC_OK;
}

extern "C" kvc_status kvc_allocate_rank_bits(int32_t n_cells, int32_t n_options,
                                             const double* bytes, const double* distortion,
                                             double budget, int32_t* choice, double* lambda) {
  if (n_cells < 1 || n_options < 1 || !bytes || !distortion || !choice)
    return kvc::report_error(KVC_EINVAL, "kvc_allocate_rank_bits: NULL argument or empty size");
  for (size_t i = 0; i < (size_t)n_cells * n_options; ++i) {
    if (!(bytes[i] >= 0.0) || !isfinite(bytes[i]) || !isfinite(distortion[i]))
      return kvc::report_error(KVC_EINVAL, "kvc_allocate_rank_bits: entry %zu not finite / negative",
                               i);
  }
  std::vector<double> pts;
  pts.push_back(0.0);
  for (int c = 0; c < n_cells; ++c) {
    const double* B = bytes + (size_t)c * n_options;
    const double* D = distortion + (size_t)c * n_options;
    for (int a = 0; a < n_options; ++a)
      for (int b = 0; b < n_options; ++b)
        if (B[a] < B[b] && D[a] > D[b]) pts.push_back((D[a] - D[b]) / (B[b] - B[a]));
  }
  std::sort(pts.begin(), pts.end());
  pts.erase(std::unique(pts.begin(), pts.end()), pts.end());
  size_t lo = 0, hi = pts.size() - 1;
  if (total_bytes(n_cells, n_options, bytes, distortion, pts[hi], nullptr) > budget)
    return kvc::report_error(KVC_ECAPACITY,
                             "kvc_allocate_rank_bits: the cheapest options need more than %.17g bytes",
                             budget);
  while (lo < hi) {
    const size_t mid = (lo + hi) / 2;
    if (total_bytes(n_cells, n_options, bytes, distortion, pts[mid], nullptr) <= budget) hi = mid;
    else lo = mid + 1;
  }
  total_bytes(n_cells, n_options, bytes, distortion, pts[lo], choice);
  if (lambda) *lambda = pts[lo];
  return KVC_OK;
}
