// PrinMix-style bit allocation and reconstruction-target correction (offline, host, fp64).
//
// "Enhancing Delta Compression in LLMs via SVD-based Quantization Error Minimization" (PrinMix,
// a follow-up to Delta-CoMe that keeps its factorisation W = U Sigma V):
//   - section 2.1, eq. 5: quantising row i of V changes the output on calibration activations X by
//     about Sigma_ii^2 * dV_i X X^T dV_i^T, dV_i the row's quantisation error (exact for a single
//     row when U has orthonormal columns);
//   - section 2.2: one width per row from a candidate set, a bit budget, at most K distinct widths,
//     minimising the summed error: a 0/1 integer linear program;
//   - section 2.3: after V is quantised, U is refit so that U~ Sigma V^ X matches U Sigma V X in the
//     least-squares sense before U is quantised (reconstruction-target correction, RTC).
// Readings: the error of width b for row i takes dV_i = v_i - RTN_b(v_i) (the serving quantiser,
// groups of 128 along d_in) and dV_i = v_i for 0 bits; a width costs b (d_out + d_in) code bits per
// rank, the budget being ratio * 16 * d_out * d_in code bits as for the greedy plans; RTC refits the
// kept ranks only.  The ILP is solved exactly: for every allowed set of at most K nonzero widths,
// a dynamic program over the budget (costs are integer multiples of d_out + d_in bits) gives the
// best assignment; the best over the sets is the optimum.  Ranks are then grouped by width,
// widest first, into the serving bands (8, 3, 2 bits; 0 = dropped), keeping singular-value order
// inside a band.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <thread>
#include <vector>

#include "dc.h"
#include "dc_internal.h"

namespace {

int n_threads() {
  unsigned n = std::thread::hardware_concurrency();
  return (int)std::max(1u, std::min(n, 32u));
}

template <class F>
void parallel_for(int n, F f) {
  const int nth = std::min(n_threads(), std::max(n, 1));
  std::vector<std::thread> th;
  for (int t = 1; t < nth; ++t) th.emplace_back([&, t] {
      for (int i = t; i < n; i += nth) f(i);
    });
  for (int i = 0; i < n; i += nth) f(i);
  for (auto& x : th) x.join();
}

// v_hat of one vector at `bits` (the serving RTN rule, groups of 128), fp64.
bool dequant_vector(const float* v, int n, int bits, std::vector<double>& out) {
  out.assign(n, 0.0);
  if (bits == 0) return true;
  std::vector<uint8_t> codes(128);
  for (int g = 0; g < n; g += 128) {
    uint16_t sz[2];
    if (!dc_rtn_group(v + g, 1, 128, bits, codes.data(), 1, sz)) return false;
    const double sc = dc_f16_to_f64(sz[0]), z = dc_f16_to_f64(sz[1]);
    for (int k = 0; k < 128; ++k) out[g + k] = ((double)codes[k] - z) * sc;
  }
  return true;
}

bool width_ok(int b) { return b == 0 || b == 2 || b == 3 || b == 8; }

}  // namespace

extern "C" dc_status dc_prinmix_scores(const float* Vt, const float* S, int32_t r, int32_t d_in, const float* X,
                                       int32_t n, const int32_t* widths, int32_t n_widths, double* scores) {
  DC_NVTX("dc_prinmix_scores");
  dc_clear_error();
  if (!Vt || !S || !X || !widths || !scores) return dc_fail(DC_ERR_INVALID_ARG, "null pointer");
  if (r <= 0 || d_in <= 0 || d_in % 128 || n <= 0 || n_widths <= 0 || n_widths > 8)
    return dc_fail(DC_ERR_SHAPE, "prinmix scores: bad sizes");
  for (int j = 0; j < n_widths; ++j)
    if (!width_ok(widths[j])) return dc_fail(DC_ERR_BITS, "width %d not in {0, 2, 3, 8}", widths[j]);
  std::vector<int> bad(r, 0);
  parallel_for(r, [&](int i) {
    std::vector<double> vh;
    std::vector<double> dv(d_in);
    const float* v = Vt + (int64_t)i * d_in;
    const double s2 = (double)S[i] * (double)S[i];
    for (int j = 0; j < n_widths; ++j) {
      if (!dequant_vector(v, d_in, widths[j], vh)) {
        bad[i] = 1;
        return;
      }
      for (int k = 0; k < d_in; ++k) dv[k] = (double)v[k] - vh[k];
      double e = 0.0;
      for (int t = 0; t < n; ++t) {
        const float* x = X + (int64_t)t * d_in;
        double p = 0.0;
        for (int k = 0; k < d_in; ++k) p += dv[k] * (double)x[k];
        e += p * p;
      }
      scores[(int64_t)i * n_widths + j] = s2 * e;
    }
  });
  for (int i = 0; i < r; ++i)
    if (bad[i]) return dc_fail(DC_ERR_INVALID_ARG, "rank %d: non-finite value or fp16 scale overflow", i);
  return DC_OK;
}

extern "C" dc_status dc_prinmix_allocate(const double* scores, int32_t r, const int32_t* widths, int32_t n_widths,
                                         int32_t d_out, int32_t d_in, double ratio, int32_t max_kinds,
                                         int32_t* width_out, double* objective) {
  DC_NVTX("dc_prinmix_allocate");
  dc_clear_error();
  if (!scores || !widths || !width_out) return dc_fail(DC_ERR_INVALID_ARG, "null pointer");
  if (r <= 0 || n_widths <= 0 || n_widths > 8 || d_out <= 0 || d_in <= 0 || !(ratio > 0.0) || max_kinds < 1)
    return dc_fail(DC_ERR_INVALID_ARG, "prinmix allocate: bad arguments");
  int zero_col = -1;
  std::vector<int> nz;  // columns of nonzero widths
  for (int j = 0; j < n_widths; ++j) {
    if (!width_ok(widths[j])) return dc_fail(DC_ERR_BITS, "width %d not in {0, 2, 3, 8}", widths[j]);
    if (widths[j] == 0)
      zero_col = j;
    else
      nz.push_back(j);
  }
  if (zero_col < 0) return dc_fail(DC_ERR_INVALID_ARG, "the candidate widths must include 0 (dropping a rank)");
  const double budget_bits = ratio * 16.0 * (double)d_out * (double)d_in;
  const int64_t cap64 = (int64_t)std::floor(budget_bits / (double)(d_out + d_in) + 1e-9);
  const int cap = (int)std::min<int64_t>(cap64, (int64_t)8 * r);
  if (cap < 0) return dc_fail(DC_ERR_INVALID_ARG, "negative budget");
  const int ns = (int)nz.size();
  double best = INFINITY;
  std::vector<int32_t> best_w(r, 0);
  std::vector<double> dp(cap + 1), nd(cap + 1);
  std::vector<uint8_t> choice((size_t)r * (cap + 1));
  for (int mask = 0; mask < (1 << ns); ++mask) {
    if (__builtin_popcount(mask) > max_kinds) continue;
    std::vector<int> cols{zero_col};
    for (int k = 0; k < ns; ++k)
      if (mask & (1 << k)) cols.push_back(nz[k]);
    // dp[c]: least error of the rows so far using at most c budget units
    std::fill(dp.begin(), dp.end(), 0.0);
    for (int i = 0; i < r; ++i) {
      const double* sc = scores + (int64_t)i * n_widths;
      uint8_t* ch = choice.data() + (size_t)i * (cap + 1);
      for (int c = 0; c <= cap; ++c) {
        double v = INFINITY;
        uint8_t arg = 0;
        for (size_t k = 0; k < cols.size(); ++k) {
          const int w = widths[cols[k]];
          if (w > c) continue;
          const double cand = dp[c - w] + sc[cols[k]];
          if (cand < v) {  // first (narrowest-listed) width wins a tie
            v = cand;
            arg = (uint8_t)k;
          }
        }
        nd[c] = v;
        ch[c] = arg;
      }
      std::swap(dp, nd);
    }
    if (dp[cap] < best) {
      best = dp[cap];
      int c = cap;
      for (int i = r - 1; i >= 0; --i) {
        const int w = widths[cols[choice[(size_t)i * (cap + 1) + c]]];
        best_w[i] = w;
        c -= w;
      }
    }
  }
  std::memcpy(width_out, best_w.data(), sizeof(int32_t) * r);
  if (objective) *objective = best;
  return DC_OK;
}

extern "C" dc_status dc_prinmix_rtc(const float* U, const float* S, const float* Vt, const float* Vt_hat, int32_t k,
                                    int32_t d_out, int32_t d_in, const float* X, int32_t n, float* U_out) {
  DC_NVTX("dc_prinmix_rtc");
  dc_clear_error();
  if (!U || !S || !Vt || !Vt_hat || !X || !U_out) return dc_fail(DC_ERR_INVALID_ARG, "null pointer");
  if (k <= 0 || d_out <= 0 || d_in <= 0 || n <= 0) return dc_fail(DC_ERR_SHAPE, "prinmix rtc: bad sizes");
  // A = Sigma V_hat X^T, B = Sigma V X^T  (k x n)
  std::vector<double> A((size_t)k * n), B((size_t)k * n);
  parallel_for(k, [&](int i) {
    const float* v = Vt + (int64_t)i * d_in;
    const float* vh = Vt_hat + (int64_t)i * d_in;
    for (int t = 0; t < n; ++t) {
      const float* x = X + (int64_t)t * d_in;
      double a = 0.0, b = 0.0;
      for (int c = 0; c < d_in; ++c) {
        a += (double)vh[c] * x[c];
        b += (double)v[c] * x[c];
      }
      A[(size_t)i * n + t] = (double)S[i] * a;
      B[(size_t)i * n + t] = (double)S[i] * b;
    }
  });
  // G = A A^T (k x k, SPD when the calibration set spans the kept rows), H = B A^T
  std::vector<double> G((size_t)k * k), H((size_t)k * k);
  parallel_for(k, [&](int i) {
    for (int j = 0; j < k; ++j) {
      double g = 0.0, h = 0.0;
      for (int t = 0; t < n; ++t) {
        g += A[(size_t)i * n + t] * A[(size_t)j * n + t];
        h += B[(size_t)i * n + t] * A[(size_t)j * n + t];
      }
      G[(size_t)i * k + j] = g;
      H[(size_t)i * k + j] = h;
    }
  });
  // a tiny ridge keeps the factorisation defined when X does not span every kept row
  double tr = 0.0;
  for (int i = 0; i < k; ++i) tr += G[(size_t)i * k + i];
  const double ridge = 1e-12 * (tr > 0 ? tr / k : 1.0);
  for (int i = 0; i < k; ++i) G[(size_t)i * k + i] += ridge;
  // Cholesky G = L L^T (lower, in place)
  for (int j = 0; j < k; ++j) {
    double d = G[(size_t)j * k + j];
    for (int p = 0; p < j; ++p) d -= G[(size_t)j * k + p] * G[(size_t)j * k + p];
    if (!(d > 0.0)) return dc_fail(DC_ERR_INVALID_ARG, "prinmix rtc: calibration Gram matrix not positive definite");
    const double ljj = std::sqrt(d);
    G[(size_t)j * k + j] = ljj;
    for (int i = j + 1; i < k; ++i) {
      double v = G[(size_t)i * k + j];
      for (int p = 0; p < j; ++p) v -= G[(size_t)i * k + p] * G[(size_t)j * k + p];
      G[(size_t)i * k + j] = v / ljj;
    }
  }
  // M = H G^-1: each row m of M solves G m^T = h^T (G symmetric), by forward and back substitution
  std::vector<double> M((size_t)k * k);
  parallel_for(k, [&](int i) {
    std::vector<double> y(k);
    const double* h = H.data() + (size_t)i * k;
    for (int a = 0; a < k; ++a) {
      double v = h[a];
      for (int p = 0; p < a; ++p) v -= G[(size_t)a * k + p] * y[p];
      y[a] = v / G[(size_t)a * k + a];
    }
    for (int a = k - 1; a >= 0; --a) {
      double v = y[a];
      for (int p = a + 1; p < k; ++p) v -= G[(size_t)p * k + a] * M[(size_t)i * k + p];
      M[(size_t)i * k + a] = v / G[(size_t)a * k + a];
    }
  });
  // U~ = U M: column j of U~ = sum_i M[i][j] u_i  (U, U_out column-major [d_out, k])
  parallel_for(k, [&](int j) {
    std::vector<double> col(d_out, 0.0);
    for (int i = 0; i < k; ++i) {
      const double m = M[(size_t)i * k + j];
      const float* u = U + (int64_t)i * d_out;
      for (int o = 0; o < d_out; ++o) col[o] += m * (double)u[o];
    }
    for (int o = 0; o < d_out; ++o) U_out[(int64_t)j * d_out + o] = (float)col[o];
  });
  return DC_OK;
}

extern "C" dc_status dc_prinmix_compress(const float* U, const float* S, const float* Vt, int32_t r, int32_t d_out,
                                         int32_t d_in, const float* X, int32_t n, double ratio,
                                         const int32_t* widths, int32_t n_widths, int32_t max_kinds, int32_t rtc,
                                         dc_factor_desc* desc_out, int32_t* perm_out, float* U_out, float* S_out,
                                         float* Vt_out, double* objective) {
  DC_NVTX("dc_prinmix_compress");
  dc_clear_error();
  if (!U || !S || !Vt || !X || !widths || !desc_out || !perm_out || !U_out || !S_out || !Vt_out)
    return dc_fail(DC_ERR_INVALID_ARG, "null pointer");
  if (r <= 0 || d_out <= 0 || d_in <= 0 || d_out % 128 || d_in % 128 || r > std::min(d_out, d_in))
    return dc_fail(DC_ERR_SHAPE, "prinmix: bad sizes");
  std::vector<double> sc((size_t)r * n_widths);
  dc_status st = dc_prinmix_scores(Vt, S, r, d_in, X, n, widths, n_widths, sc.data());
  if (st) return st;
  std::vector<int32_t> w(r);
  st = dc_prinmix_allocate(sc.data(), r, widths, n_widths, d_out, d_in, ratio, max_kinds, w.data(), objective);
  if (st) return st;
  // bands, widest first; singular-value order inside a band
  const int order[3] = {8, 3, 2};
  std::memset(desc_out, 0, sizeof(*desc_out));
  desc_out->d_out = d_out;
  desc_out->d_in = d_in;
  int k = 0;
  for (int b : order) {
    int cnt = 0;
    for (int i = 0; i < r; ++i)
      if (w[i] == b) perm_out[k + cnt++] = i;
    if (cnt > 0) {
      desc_out->bits[desc_out->n_bands] = b;
      desc_out->rank[desc_out->n_bands] = cnt;
      ++desc_out->n_bands;
    }
    k += cnt;
  }
  for (int i = k; i < r; ++i) perm_out[i] = -1;
  for (int i = 0; i < k; ++i) {
    const int src = perm_out[i];
    S_out[i] = S[src];
    std::memcpy(Vt_out + (int64_t)i * d_in, Vt + (int64_t)src * d_in, sizeof(float) * d_in);
    std::memcpy(U_out + (int64_t)i * d_out, U + (int64_t)src * d_out, sizeof(float) * d_out);
  }
  if (!rtc || k == 0) return DC_OK;
  // V_hat of the kept rows at their widths, then U refit to it
  std::vector<float> vh((size_t)k * d_in);
  std::vector<int> bad(k, 0);
  parallel_for(k, [&](int i) {
    std::vector<double> d;
    if (!dequant_vector(Vt_out + (int64_t)i * d_in, d_in, w[perm_out[i]], d)) bad[i] = 1;
    for (int c = 0; c < d_in && !bad[i]; ++c) vh[(size_t)i * d_in + c] = (float)d[c];
  });
  for (int i = 0; i < k; ++i)
    if (bad[i]) return dc_fail(DC_ERR_INVALID_ARG, "rank %d: non-finite value or fp16 scale overflow", perm_out[i]);
  std::vector<float> Uk(U_out, U_out + (size_t)k * d_out);
  return dc_prinmix_rtc(Uk.data(), S_out, Vt_out, vh.data(), k, d_out, d_in, X, n, U_out);
}
