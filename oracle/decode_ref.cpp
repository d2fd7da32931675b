// decode_ref.cpp -- plain C++ oracle of the SAGA + Atop-N decode step, in double.
//
// TEST INFRASTRUCTURE ONLY: loaded by tests/ and by the bench's CPU legs, never
// by the CUDA library or its binding, with which it shares no code.
//
// "More Value per Key" (Elata et al.): for every batch row b and query head j,
//   z_i = (q_j . k_i) / sqrt(d) over the L_b cached positions        Eq. (2), (5)
//   I   = the N_b = min(N, L_b) positions with the largest z, ties to
//         the lowest position (the exact N-th score as the threshold)  Eq. (6), §3.1
//   p_i = exp(z_i - max_I z) / sum_{l in I} exp(z_l - max_I z)         Eq. (7)
//   out = sum_{i in I} p_i v_i                                        Eq. (7)
// with query head j reading key head j / (h_q / h_k) and value head
// j / (h_q / h_v) (§3.2, App. B Eq. (29)).  Inputs are bf16 bit patterns, widened
// exactly to double; every product and sum is in double.  Rows run on `threads`
// std::threads (1 = single-threaded).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <thread>
#include <vector>

namespace {

double bf16_to_double(uint16_t h) {
  const uint32_t bits = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &bits, sizeof(f));
  return static_cast<double>(f);
}

struct Problem {
  const uint16_t *q, *k, *v;
  const int32_t* seq_lens;
  int B, L_max, h_q, h_k, h_v, d, N;
  double* out;          // [B][h_q][d]
  int32_t* sel_idx;     // [B][h_q][N], -1 padding
  double* sel_logit;    // [B][h_q][N], -inf padding
};

void one_row(const Problem& P, int b, int j) {
  const int g = P.h_q / P.h_k, g_v = P.h_q / P.h_v, d = P.d;
  const int L = P.seq_lens[b];
  double* o = P.out + (static_cast<long long>(b) * P.h_q + j) * d;
  int32_t* idx_out = P.sel_idx + (static_cast<long long>(b) * P.h_q + j) * P.N;
  double* logit_out = P.sel_logit + (static_cast<long long>(b) * P.h_q + j) * P.N;
  for (int r = 0; r < P.N; ++r) { idx_out[r] = -1; logit_out[r] = -INFINITY; }
  for (int t = 0; t < d; ++t) o[t] = 0.0;
  if (L < 1 || L > P.L_max) return;
  std::vector<double> q(d);
  for (int t = 0; t < d; ++t) q[t] = bf16_to_double(P.q[(static_cast<long long>(b) * P.h_q + j) * d + t]);
  const uint16_t* krow = P.k + (static_cast<long long>(b) * P.h_k + j / g) * P.L_max * d;
  const uint16_t* vrow = P.v + (static_cast<long long>(b) * P.h_v + j / g_v) * P.L_max * d;
  const double scale = 1.0 / std::sqrt(static_cast<double>(d));
  std::vector<double> z(L);
  for (int i = 0; i < L; ++i) {
    double acc = 0.0;
    for (int t = 0; t < d; ++t) acc += q[t] * bf16_to_double(krow[static_cast<long long>(i) * d + t]);
    z[i] = acc * scale;
  }
  // order by (z descending, position ascending); the first N_b are I
  std::vector<int> order(L);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int a, int c) { return z[a] > z[c]; });
  const int n_b = std::min(P.N, L);
  std::vector<int> sel(order.begin(), order.begin() + n_b);
  std::sort(sel.begin(), sel.end());
  double m = -INFINITY;
  for (int i : sel) m = std::max(m, z[i]);
  double denom = 0.0;
  for (int i : sel) denom += std::exp(z[i] - m);
  for (int r = 0; r < n_b; ++r) {
    const int i = sel[r];
    idx_out[r] = i;
    logit_out[r] = z[i];
    const double p = std::exp(z[i] - m) / denom;
    for (int t = 0; t < d; ++t) o[t] += p * bf16_to_double(vrow[static_cast<long long>(i) * d + t]);
  }
}

}  // namespace

extern "C" int saga_oracle_decode(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                  const int32_t* seq_lens, int B, int L_max, int h_q, int h_k,
                                  int h_v, int d, int N, int threads, double* out, int32_t* sel_idx,
                                  double* sel_logit) {
  if (!q || !k || !v || !seq_lens || !out || !sel_idx || !sel_logit) return 1;
  if (B < 1 || L_max < 1 || h_q < 1 || h_k < 1 || h_v < 1 || d < 1 || N < 1) return 1;
  if (h_q % h_k != 0 || h_q % h_v != 0) return 1;
  const Problem P{q, k, v, seq_lens, B, L_max, h_q, h_k, h_v, d, N, out, sel_idx, sel_logit};
  const int rows = B * h_q;
  const int nt = std::max(1, std::min(threads, rows));
  std::vector<std::thread> pool;
  for (int w = 0; w < nt; ++w)
    pool.emplace_back([&P, rows, nt, w]() {
      for (int r = w; r < rows; r += nt) one_row(P, r / P.h_q, r % P.h_q);
    });
  for (auto& t : pool) t.join();
  return 0;
}
