// TEST INFRASTRUCTURE -- not part of the product.
//
// A plain, slow, double-precision CPU statement of the Walsh-Hadamard adapter
// (WHA) layer of "QWHA: Quantization-Aware Walsh-Hadamard Adaptation for
// Parameter-Efficient Fine-Tuning on Large Language Models". Only the test
// suite, the package smoke check and the benchmark's CPU-baseline leg load it.
// It shares no code, header, table or helper with the CUDA library; the two are
// compared on the same seeded inputs.
//
// Sources (page title, then section):
//   [P1] papernotes.org "QWHA ...", 整体框架 (framework), 关键设计 1/2/3,
//        损失函数 / 训练策略
//   [P2] gist.science "Technical Summary: QWHA ...", 2.1 Adapter Design,
//        2.2 Quantization-Aware Initialization
//
// Readings taken where the pages are silent (each also listed in the design
// notes of the repository):
//   * H is the Sylvester-ordered Walsh-Hadamard matrix, normalised to be
//     orthonormal: H_n[i][j] = (-1)^popcount(i & j) / sqrt(n). Then H is
//     symmetric and its own inverse, so the adapter update dW = F H^-1 [P1 设计1,
//     P2 2.1] equals F H.
//   * A layer whose d_in is not a power of two uses the block-diagonal matrix
//     of d_in/n equal blocks H_n.
//   * Forward Y = X W_Q^T + alpha X dW^T, with alpha the adapter scale
//     [P1 训练策略: alpha ~ 1].
//   * Backward, only c trainable [P1 整体框架]: dc_j = dL/dc_j and dX = dL/dX
//     for L = <Y, dY>.
//   * AdaAlloc [P1 设计2, P2 2.2]: the per-channel budget formula is lost from
//     the page, so the budget is proportional to the error norm of the
//     channel, ||dW_Q[i,:]||_2 (no calibration activations: X = I), after a
//     floor of min_per_row per channel; rounding remainder to the channels
//     chosen by `mode`; per-channel cap d_in with the surplus re-shared.
//     Within a channel the largest |(dW_Q H)[i,k]| win, ties to the lower k;
//     the values are the dense solution (dW_Q H)[i,k] [P1 设计3, x0].
//   * Sums that decide an integer (the budgets) use a fixed pairwise tree in
//     index order over the zero-padded power-of-two length, and the transform
//     used for ranking runs its butterfly stages in the textbook order
//     h = 1, 2, 4, ..., n/2 in double, unnormalised. This fixes every rounding
//     so that a GPU implementation can reproduce E and the budgets bit for bit.
//
// Build: g++ -O2 -std=c++17 -ffp-contract=off -fPIC -shared -pthread
// (never -ffast-math).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <mutex>
#include <numeric>
#include <thread>
#include <vector>

namespace {

int g_threads = 0;

int thread_count() {
  if (g_threads > 0) return g_threads;
  const char *env = std::getenv("QWHA_ORACLE_THREADS");
  int n = env ? std::atoi(env) : 0;
  if (n <= 0) n = (int)std::thread::hardware_concurrency();
  if (n <= 0) n = 1;
  return n;
}

// Run f(i) for i in [0, n), split into contiguous static ranges.
template <class F>
void parallel_for(int64_t n, F f) {
  int nt = thread_count();
  if (n < 2 || nt == 1) {
    for (int64_t i = 0; i < n; ++i) f(i);
    return;
  }
  if ((int64_t)nt > n) nt = (int)n;
  std::vector<std::thread> pool;
  pool.reserve(nt);
  for (int t = 0; t < nt; ++t) {
    int64_t lo = n * t / nt, hi = n * (t + 1) / nt;
    pool.emplace_back([lo, hi, &f] {
      for (int64_t i = lo; i < hi; ++i) f(i);
    });
  }
  for (auto &th : pool) th.join();
}

bool is_pow2(int64_t n) { return n > 0 && (n & (n - 1)) == 0; }

// Entry (a, b) of the orthonormal Sylvester matrix H_n; inv = 1/sqrt(n).
double hadamard_entry(double inv, int a, int b) {
  int parity = __builtin_popcount((unsigned)(a & b)) & 1;
  return parity ? -inv : inv;
}

// Entry (a, b) of the block-diagonal matrix made of equal blocks H_n.
double blockdiag_entry(int n, double inv, int a, int b) {
  if (a / n != b / n) return 0.0;
  return hadamard_entry(inv, a % n, b % n);
}

double inv_sqrt(int n) { return 1.0 / std::sqrt((double)n); }

bool shape_ok(int d, int n) { return d > 0 && is_pow2(n) && d % n == 0; }

// Textbook in-place Walsh-Hadamard butterflies on one block of length n,
// stages h = 1, 2, 4, ..., n/2: (x[j], x[j+h]) <- (x[j] + x[j+h], x[j] - x[j+h]).
void butterflies(double *x, int n) {
  for (int h = 1; h < n; h <<= 1)
    for (int j = 0; j < n; ++j)
      if ((j & h) == 0) {
        double a = x[j], b = x[j + h];
        x[j] = a + b;
        x[j + h] = a - b;
      }
}

// Pairwise sum in index order over the length rounded up to a power of two
// (missing terms are zero): sum(v[0:m]) = sum(v[0:m/2]) + sum(v[m/2:m]).
double pairwise_sum(const double *v, int64_t len) {
  int64_t m = 1;
  while (m < len) m <<= 1;
  std::vector<double> buf(m, 0.0);
  for (int64_t i = 0; i < len; ++i) buf[i] = v[i];
  for (int64_t w = m; w > 1; w >>= 1)
    for (int64_t i = 0; i < w / 2; ++i) buf[i] = buf[2 * i] + buf[2 * i + 1];
  return buf[0];
}

// Dense dW = F H, F given in CSR by output row. [P1 设计1; P2 2.1: dW = F H^-1]
void delta_w(int d_out, int d_in, int n, const int32_t *row_ptr, const int32_t *col_idx,
             const double *coef, double *dW) {
  const double inv = inv_sqrt(n);
  parallel_for(d_out, [&](int64_t r) {
    double *row = dW + r * (int64_t)d_in;
    for (int k = 0; k < d_in; ++k) row[k] = 0.0;
    for (int32_t j = row_ptr[r]; j < row_ptr[r + 1]; ++j)
      for (int k = 0; k < d_in; ++k) row[k] += coef[j] * blockdiag_entry(n, inv, col_idx[j], k);
  });
}

}  // namespace

extern "C" {

// Thread count override for timing (0 = automatic). Returns the count in use.
int oracle_set_threads(int n) {
  g_threads = n;
  return thread_count();
}

// Dense orthonormal Sylvester Hadamard matrix H_n, n a power of two. [P2 2.1:
// H is fixed in advance and never trained; P1 设计1: its entries are +-1 up to
// the scale]
int oracle_hadamard(int32_t n, double *H) {
  if (!is_pow2(n)) return 1;
  const double inv = inv_sqrt(n);
  for (int a = 0; a < n; ++a)
    for (int b = 0; b < n; ++b) H[(int64_t)a * n + b] = hadamard_entry(inv, a, b);
  return 0;
}

// Z = X H by the definition of a matrix product with the dense (block-diagonal)
// H. X is [rows, d] row-major.
int oracle_transform_dense(const double *X, int64_t rows, int32_t d, int32_t n, double *Z) {
  if (!shape_ok(d, n)) return 1;
  const double inv = inv_sqrt(n);
  parallel_for(rows, [&](int64_t t) {
    const double *x = X + t * d;
    double *z = Z + t * d;
    for (int k = 0; k < d; ++k) {
      double acc = 0.0;
      for (int i = 0; i < d; ++i) acc += x[i] * blockdiag_entry(n, inv, i, k);
      z[k] = acc;
    }
  });
  return 0;
}

// The fast transform [P1 设计1 and P2 2.1: because every entry of H is +-1, the
// transform is a recursion of sums and differences with no multiplications],
// per block of n, textbook stage order; then, if `normalize`, each output times
// 1/sqrt(n).
int oracle_fwht(const double *X, int64_t rows, int32_t d, int32_t n, int32_t normalize, double *Z) {
  if (!shape_ok(d, n)) return 1;
  const double inv = inv_sqrt(n);
  parallel_for(rows, [&](int64_t t) {
    std::vector<double> b(n);
    for (int blk = 0; blk < d / n; ++blk) {
      const double *x = X + t * d + (int64_t)blk * n;
      double *z = Z + t * d + (int64_t)blk * n;
      for (int i = 0; i < n; ++i) b[i] = x[i];
      butterflies(b.data(), n);
      for (int i = 0; i < n; ++i) z[i] = normalize ? b[i] * inv : b[i];
    }
  });
  return 0;
}

// W_Q[i,k] = s[i,g] * (q[i,k] - z[i,g]) in single precision, g = k / group;
// q[i,k] is bits [bits*k, bits*k + bits) of row i's little-endian bit stream
// (row stride d_in*bits/8 bytes). Returned widened to double.
int oracle_dequant(int32_t bits, int32_t group, int32_t d_out, int32_t d_in, const uint8_t *qweight,
                   const float *scales, const uint8_t *zeros, double *Wq) {
  if (bits < 1 || bits > 8 || group <= 0 || d_in % group || (d_in * bits) % 8) return 1;
  const int64_t stride = (int64_t)d_in * bits / 8;
  const int ng = d_in / group;
  parallel_for(d_out, [&](int64_t i) {
    const uint8_t *row = qweight + i * stride;
    for (int k = 0; k < d_in; ++k) {
      int q = 0;
      for (int b = 0; b < bits; ++b) {
        int64_t bit = (int64_t)bits * k + b;
        q |= ((row[bit >> 3] >> (bit & 7)) & 1) << b;
      }
      float s = scales[i * ng + k / group];
      float diff = (float)q - (float)zeros[i * ng + k / group];
      float w = s * diff;
      Wq[i * d_in + k] = (double)w;
    }
  });
  return 0;
}

// Dense dW = F H for inspection by the tests.
int oracle_delta_w(int32_t d_out, int32_t d_in, int32_t n, const int32_t *row_ptr,
                   const int32_t *col_idx, const double *coef, double *dW) {
  if (!shape_ok(d_in, n) || d_out <= 0) return 1;
  delta_w(d_out, d_in, n, row_ptr, col_idx, coef, dW);
  return 0;
}

// Forward of the adapted layer by its definition [P1 整体框架, P2 2.1]:
//   Z = X H,   Y = X W_Q^T + alpha * X (F H)^T.
// Wq may be null (adapter only). X [T, d_in]; Z [T, d_in] (nullable); Y [T, d_out].
int oracle_adapter_fwd(int32_t d_out, int32_t d_in, int32_t n, const int32_t *row_ptr,
                       const int32_t *col_idx, const double *coef, const double *Wq, const double *X,
                       int64_t T, double alpha, double *Z, double *Y) {
  if (!shape_ok(d_in, n) || d_out <= 0 || T < 0) return 1;
  std::vector<double> dW((size_t)d_out * d_in);
  delta_w(d_out, d_in, n, row_ptr, col_idx, coef, dW.data());
  if (Z) oracle_transform_dense(X, T, d_in, n, Z);
  parallel_for(T, [&](int64_t t) {
    const double *x = X + t * d_in;
    for (int r = 0; r < d_out; ++r) {
      const double *a = dW.data() + (int64_t)r * d_in;
      double base = 0.0, ad = 0.0;
      if (Wq) {
        const double *w = Wq + (int64_t)r * d_in;
        for (int k = 0; k < d_in; ++k) base += x[k] * w[k];
      }
      for (int k = 0; k < d_in; ++k) ad += x[k] * a[k];
      Y[t * d_out + r] = base + alpha * ad;
    }
  });
  return 0;
}

// The same adapter output by the sparse route [P1 整体框架: F = Scatter(c, E)]:
//   Y_ad[t, r] = alpha * sum over nonzeros j of row r of c_j * (X H)[t, k_j],
// with X H from the fast transform. Used to cross-check the dense route.
int oracle_adapter_fwd_sparse(int32_t d_out, int32_t d_in, int32_t n, const int32_t *row_ptr,
                              const int32_t *col_idx, const double *coef, const double *X, int64_t T,
                              double alpha, double *Y) {
  if (!shape_ok(d_in, n) || d_out <= 0 || T < 0) return 1;
  std::vector<double> Z((size_t)T * d_in);
  oracle_fwht(X, T, d_in, n, 1, Z.data());
  parallel_for(T, [&](int64_t t) {
    const double *z = Z.data() + t * d_in;
    for (int r = 0; r < d_out; ++r) {
      double acc = 0.0;
      for (int32_t j = row_ptr[r]; j < row_ptr[r + 1]; ++j) acc += coef[j] * z[col_idx[j]];
      Y[t * d_out + r] = alpha * acc;
    }
  });
  return 0;
}

// Backward, input gradient, for L = <Y, dY>:
//   dX = dY W_Q + alpha * dY (F H).
// Wq nullable. dY [T, d_out]; dX [T, d_in].
int oracle_adapter_bwd_dx(int32_t d_out, int32_t d_in, int32_t n, const int32_t *row_ptr,
                          const int32_t *col_idx, const double *coef, const double *Wq,
                          const double *dY, int64_t T, double alpha, double *dX) {
  if (!shape_ok(d_in, n) || d_out <= 0 || T < 0) return 1;
  std::vector<double> dW((size_t)d_out * d_in);
  delta_w(d_out, d_in, n, row_ptr, col_idx, coef, dW.data());
  parallel_for(T, [&](int64_t t) {
    const double *g = dY + t * d_out;
    double *o = dX + t * d_in;
    for (int k = 0; k < d_in; ++k) {
      double base = 0.0, ad = 0.0;
      for (int r = 0; r < d_out; ++r) {
        if (Wq) base += g[r] * Wq[(int64_t)r * d_in + k];
        ad += g[r] * dW[(int64_t)r * d_in + k];
      }
      o[k] = base + alpha * ad;
    }
  });
  return 0;
}

// Backward, coefficient gradient at m given positions (r_j, k_j):
//   dc_j = alpha * sum_t dY[t, r_j] * (X H)[t, k_j],
// with (X H)[t, k] = sum_i X[t, i] H[i, k] by the definition of the product.
// X [T, d_in]; dY [T, d_out]; dc [m].
int oracle_adapter_bwd_dc(int32_t d_out, int32_t d_in, int32_t n, const double *X, const double *dY,
                          int64_t T, double alpha, int64_t m, const int32_t *rows,
                          const int32_t *cols, double *dc) {
  if (!shape_ok(d_in, n) || d_out <= 0 || T < 0) return 1;
  const double inv = inv_sqrt(n);
  parallel_for(m, [&](int64_t j) {
    const int r = rows[j], k = cols[j];
    double acc = 0.0;
    for (int64_t t = 0; t < T; ++t) {
      const double *x = X + t * d_in;
      double z = 0.0;
      for (int i = 0; i < d_in; ++i) z += x[i] * blockdiag_entry(n, inv, i, k);
      acc += dY[t * d_out + r] * z;
    }
    dc[j] = alpha * acc;
  });
  return 0;
}

// AdaAlloc initialisation [P1 设计2 and 设计3 (dense solution x0); P2 2.2].
//   e_i    = ||dW_Q[i,:]||_2 (squares in double, pairwise tree)       -> err_norm
//   budget = min_per_row + floor(pool * e_i / sum_active e), pool = p - min_per_row*d_out,
//            capped at d_in (capped rows leave; the rest re-share what is left);
//            remainder p - sum(budget) given one each, in order, to
//            mode 0: the least-allocated rows (budget asc, index asc)  [P1 设计2]
//            mode 1: the largest-error rows (e_i desc, index asc)
//   V      = dW_Q[i,:] H, unnormalised butterflies in textbook order, double
//   E row i = the budget_i indices of largest |V| (ties: lower index), ascending
//   c      = float(V * (1/sqrt(n)))
// Outputs: budgets [d_out], row_ptr [d_out+1], col_idx [p], coef [p],
// err_norm [d_out] (nullable).
// Step 1: e_i = ||dW_Q[i,:]||_2 for `rows` rows (fp64 squares, pairwise sum).
int oracle_init_norms(const float *dWq, int32_t rows, int32_t d_in, double *e) {
  if (rows < 0 || d_in <= 0) return 1;
  parallel_for(rows, [&](int64_t i) {
    std::vector<double> sq(d_in);
    for (int k = 0; k < d_in; ++k) {
      double w = (double)dWq[i * d_in + k];
      sq[k] = w * w;
    }
    e[i] = std::sqrt(pairwise_sum(sq.data(), d_in));
  });
  return 0;
}

// Step 2: budgets from all d_out norms. Floor share of the pool, capped at
// d_in, surplus re-shared; the remainder one each in the order of `mode`.
int oracle_init_budgets(const double *e, int32_t d_out, int32_t d_in, int64_t p, int32_t min_per_row,
                        int32_t mode, int32_t *budgets, int32_t *row_ptr) {
  if (d_out <= 0 || d_in <= 0 || min_per_row < 0 || min_per_row > d_in) return 1;
  if (p < (int64_t)min_per_row * d_out || p > (int64_t)d_in * d_out || p > 2147483647LL) return 1;
  if (mode != 0 && mode != 1) return 1;
  std::vector<int64_t> b(d_out, min_per_row);
  std::vector<char> capped(d_out, 0);
  double pool = (double)(p - (int64_t)min_per_row * d_out);
  for (;;) {
    std::vector<double> ea(d_out);
    int64_t n_active = 0;
    for (int i = 0; i < d_out; ++i) {
      ea[i] = capped[i] ? 0.0 : e[i];
      n_active += !capped[i];
    }
    if (n_active == 0) break;
    const double S = pairwise_sum(ea.data(), d_out);
    bool any_new = false;
    for (int i = 0; i < d_out; ++i) {
      if (capped[i]) continue;
      double share = S > 0.0 ? std::floor((pool * e[i]) / S) : std::floor(pool / (double)n_active);
      b[i] = min_per_row + (int64_t)share;
      if (b[i] > d_in) any_new = true;
    }
    if (!any_new) break;
    for (int i = 0; i < d_out; ++i)
      if (!capped[i] && b[i] > d_in) {
        b[i] = d_in;
        capped[i] = 1;
        pool -= (double)(d_in - min_per_row);
      }
  }
  int64_t R = p - std::accumulate(b.begin(), b.end(), (int64_t)0);
  std::vector<int> order(d_out);
  std::iota(order.begin(), order.end(), 0);
  if (mode == 0)
    std::stable_sort(order.begin(), order.end(), [&](int a, int c) { return b[a] < b[c]; });
  else
    std::stable_sort(order.begin(), order.end(), [&](int a, int c) { return e[a] > e[c]; });
  while (R > 0)
    for (int i : order)
      if (R > 0 && b[i] < d_in) {
        ++b[i];
        --R;
      }
  row_ptr[0] = 0;
  for (int i = 0; i < d_out; ++i) {
    budgets[i] = (int32_t)b[i];
    row_ptr[i + 1] = row_ptr[i] + (int32_t)b[i];
  }
  return 0;
}

// Step 3: in-channel selection of the largest transform magnitudes for `rows`
// rows; row i's entries go to [row_ptr[i] - row_ptr[0], + budgets[i]).
int oracle_init_select(const float *dWq, int32_t rows, int32_t d_in, int32_t n, const int32_t *budgets,
                       const int32_t *row_ptr, int32_t *col_idx, float *coef) {
  if (rows < 0 || !shape_ok(d_in, n)) return 1;
  for (int i = 0; i < rows; ++i)
    if (budgets[i] < 0 || budgets[i] > d_in || row_ptr[i + 1] - row_ptr[i] != budgets[i]) return 1;
  const double inv = inv_sqrt(n);
  const int32_t base = rows > 0 ? row_ptr[0] : 0;
  parallel_for(rows, [&](int64_t i) {
    std::vector<double> v(d_in);
    for (int k = 0; k < d_in; ++k) v[k] = (double)dWq[i * d_in + k];
    for (int blk = 0; blk < d_in / n; ++blk) butterflies(v.data() + (int64_t)blk * n, n);
    std::vector<int> idx(d_in);
    std::iota(idx.begin(), idx.end(), 0);
    std::sort(idx.begin(), idx.end(), [&](int a, int c) {
      double fa = std::fabs(v[a]), fc = std::fabs(v[c]);
      return fa > fc || (fa == fc && a < c);
    });
    std::vector<int> pick(idx.begin(), idx.begin() + budgets[i]);
    std::sort(pick.begin(), pick.end());
    for (int q = 0; q < budgets[i]; ++q) {
      col_idx[row_ptr[i] - base + q] = pick[q];
      coef[row_ptr[i] - base + q] = (float)(v[pick[q]] * inv);
    }
  });
  return 0;
}

int oracle_init_alloc(const float *dWq, int32_t d_out, int32_t d_in, int32_t n, int64_t p,
                      int32_t min_per_row, int32_t mode, int32_t *budgets, int32_t *row_ptr,
                      int32_t *col_idx, float *coef, double *err_norm) {
  if (!shape_ok(d_in, n) || d_out <= 0) return 1;
  std::vector<double> e(d_out);
  if (oracle_init_norms(dWq, d_out, d_in, e.data())) return 1;
  if (err_norm)
    for (int i = 0; i < d_out; ++i) err_norm[i] = e[i];
  if (oracle_init_budgets(e.data(), d_out, d_in, p, min_per_row, mode, budgets, row_ptr)) return 1;
  return oracle_init_select(dWq, d_out, d_in, n, budgets, row_ptr, col_idx, coef);
}

// SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
// generators", 2014): output n >= 1 of the generator seeded with `seed` is the
// finaliser applied to seed + n * 0x9E3779B97F4A7C15 (mod 2^64).
uint64_t splitmix64_output(uint64_t seed, uint64_t n) {
  uint64_t z = seed + n * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Selection over the whole matrix, the alternatives to AdaAlloc that the
// pages compare it with (papernotes.org 消融实验, table 4: random and
// magnitude selection; gist.science 2.2: they may cluster the parameters in
// a few channels). V = dW_Q H (unnormalised, textbook stage order, double);
// flat index j = i * d_in + k.
//   sel 0 (magnitude): the p entries of largest |V|, ties to the lower j;
//   sel 1 (random):    the p entries of smallest u_j = SplitMix64 output
//                      j + 1 for `seed`, ties to the lower j;
// c = float(V * (1/sqrt(n))) at E (the dense solution, as in AdaAlloc).
// Outputs: budgets [d_out] (entries per row), row_ptr [d_out+1], col_idx [p]
// ascending within a row, coef [p].
int oracle_init_select_global(const float *dWq, int32_t d_out, int32_t d_in, int32_t n, int64_t p, int32_t sel,
                              uint64_t seed, int32_t *budgets, int32_t *row_ptr, int32_t *col_idx, float *coef) {
  if (!shape_ok(d_in, n) || d_out <= 0 || (sel != 0 && sel != 1)) return 1;
  const int64_t N = (int64_t)d_out * d_in;
  if (p < 0 || p > N || p > 2147483647LL) return 1;
  std::vector<double> V((size_t)N);
  parallel_for(d_out, [&](int64_t i) {
    double *v = V.data() + i * d_in;
    for (int k = 0; k < d_in; ++k) v[k] = (double)dWq[i * d_in + k];
    for (int blk = 0; blk < d_in / n; ++blk) butterflies(v + (int64_t)blk * n, n);
  });
  std::vector<int64_t> order((size_t)N);
  std::iota(order.begin(), order.end(), (int64_t)0);
  if (sel == 0) {
    std::sort(order.begin(), order.end(), [&](int64_t a, int64_t b) {
      const double fa = std::fabs(V[a]), fb = std::fabs(V[b]);
      return fa > fb || (fa == fb && a < b);
    });
  } else {
    std::vector<uint64_t> u((size_t)N);
    for (int64_t j = 0; j < N; ++j) u[j] = splitmix64_output(seed, (uint64_t)j + 1);
    std::sort(order.begin(), order.end(), [&](int64_t a, int64_t b) { return u[a] < u[b] || (u[a] == u[b] && a < b); });
  }
  std::vector<int64_t> pick(order.begin(), order.begin() + p);
  std::sort(pick.begin(), pick.end());  // row-major order = CSR order with ascending columns
  for (int i = 0; i < d_out; ++i) budgets[i] = 0;
  for (int64_t j : pick) ++budgets[j / d_in];
  row_ptr[0] = 0;
  for (int i = 0; i < d_out; ++i) row_ptr[i + 1] = row_ptr[i] + budgets[i];
  const double inv = inv_sqrt(n);
  for (int64_t q = 0; q < p; ++q) {
    col_idx[q] = (int32_t)(pick[q] % d_in);
    coef[q] = (float)(V[pick[q]] * inv);
  }
  return 0;
}

// Value Refinement [P1 设计3]: the values at E that minimise the layer-output
// error for calibration inputs, instead of the dense solution x0. For channel
// i the page states min_x ||v - x B||^2 with v = dW_Q[i,:] R, B = H^-1 R,
// R R^T = X X^T (the calibration Hessian, called S here), x non-zero only at
// E_i; the closed form itself is lost from the page. Its plain reading, the
// least-squares solution over the selected rows B' of B, is
//   x* = v B'^T (B' B'^T)^-1 = u_i[E_i] (G[E_i, E_i])^-1,
//   G = H S H,  u_i = dW_Q[i,:] S H   (H orthonormal, symmetric, H^-1 = H),
// which equals x0 = (dW_Q H)[i, E_i] when S = I. `damp` adds damp * mean(diag S)
// to the diagonal of S first (0: none). S is [d_in, d_in] (the caller forms
// X^T X from calibration rows X [T, d_in]). Rows `rows` (all when NULL) get
// their coef entries written as float(x*); returns 2 if a system is not
// positive definite.
// Steps in double: A = S H (rows), G^T = (A^T) H (rows of the transpose), and
// per row y = w S, u = y H, then a plain Cholesky factorisation and the two
// triangular solves.
int oracle_refine_values(const float *dWq, int32_t d_out, int32_t d_in, int32_t n, const double *S, double damp,
                         const int32_t *row_ptr, const int32_t *col_idx, int32_t n_rows, const int32_t *rows,
                         float *coef) {
  if (!shape_ok(d_in, n) || d_out <= 0 || damp < 0) return 1;
  const double inv = inv_sqrt(n);
  const size_t D = (size_t)d_in;
  std::vector<double> Sd(S, S + D * D);
  double tr = 0;
  for (size_t k = 0; k < D; ++k) tr += Sd[k * D + k];
  const double lam = damp * tr / (double)d_in;
  for (size_t k = 0; k < D; ++k) Sd[k * D + k] += lam;
  auto transform_rows = [&](std::vector<double> &M) {
    parallel_for(d_in, [&](int64_t r) {
      for (int blk = 0; blk < d_in / n; ++blk) {
        double *x = M.data() + (size_t)r * D + (size_t)blk * n;
        butterflies(x, n);
        for (int k = 0; k < n; ++k) x[k] *= inv;
      }
    });
  };
  auto transpose = [&](const std::vector<double> &M) {
    std::vector<double> T(D * D);
    for (size_t a = 0; a < D; ++a)
      for (size_t b = 0; b < D; ++b) T[b * D + a] = M[a * D + b];
    return T;
  };
  std::vector<double> A = Sd;
  transform_rows(A);                // A = S H
  std::vector<double> Gt = transpose(A);
  transform_rows(Gt);               // Gt = A^T H = (H A)^T = G^T
  std::vector<int32_t> all;
  if (!rows) {
    all.resize(d_out);
    std::iota(all.begin(), all.end(), 0);
    rows = all.data();
    n_rows = d_out;
  }
  int status = 0;
  std::mutex mu;
  parallel_for(n_rows, [&](int64_t q) {
    const int i = rows[q];
    if (i < 0 || i >= d_out) return;
    std::vector<double> y(D, 0.0);
    for (size_t a = 0; a < D; ++a) {
      const double w = (double)dWq[(size_t)i * D + a];
      const double *srow = Sd.data() + a * D;
      for (size_t b = 0; b < D; ++b) y[b] += w * srow[b];
    }
    for (int blk = 0; blk < d_in / n; ++blk) {
      double *x = y.data() + (size_t)blk * n;
      butterflies(x, n);
      for (int k = 0; k < n; ++k) x[k] *= inv;
    }
    const int b0 = row_ptr[i], m = row_ptr[i + 1] - row_ptr[i];
    if (m <= 0) return;
    std::vector<double> L((size_t)m * m), z(m);
    for (int r = 0; r < m; ++r)
      for (int c = 0; c <= r; ++c)  // G[E_r][E_c] = Gt[E_c][E_r]
        L[(size_t)r * m + c] = Gt[(size_t)col_idx[b0 + c] * D + col_idx[b0 + r]];
    for (int j = 0; j < m; ++j) {  // Cholesky, lower triangle in place
      double d = L[(size_t)j * m + j];
      for (int k = 0; k < j; ++k) d -= L[(size_t)j * m + k] * L[(size_t)j * m + k];
      if (!(d > 0)) {
        std::lock_guard<std::mutex> g(mu);
        status = 2;
        return;
      }
      d = std::sqrt(d);
      L[(size_t)j * m + j] = d;
      for (int r = j + 1; r < m; ++r) {
        double v = L[(size_t)r * m + j];
        for (int k = 0; k < j; ++k) v -= L[(size_t)r * m + k] * L[(size_t)j * m + k];
        L[(size_t)r * m + j] = v / d;
      }
    }
    for (int r = 0; r < m; ++r) {  // L z = u[E]
      double v = y[col_idx[b0 + r]];
      for (int k = 0; k < r; ++k) v -= L[(size_t)r * m + k] * z[k];
      z[r] = v / L[(size_t)r * m + r];
    }
    for (int r = m - 1; r >= 0; --r) {  // L^T x = z
      double v = z[r];
      for (int k = r + 1; k < m; ++k) v -= L[(size_t)k * m + r] * z[k];
      z[r] = v / L[(size_t)r * m + r];
    }
    for (int r = 0; r < m; ++r) coef[b0 + r] = (float)z[r];
  });
  return status;
}

// Diagnostics of the selection (the pages' argument for AdaAlloc).
//
// [P1 设计1]: F = Scatter(c, E) is full rank with high probability once every
// row and every column holds more than two nonzeros on average, and rank(dW) =
// rank(F) because H is orthogonal. [P1 设计2; P2 2.2]: choosing E by magnitude
// over the whole matrix crowds the parameters into the few channels that hold
// outliers, and F degenerates to low rank. A row or a column of F without any
// entry cannot add to the rank, so rank(F) <= min(non-empty rows, non-empty
// columns); the numerical rank itself is computed in the Python wrapper.
// stats (8 entries):
//   [0] rows without entries        [1] columns without entries
//   [2] fewest entries in a row     [3] most entries in a row
//   [4] fewest entries in a column  [5] most entries in a column
//   [6] min(d_out - [0], d_in - [1])
//   [7] the fewest rows that together hold at least ceil(p / 2) entries
// col_counts [d_in] receives the entries of every column.
int oracle_pattern_stats(int32_t d_out, int32_t d_in, int64_t p, const int32_t *row_ptr, const int32_t *col_idx,
                         int32_t *col_counts, int64_t *stats) {
  if (d_out <= 0 || d_in <= 0 || p < 0 || row_ptr[0] != 0 || row_ptr[d_out] != p) return 1;
  std::vector<int64_t> rows((size_t)d_out);
  for (int i = 0; i < d_out; ++i) {
    rows[i] = (int64_t)row_ptr[i + 1] - row_ptr[i];
    if (rows[i] < 0) return 1;
  }
  for (int k = 0; k < d_in; ++k) col_counts[k] = 0;
  for (int64_t j = 0; j < p; ++j) {
    if (col_idx[j] < 0 || col_idx[j] >= d_in) return 1;
    col_counts[col_idx[j]]++;
  }
  int64_t empty_r = 0, empty_c = 0;
  for (int i = 0; i < d_out; ++i) empty_r += rows[i] == 0;
  for (int k = 0; k < d_in; ++k) empty_c += col_counts[k] == 0;
  stats[0] = empty_r;
  stats[1] = empty_c;
  stats[2] = *std::min_element(rows.begin(), rows.end());
  stats[3] = *std::max_element(rows.begin(), rows.end());
  stats[4] = *std::min_element(col_counts, col_counts + d_in);
  stats[5] = *std::max_element(col_counts, col_counts + d_in);
  stats[6] = std::min<int64_t>(d_out - empty_r, d_in - empty_c);
  // the most crowded rows first: how many are needed to reach half the entries
  std::vector<int64_t> sorted = rows;
  std::sort(sorted.begin(), sorted.end(), [](int64_t a, int64_t b) { return a > b; });
  const int64_t half = (p + 1) / 2;
  int64_t taken = 0, m = 0;
  while (taken < half) taken += sorted[(size_t)m++];
  stats[7] = m;
  return 0;
}

// Energy concentration of the transform coefficients [P1 设计1, "why the
// WHT"]: the magnitudes of the coefficients of dW_Q after the transform are
// fitted with a Pareto law, whose Hill exponent eta measures how steep the
// tail is (the smaller eta, the more of the error energy sits in few
// coefficients); with the same number of parameters the transform with the
// smallest eta reconstructs the most error energy (the cumulative-energy
// curve). Reading taken (the pages give no formula): a = |V| over all
// d_out * d_in coefficients, V = dW_Q H_unnormalised (fp64 butterflies, as
// in AdaAlloc), sorted a_(1) >= a_(2) >= ...; Hill's estimate over the k
// largest is
//   xi = (1/k) sum_{i=1..k} ln(a_(i) / a_(k+1)),   eta = 1 / xi
// (eta is the Pareto tail index; NaN when a_(k+1) = 0 or xi = 0), and the
// cumulative energy at k is sum_{i<=k} a_(i)^2 / sum_all a^2 (NaN for an
// all-zero dW_Q). Both are scale-free, so the normalisation of H does not
// enter. out: [0] eta, [1] energy fraction of the k largest, [2] a_(k+1),
// [3] sum of all a^2. Requires 1 <= k < d_out * d_in.
int oracle_energy_stats(const float *dWq, int32_t d_out, int32_t d_in, int32_t n, int64_t k, double *out) {
  if (!shape_ok(d_in, n) || d_out <= 0) return 1;
  const int64_t N = (int64_t)d_out * d_in;
  if (k < 1 || k >= N) return 1;
  std::vector<double> a((size_t)N);
  parallel_for(d_out, [&](int64_t i) {
    double *v = a.data() + i * d_in;
    for (int c = 0; c < d_in; ++c) v[c] = (double)dWq[i * d_in + c];
    for (int blk = 0; blk < d_in / n; ++blk) butterflies(v + (int64_t)blk * n, n);
    for (int c = 0; c < d_in; ++c) v[c] = std::fabs(v[c]);
  });
  std::sort(a.begin(), a.end(), [](double x, double y) { return x > y; });
  const double thr = a[(size_t)k];  // a_(k+1), zero-based
  double hill = 0.0, top = 0.0, all = 0.0;
  for (int64_t i = 0; i < k; ++i) {
    hill += std::log(a[(size_t)i] / thr);
    top += a[(size_t)i] * a[(size_t)i];
  }
  for (int64_t i = 0; i < N; ++i) all += a[(size_t)i] * a[(size_t)i];
  const double xi = hill / (double)k;
  out[0] = (thr > 0.0 && xi > 0.0) ? 1.0 / xi : NAN;
  out[1] = all > 0.0 ? top / all : NAN;
  out[2] = thr;
  out[3] = all;
  return 0;
}

// Column view of the CSR pattern: for every column k the nonzeros j with
// col_idx[j] == k, in increasing j: col_ptr [d_in+1], row_idx [p] (their rows),
// perm [p] (their CSR positions).
int oracle_plan_build(int32_t d_out, int32_t d_in, int64_t p, const int32_t *row_ptr,
                      const int32_t *col_idx, int32_t *col_ptr, int32_t *row_idx, int32_t *perm) {
  if (d_out <= 0 || d_in <= 0 || p < 0 || row_ptr[d_out] != p) return 1;
  for (int k = 0; k <= d_in; ++k) col_ptr[k] = 0;
  for (int64_t j = 0; j < p; ++j) {
    if (col_idx[j] < 0 || col_idx[j] >= d_in) return 1;
    col_ptr[col_idx[j] + 1]++;
  }
  for (int k = 0; k < d_in; ++k) col_ptr[k + 1] += col_ptr[k];
  std::vector<int32_t> next(col_ptr, col_ptr + d_in);
  for (int r = 0; r < d_out; ++r)
    for (int32_t j = row_ptr[r]; j < row_ptr[r + 1]; ++j) {
      int32_t pos = next[col_idx[j]]++;
      row_idx[pos] = r;
      perm[pos] = j;
    }
  return 0;
}

}  // extern "C"
