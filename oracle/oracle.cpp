// oracle.cpp - plain fp64 CPU oracle of the tensor-parallel layer pair.
//
// TEST INFRASTRUCTURE ONLY: only tests/, __graft_entry__.smoke() and the CPU
// legs of bench.py load it (through oracle/__init__.py).  It shares no code
// with the CUDA library; the two meet only in the seeded input generator.
//
// What it computes (Diffusers documentation, page "Tensor parallelism",
// Portuguese "main" and Chinese v0.43.0 editions, which state the same facts;
// page "Context parallelism" for the Ring / Ulysses pieces at the end):
//   * opening paragraph: each device holds a colwise or rowwise slice of a
//     layer's weight and computes a partial result, combined at the layer
//     boundary (by the AllReduce of a colwise -> rowwise pair);
//   * section "Colwise and rowwise", style table: colwise shards the output
//     features (weight dim 0), rowwise the input features (weight dim 1); the
//     paragraph under the table: the colwise output stays sharded, the
//     rowwise projection consumes it, a single AllReduce rebuilds the result;
//     colwise Q/K/V give each rank a subset of the heads;
//   * section "Fused projections": a packed Linear is sharded block by block
//     (fused Q/K/V: blocks [1, 1, 1]; SwiGLU gate/up: [1, 1]);
//   * section "Constraints and validation": the degree divides the head
//     count and every packed block; sharded output == single-device output.
// Sharding only moves the arithmetic, so each sharded layer reaches exactly
// (up to rounding order) the unsharded one; every function below is the plain
// definition written out in fp64, loops in the order the definitions give:
//   Y[i][j] = sum_{k ascending} X[i][k] * W[j][k] (+ b[j])   (nn.Linear),
//   GELU(x) = 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))  (Hendrycks &
//   Gimpel 2016, the tanh form), SiLU(x) = x / (1 + exp(-x)) (Elfwing et al.
//   2018), softmax two-pass (row max subtracted, exp, divided by the sum),
//   sums over shards in ascending shard order, the rowwise bias added once.
// Readings where the pages are silent are stated where used.
//
// Performance without changing any result: OpenMP runs over output rows (the
// linear map over blocks of output rows and columns, each weight row read
// once per 64 rows).  Every output element is still the same k-ascending sum.
// Built with -ffp-contract=fast, so each multiply-add step may be one fused
// operation; that rounds once per step instead of twice (fp64 either way).
//
// Every entry point returns 0 or a status (negative values name the failed
// constraint, see kStatus below); it writes only its output arrays.
#include <omp.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

constexpr int64_t kHeadDim = 128;

enum Status : int {
  kOk = 0,
  kBadDegree = -1,        // tp_degree < 1
  kBadRank = -2,          // rank outside [0, tp_degree)
  kIndivisible = -3,      // a sharded dimension (or packed block) % tp_degree != 0
  kHeadsIndivisible = -4, // heads % tp_degree != 0
  kBadHidden = -5,        // D != heads * 128
  kBadBlocks = -6,        // packed blocks: empty, a block < 1, or their sum not dividing the dimension
  kBadShape = -7,         // a size that does not fit (W_qkv rows != 3 D, ...)
};

int check_degree(int T, int rank) {
  if (T < 1) return kBadDegree;
  if (rank >= T || rank < -1) return kBadRank;  // rank -1: no rank given
  return kOk;
}

int check_heads(int64_t D, int heads, int T) {
  if (heads < 1 || heads % T != 0) return kHeadsIndivisible;
  if (D != heads * kHeadDim) return kBadHidden;
  return kOk;
}

// ---------------------------------------------------------------------------
// Shard slicing: index arithmetic on elements of `es` bytes (any dtype).
// ---------------------------------------------------------------------------

// colwise (style table: weight dim 0): rows [r*N/T, (r+1)*N/T) of W[N x K].
int slice_colwise(const uint8_t* W, int64_t rows, int64_t cols, int64_t es, int T, int r, uint8_t* out) {
  if (int s = check_degree(T, r)) return s;
  if (r < 0) return kBadRank;
  if (rows % T != 0) return kIndivisible;
  const int64_t step = rows / T;
  std::memcpy(out, W + r * step * cols * es, size_t(step * cols * es));
  return kOk;
}

// rowwise (style table: weight dim 1): columns [r*K/T, (r+1)*K/T) of every row.
int slice_rowwise(const uint8_t* W, int64_t rows, int64_t cols, int64_t es, int T, int r, uint8_t* out) {
  if (int s = check_degree(T, r)) return s;
  if (r < 0) return kBadRank;
  if (cols % T != 0) return kIndivisible;
  const int64_t step = cols / T;
  for (int64_t i = 0; i < rows; ++i)
    std::memcpy(out + i * step * es, W + (i * cols + r * step) * es, size_t(step * es));
  return kOk;
}

// "Fused projections": proportional blocks whose sum divides the packed
// dimension (absolute sizes, as stored on a Linear, are the case sum == dim);
// every block divisible by the degree on its own ("Constraints and validation").
int packed_block_sizes(int64_t dim, const int64_t* blocks, int nb, int T, int64_t* sizes) {
  if (T < 1) return kBadDegree;
  if (nb < 1) return kBadBlocks;
  int64_t total = 0;
  for (int b = 0; b < nb; ++b) {
    if (blocks[b] < 1) return kBadBlocks;
    total += blocks[b];
  }
  if (dim % total != 0) return kBadBlocks;
  for (int b = 0; b < nb; ++b) {
    sizes[b] = blocks[b] * (dim / total);
    if (sizes[b] % T != 0) return kIndivisible;
  }
  return kOk;
}

// Packed colwise: each block of dim 0 sliced colwise on its own, the slices
// stacked in block order.
int slice_packed_colwise(const uint8_t* W, int64_t rows, int64_t cols, int64_t es, const int64_t* blocks, int nb,
                         int T, int r, uint8_t* out) {
  if (int s = check_degree(T, r)) return s;
  std::vector<int64_t> sizes(size_t(std::max(nb, 1)));
  if (int s = packed_block_sizes(rows, blocks, nb, T, sizes.data())) return s;
  int64_t start = 0, off = 0;
  for (int b = 0; b < nb; ++b) {
    if (int s = slice_colwise(W + start * cols * es, sizes[b], cols, es, T, r, out + off * cols * es)) return s;
    start += sizes[b];
    off += sizes[b] / T;
  }
  return kOk;
}

// Packed rowwise: each block of dim 1 sliced rowwise on its own, the slices
// concatenated along dim 1 in block order.
int slice_packed_rowwise(const uint8_t* W, int64_t rows, int64_t cols, int64_t es, const int64_t* blocks, int nb,
                         int T, int r, uint8_t* out) {
  if (int s = check_degree(T, r)) return s;
  if (r < 0) return kBadRank;
  std::vector<int64_t> sizes(size_t(std::max(nb, 1)));
  if (int s = packed_block_sizes(cols, blocks, nb, T, sizes.data())) return s;
  const int64_t out_cols = cols / T;
  for (int64_t i = 0; i < rows; ++i) {
    int64_t start = 0, off = 0;
    for (int b = 0; b < nb; ++b) {
      const int64_t q = sizes[b] / T;
      std::memcpy(out + (i * out_cols + off) * es, W + (i * cols + start + r * q) * es, size_t(q * es));
      start += sizes[b];
      off += q;
    }
  }
  return kOk;
}

// Head split of a fused [Q; K; V] weight (D rows each, head h at rows h*128..
// inside each block): packed colwise with blocks [1, 1, 1], shard r =
// [Q_r; K_r; V_r].
int slice_qkv_heads(const uint8_t* W, int64_t rows, int64_t D, int64_t es, int heads, int T, int r, uint8_t* out) {
  if (int s = check_degree(T, r)) return s;
  if (int s = check_heads(D, heads, T)) return s;
  if (rows != 3 * D) return kBadShape;
  const int64_t blocks[3] = {1, 1, 1};
  return slice_packed_colwise(W, rows, D, es, blocks, 3, T, r, out);
}

// ---------------------------------------------------------------------------
// Dense pieces.
// ---------------------------------------------------------------------------

// nn.Linear: Y[i][j] = sum_{k = 0..K-1} X[i][k] * W[j][k] (+ b[j]), W [N x K].
// Each Y[i][j] is accumulated from 0 over k in ascending order, then the bias
// is added.  Loop order only: X is first copied into groups of 8 rows stored
// k-major ([M/8][K][8]), and the output is cut into 64-row x 256-column tasks
// that run 8 rows against 4 weight rows at a time, so 32 independent sums
// advance together and each weight row is read once per 64 rows.
void linear(const double* X, int64_t M, int64_t K, const double* W, int64_t N, const double* b, double* Y) {
  constexpr int64_t R = 8, J = 4, RB = 64, JB = 256;
  const int64_t n_g = (M + R - 1) / R;
  std::vector<double> xg(size_t(n_g * K * R));
#pragma omp parallel for schedule(static)
  for (int64_t g = 0; g < n_g; ++g)
    for (int64_t k = 0; k < K; ++k)
      for (int64_t r = 0; r < R; ++r)
        xg[size_t((g * K + k) * R + r)] = g * R + r < M ? X[(g * R + r) * K + k] : 0.0;
  const int64_t n_ib = (M + RB - 1) / RB, n_jb = (N + JB - 1) / JB;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t task = 0; task < n_ib * n_jb; ++task) {
    const int64_t ib = task / n_jb, jb = task % n_jb;
    const int64_t j_end = std::min(N, (jb + 1) * JB), g_end = std::min(n_g, (ib + 1) * (RB / R));
    for (int64_t j0 = jb * JB; j0 < j_end; j0 += J) {
      const int64_t nj = std::min(J, j_end - j0);
      const double* w[J];
      for (int64_t q = 0; q < J; ++q) w[q] = W + (j0 + (q < nj ? q : 0)) * K;
      for (int64_t g = ib * (RB / R); g < g_end; ++g) {
        const double* xk = &xg[size_t(g * K * R)];
        double acc[J][R] = {};
        for (int64_t k = 0; k < K; ++k) {
          const double* x = xk + k * R;
          for (int64_t q = 0; q < J; ++q) {
            const double wk = w[q][k];
            for (int64_t r = 0; r < R; ++r) acc[q][r] += x[r] * wk;
          }
        }
        const int64_t nr = std::min(R, M - g * R);
        for (int64_t q = 0; q < nj; ++q)
          for (int64_t r = 0; r < nr; ++r) Y[(g * R + r) * N + j0 + q] = b ? acc[q][r] + b[j0 + q] : acc[q][r];
      }
    }
  }
}

double gelu_tanh1(double x) {
  const double c = std::sqrt(2.0 / M_PI);
  return 0.5 * x * (1.0 + std::tanh(c * (x + 0.044715 * x * x * x)));
}

double silu1(double x) { return x / (1.0 + std::exp(-x)); }

// act: 0 identity, 1 tanh-form GELU.
void apply_act(double* x, int64_t n, int act) {
  if (act == 0) return;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) x[i] = gelu_tanh1(x[i]);
}

// Two-pass softmax over each row of S [rows x cols]: subtract the row max,
// exponentiate, divide by the row sum.
void softmax_rows(const double* S, int64_t rows, int64_t cols, double* P) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < rows; ++i) {
    const double* s = S + i * cols;
    double* p = P + i * cols;
    double m = -INFINITY;
    for (int64_t j = 0; j < cols; ++j) m = std::max(m, s[j]);
    double l = 0.0;
    for (int64_t j = 0; j < cols; ++j) {
      p[j] = std::exp(s[j] - m);
      l += p[j];
    }
    for (int64_t j = 0; j < cols; ++j) p[j] /= l;
  }
}

// One head: O = softmax(Q K^T * scale) V for Q [Mq x d], K and V [Mk x d]
// given as column blocks (row strides ldq, ldk, ldv, ldo).  Also returns, if
// lse != nullptr, each row's log-sum-exp of the scaled scores
// (log sum_j exp(s_j * scale)), the statistic that the Ring merge combines.
// Query rows go in chunks to bound the score matrix's memory.
void sdpa_head(const double* Q, int64_t ldq, int64_t Mq, const double* K, int64_t ldk, const double* V, int64_t ldv,
               int64_t Mk, int64_t d, double scale, double* O, int64_t ldo, double* lse) {
  std::vector<double> k(size_t(Mk * d)), vt(size_t(d * Mk));
  for (int64_t j = 0; j < Mk; ++j)
    for (int64_t c = 0; c < d; ++c) {
      k[size_t(j * d + c)] = K[j * ldk + c];
      vt[size_t(c * Mk + j)] = V[j * ldv + c];
    }
  const int64_t chunk = 256;
  std::vector<double> q(size_t(chunk * d)), S(size_t(chunk * Mk)), o(size_t(chunk * d));
  for (int64_t i0 = 0; i0 < Mq; i0 += chunk) {
    const int64_t n = std::min(chunk, Mq - i0);
    for (int64_t i = 0; i < n; ++i)
      for (int64_t c = 0; c < d; ++c) q[size_t(i * d + c)] = Q[(i0 + i) * ldq + c];
    linear(q.data(), n, d, k.data(), Mk, nullptr, S.data());  // S = Q K^T
    for (int64_t t = 0; t < n * Mk; ++t) S[size_t(t)] *= scale;
    if (lse) {
      for (int64_t i = 0; i < n; ++i) {
        const double* s = &S[size_t(i * Mk)];
        double m = -INFINITY, l = 0.0;
        for (int64_t j = 0; j < Mk; ++j) m = std::max(m, s[j]);
        for (int64_t j = 0; j < Mk; ++j) l += std::exp(s[j] - m);
        lse[i0 + i] = m + std::log(l);
      }
    }
    softmax_rows(S.data(), n, Mk, S.data());
    linear(S.data(), n, Mk, vt.data(), d, nullptr, o.data());  // O = P V: sum over keys in ascending order
    for (int64_t i = 0; i < n; ++i)
      for (int64_t c = 0; c < d; ++c) O[(i0 + i) * ldo + c] = o[size_t(i * d + c)];
  }
}

// Per-head SDPA over column blocks of width 128: O = concat_h O_h.
void heads_attention(const double* Qs, int64_t ldq, int64_t Mq, const double* Ks, int64_t ldk, const double* Vs,
                     int64_t ldv, int64_t Mk, int n_heads, double* O, int64_t ldo) {
  const double scale = 1.0 / std::sqrt(double(kHeadDim));
  for (int h = 0; h < n_heads; ++h)
    sdpa_head(Qs + h * kHeadDim, ldq, Mq, Ks + h * kHeadDim, ldk, Vs + h * kHeadDim, ldv, Mk, kHeadDim, scale,
              O + h * kHeadDim, ldo, nullptr);
}

// sum_r parts[r] (r ascending) + bias once: the per-element meaning of the
// AllReduce at the block boundary.
void reduce_partials(const double* parts, int T, int64_t M, int64_t N, const double* bias, double* Y) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < M; ++i)
    for (int64_t j = 0; j < N; ++j) {
      double acc = 0.0;
      for (int r = 0; r < T; ++r) acc += parts[(int64_t(r) * M + i) * N + j];
      Y[i * N + j] = bias ? acc + bias[j] : acc;
    }
}

std::vector<double> colwise_slice_f64(const double* W, int64_t rows, int64_t cols, int T, int r) {
  std::vector<double> out(size_t(rows / T * cols));
  slice_colwise(reinterpret_cast<const uint8_t*>(W), rows, cols, 8, T, r, reinterpret_cast<uint8_t*>(out.data()));
  return out;
}

std::vector<double> rowwise_slice_f64(const double* W, int64_t rows, int64_t cols, int T, int r) {
  std::vector<double> out(size_t(rows * (cols / T)));
  slice_rowwise(reinterpret_cast<const uint8_t*>(W), rows, cols, 8, T, r, reinterpret_cast<uint8_t*>(out.data()));
  return out;
}

std::vector<double> qkv_slice_f64(const double* W, int64_t D, int heads, int T, int r) {
  std::vector<double> out(size_t(3 * (D / T) * D));
  slice_qkv_heads(reinterpret_cast<const uint8_t*>(W), 3 * D, D, 8, heads, T, r,
                  reinterpret_cast<uint8_t*>(out.data()));
  return out;
}

// ---------------------------------------------------------------------------
// MLP pair: colwise FFN-in (+ bias, activation) -> rowwise FFN-out (+ bias once).
// ---------------------------------------------------------------------------

// H_r = act(X W_up,r^T + b_up,r): shard r's slice of the hidden activations.
int mlp_colwise_shard(const double* X, int64_t M, int64_t D, const double* W_up, const double* b_up, int64_t F,
                      int T, int r, int act, double* H) {
  if (int s = check_degree(T, r)) return s;
  if (r < 0) return kBadRank;
  if (F % T != 0) return kIndivisible;
  const auto w = colwise_slice_f64(W_up, F, D, T, r);
  std::vector<double> b;
  if (b_up) b = colwise_slice_f64(b_up, F, 1, T, r);
  linear(X, M, D, w.data(), F / T, b_up ? b.data() : nullptr, H);
  apply_act(H, M * (F / T), act);
  return kOk;
}

// Part_r = H_r W_down,r^T: shard r's partial sum of the FFN output (no bias).
int mlp_rowwise_partial(const double* H, int64_t M, const double* W_down, int64_t D, int64_t F, int T, int r,
                        double* P) {
  if (int s = check_degree(T, r)) return s;
  if (r < 0) return kBadRank;
  if (F % T != 0) return kIndivisible;
  const auto w = rowwise_slice_f64(W_down, D, F, T, r);
  linear(H, M, F / T, w.data(), D, nullptr, P);
  return kOk;
}

int mlp_sharded_summed(const double* X, int64_t M, int64_t D, const double* W_up, const double* b_up, int64_t F,
                       const double* W_down, const double* b_down, int T, int act, double* Y) {
  if (int s = check_degree(T, -1)) return s;
  if (F % T != 0) return kIndivisible;
  std::vector<double> parts(size_t(T * M * D)), H(size_t(M * (F / T)));
  for (int r = 0; r < T; ++r) {
    mlp_colwise_shard(X, M, D, W_up, b_up, F, T, r, act, H.data());
    mlp_rowwise_partial(H.data(), M, W_down, D, F, T, r, &parts[size_t(r * M * D)]);
  }
  reduce_partials(parts.data(), T, M, D, b_down, Y);
  return kOk;
}

int mlp_unsharded(const double* X, int64_t M, int64_t D, const double* W_up, const double* b_up, int64_t F,
                  const double* W_down, const double* b_down, int act, double* Y) {
  std::vector<double> H(size_t(M * F));
  linear(X, M, D, W_up, F, b_up, H.data());
  apply_act(H.data(), M * F, act);
  linear(H.data(), M, F, W_down, D, b_down, Y);
  return kOk;
}

// ---------------------------------------------------------------------------
// SwiGLU pair ("Fused projections": gate/up packed [1, 1]).  Reading: W_in =
// [W_gate; W_up], H = silu(gate) * up (Shazeer 2020), then rowwise W_out.
// ---------------------------------------------------------------------------
void swiglu_hidden(const double* X, int64_t M, int64_t D, const double* Wg, const double* Wu, const double* bg,
                   const double* bu, int64_t Fr, double* H) {
  std::vector<double> G(size_t(M * Fr)), U(size_t(M * Fr));
  linear(X, M, D, Wg, Fr, bg, G.data());
  linear(X, M, D, Wu, Fr, bu, U.data());
  for (int64_t t = 0; t < M * Fr; ++t) H[t] = silu1(G[size_t(t)]) * U[size_t(t)];
}

int swiglu_unsharded(const double* X, int64_t M, int64_t D, const double* W_in, const double* b_in, int64_t F,
                     const double* W_out, const double* b_out, double* Y) {
  std::vector<double> H(size_t(M * F));
  swiglu_hidden(X, M, D, W_in, W_in + F * D, b_in, b_in ? b_in + F : nullptr, F, H.data());
  linear(H.data(), M, F, W_out, D, b_out, Y);
  return kOk;
}

int swiglu_sharded_summed(const double* X, int64_t M, int64_t D, const double* W_in, const double* b_in, int64_t F,
                          const double* W_out, const double* b_out, int T, double* Y) {
  if (int s = check_degree(T, -1)) return s;
  if (F % T != 0) return kIndivisible;
  const int64_t Fr = F / T;
  const int64_t halves[2] = {1, 1};
  std::vector<double> parts(size_t(T * M * D)), w(size_t(2 * Fr * D)), b(size_t(2 * Fr)), H(size_t(M * Fr));
  for (int r = 0; r < T; ++r) {
    // [gate_r; up_r] and their biases: packed colwise slices
    slice_packed_colwise(reinterpret_cast<const uint8_t*>(W_in), 2 * F, D, 8, halves, 2, T, r,
                         reinterpret_cast<uint8_t*>(w.data()));
    if (b_in)
      slice_packed_colwise(reinterpret_cast<const uint8_t*>(b_in), 2 * F, 1, 8, halves, 2, T, r,
                           reinterpret_cast<uint8_t*>(b.data()));
    swiglu_hidden(X, M, D, w.data(), w.data() + Fr * D, b_in ? b.data() : nullptr, b_in ? b.data() + Fr : nullptr,
                  Fr, H.data());
    const auto wo = rowwise_slice_f64(W_out, D, F, T, r);
    linear(H.data(), M, Fr, wo.data(), D, nullptr, &parts[size_t(r * M * D)]);
  }
  reduce_partials(parts.data(), T, M, D, b_out, Y);
  return kOk;
}

// rowwise_split_input (style table, third row): the input is replicated and
// each rank takes its own K/T columns of it; partials summed, bias once.
int rowwise_split_input(const double* X, int64_t M, int64_t K, const double* W, int64_t N, const double* b, int T,
                        double* Y) {
  if (int s = check_degree(T, -1)) return s;
  if (K % T != 0) return kIndivisible;
  std::vector<double> parts(size_t(T * M * N));
  for (int r = 0; r < T; ++r) {
    const auto x = rowwise_slice_f64(X, M, K, T, r);
    const auto w = rowwise_slice_f64(W, N, K, T, r);
    linear(x.data(), M, K / T, w.data(), N, nullptr, &parts[size_t(r * M * N)]);
  }
  reduce_partials(parts.data(), T, M, N, b, Y);
  return kOk;
}

// ---------------------------------------------------------------------------
// Attention block: head-split QKV (colwise, packed [1,1,1]) -> per-shard SDPA
// -> rowwise W_o.  softmax(Q K^T / sqrt(128)) V per head, non-causal, no mask,
// no bias (none of these is on the pages; the C ABI takes none).
// ---------------------------------------------------------------------------

// O_r [Mq x D/T] for query rows `rows` (all rows when rows == nullptr):
// shard r's attention output over its H/T heads.
int attn_shard_output_rows(const double* X, int64_t M, int64_t D, const double* W_qkv, int heads, int T, int r,
                           const int64_t* rows, int64_t nrows, double* O_r) {
  if (int s = check_degree(T, r)) return s;
  if (int s = check_heads(D, heads, T)) return s;
  const int64_t Dr = D / T;
  const auto w = qkv_slice_f64(W_qkv, D, heads, T, r);
  const int64_t Mq = rows ? nrows : M;
  std::vector<double> Xq(size_t(Mq * D)), Q(size_t(Mq * Dr)), KV(size_t(M * 2 * Dr));
  for (int64_t i = 0; i < Mq; ++i) std::memcpy(&Xq[size_t(i * D)], X + (rows ? rows[i] : i) * D, size_t(D) * 8);
  linear(Xq.data(), Mq, D, w.data(), Dr, nullptr, Q.data());          // Q_r
  linear(X, M, D, w.data() + Dr * D, 2 * Dr, nullptr, KV.data());     // [K_r V_r] of every token
  heads_attention(Q.data(), Dr, Mq, KV.data(), 2 * Dr, KV.data() + Dr, 2 * Dr, M, heads / T, O_r, Dr);
  return kOk;
}

int attn_rows(const double* X, int64_t M, int64_t D, const double* W_qkv, const double* W_o, int heads,
              const int64_t* rows, int64_t nrows, int T, double* Y) {
  if (int s = check_degree(T, -1)) return s;
  if (int s = check_heads(D, heads, T)) return s;
  const int64_t Dr = D / T, Mq = rows ? nrows : M;
  std::vector<double> parts(size_t(T * Mq * D)), O(size_t(Mq * Dr));
  for (int r = 0; r < T; ++r) {
    attn_shard_output_rows(X, M, D, W_qkv, heads, T, r, rows, nrows, O.data());
    const auto wo = rowwise_slice_f64(W_o, D, D, T, r);
    linear(O.data(), Mq, Dr, wo.data(), D, nullptr, &parts[size_t(r * Mq * D)]);
  }
  reduce_partials(parts.data(), T, Mq, D, nullptr, Y);
  return kOk;
}

int attn_unsharded(const double* X, int64_t M, int64_t D, const double* W_qkv, const double* W_o, int heads,
                   double* Y) {
  if (int s = check_heads(D, heads, 1)) return s;
  std::vector<double> QKV(size_t(M * 3 * D)), O(size_t(M * D));
  linear(X, M, D, W_qkv, 3 * D, nullptr, QKV.data());
  heads_attention(QKV.data(), 3 * D, M, QKV.data() + D, 3 * D, QKV.data() + 2 * D, 3 * D, M, heads, O.data(), D);
  linear(O.data(), M, D, W_o, D, nullptr, Y);
  return kOk;
}

// ---------------------------------------------------------------------------
// Dual-stream joint attention (the page's note that the encoder stream's
// add_q_proj / to_add_out / ff_context follow the image stream's pattern):
// both streams sharded alike, Q/K/V concatenated along tokens (image first),
// attended jointly, each stream's rows through its own out-projection.
// ---------------------------------------------------------------------------
int joint_attn_rows(const double* Xi, int64_t Mi, const double* Xt, int64_t Mt, int64_t D, const double* Wqi,
                    const double* Wqt, const double* Woi, const double* Wot, int heads, const int64_t* ri, int64_t ni,
                    const int64_t* rt, int64_t nt, int T, double* Yi, double* Yt) {
  if (int s = check_degree(T, -1)) return s;
  if (int s = check_heads(D, heads, T)) return s;
  const int64_t Dr = D / T, M = Mi + Mt, Nq = ni + nt;
  std::vector<double> parts_i(size_t(T * ni * D)), parts_t(size_t(T * nt * D));
  for (int r = 0; r < T; ++r) {
    const auto wi = qkv_slice_f64(Wqi, D, heads, T, r), wt = qkv_slice_f64(Wqt, D, heads, T, r);
    std::vector<double> Q(size_t(Nq * Dr)), KV(size_t(M * 2 * Dr)), xq(size_t(std::max<int64_t>(Nq, 1) * D));
    for (int64_t i = 0; i < ni; ++i) std::memcpy(&xq[size_t(i * D)], Xi + ri[i] * D, size_t(D) * 8);
    for (int64_t i = 0; i < nt; ++i) std::memcpy(&xq[size_t((ni + i) * D)], Xt + rt[i] * D, size_t(D) * 8);
    linear(xq.data(), ni, D, wi.data(), Dr, nullptr, Q.data());
    linear(xq.data() + ni * D, nt, D, wt.data(), Dr, nullptr, Q.data() + ni * Dr);
    linear(Xi, Mi, D, wi.data() + Dr * D, 2 * Dr, nullptr, KV.data());
    linear(Xt, Mt, D, wt.data() + Dr * D, 2 * Dr, nullptr, KV.data() + Mi * 2 * Dr);
    std::vector<double> O(size_t(Nq * Dr));
    heads_attention(Q.data(), Dr, Nq, KV.data(), 2 * Dr, KV.data() + Dr, 2 * Dr, M, heads / T, O.data(), Dr);
    const auto woi = rowwise_slice_f64(Woi, D, D, T, r), wot = rowwise_slice_f64(Wot, D, D, T, r);
    linear(O.data(), ni, Dr, woi.data(), D, nullptr, &parts_i[size_t(r * ni * D)]);
    linear(O.data() + ni * Dr, nt, Dr, wot.data(), D, nullptr, &parts_t[size_t(r * nt * D)]);
  }
  reduce_partials(parts_i.data(), T, ni, D, nullptr, Yi);
  reduce_partials(parts_t.data(), T, nt, D, nullptr, Yt);
  return kOk;
}

int joint_attn_unsharded(const double* Xi, int64_t Mi, const double* Xt, int64_t Mt, int64_t D, const double* Wqi,
                         const double* Wqt, const double* Woi, const double* Wot, int heads, double* Yi, double* Yt) {
  if (int s = check_heads(D, heads, 1)) return s;
  const int64_t M = Mi + Mt;
  std::vector<double> QKV(size_t(M * 3 * D)), O(size_t(M * D));
  linear(Xi, Mi, D, Wqi, 3 * D, nullptr, QKV.data());
  linear(Xt, Mt, D, Wqt, 3 * D, nullptr, QKV.data() + Mi * 3 * D);
  heads_attention(QKV.data(), 3 * D, M, QKV.data() + D, 3 * D, QKV.data() + 2 * D, 3 * D, M, heads, O.data(), D);
  linear(O.data(), Mi, D, Woi, D, nullptr, Yi);
  linear(O.data() + Mi * D, Mt, D, Wot, D, nullptr, Yt);
  return kOk;
}

// ---------------------------------------------------------------------------
// Context parallelism ("Context parallelism" page).  Ring attention: every
// rank attends its queries to one key/value block after another as the blocks
// travel around the ring, and the per-block results are combined.  A block b
// gives, per query row, O_b (softmax over the block's keys applied to its
// values) and lse_b = log sum_{j in b} exp(s_j); then
//   O = sum_b exp(lse_b - L) O_b / sum_b exp(lse_b - L),  L = max_b lse_b,
//   lse = L + log sum_b exp(lse_b - L),
// which is softmax over all keys applied to all values (each O_b is its
// block's weighted mean, exp(lse_b) its block's total weight).
// O_parts [nparts][M][d], lse_parts [nparts][M] -> O [M][d], lse [M].
// ---------------------------------------------------------------------------
void attn_merge(const double* O_parts, const double* lse_parts, int nparts, int64_t M, int64_t d, double* O,
                double* lse) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < M; ++i) {
    double L = -INFINITY;
    for (int b = 0; b < nparts; ++b) L = std::max(L, lse_parts[b * M + i]);
    double wsum = 0.0;
    for (int64_t c = 0; c < d; ++c) O[i * d + c] = 0.0;
    for (int b = 0; b < nparts; ++b) {
      const double w = std::exp(lse_parts[b * M + i] - L);
      wsum += w;
      for (int64_t c = 0; c < d; ++c) O[i * d + c] += w * O_parts[(b * M + i) * d + c];
    }
    for (int64_t c = 0; c < d; ++c) O[i * d + c] /= wsum;
    if (lse) lse[i] = L + std::log(wsum);
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// C entry points (ctypes).  Arrays are row-major fp64 unless an element size
// is given; outputs are caller-allocated.
// ---------------------------------------------------------------------------
extern "C" {

int oracle_num_threads(void) { return omp_get_max_threads(); }

int oracle_slice_colwise(const void* W, int64_t rows, int64_t cols, int64_t es, int T, int r, void* out) {
  return slice_colwise(static_cast<const uint8_t*>(W), rows, cols, es, T, r, static_cast<uint8_t*>(out));
}
int oracle_slice_rowwise(const void* W, int64_t rows, int64_t cols, int64_t es, int T, int r, void* out) {
  return slice_rowwise(static_cast<const uint8_t*>(W), rows, cols, es, T, r, static_cast<uint8_t*>(out));
}
int oracle_packed_block_sizes(int64_t dim, const int64_t* blocks, int nb, int T, int64_t* sizes) {
  return packed_block_sizes(dim, blocks, nb, T, sizes);
}
int oracle_slice_packed_colwise(const void* W, int64_t rows, int64_t cols, int64_t es, const int64_t* blocks, int nb,
                                int T, int r, void* out) {
  return slice_packed_colwise(static_cast<const uint8_t*>(W), rows, cols, es, blocks, nb, T, r,
                              static_cast<uint8_t*>(out));
}
int oracle_slice_packed_rowwise(const void* W, int64_t rows, int64_t cols, int64_t es, const int64_t* blocks, int nb,
                                int T, int r, void* out) {
  return slice_packed_rowwise(static_cast<const uint8_t*>(W), rows, cols, es, blocks, nb, T, r,
                              static_cast<uint8_t*>(out));
}
int oracle_slice_qkv_heads(const void* W, int64_t rows, int64_t D, int64_t es, int heads, int T, int r, void* out) {
  return slice_qkv_heads(static_cast<const uint8_t*>(W), rows, D, es, heads, T, r, static_cast<uint8_t*>(out));
}
int oracle_check_heads(int64_t D, int heads, int T) {
  if (T < 1) return kBadDegree;
  return check_heads(D, heads, T);
}

int oracle_linear(const double* X, int64_t M, int64_t K, const double* W, int64_t N, const double* b, double* Y) {
  linear(X, M, K, W, N, b, Y);
  return kOk;
}
int oracle_gelu_tanh(const double* x, int64_t n, double* y) {
  for (int64_t i = 0; i < n; ++i) y[i] = gelu_tanh1(x[i]);
  return kOk;
}
int oracle_silu(const double* x, int64_t n, double* y) {
  for (int64_t i = 0; i < n; ++i) y[i] = silu1(x[i]);
  return kOk;
}
int oracle_softmax_rows(const double* S, int64_t rows, int64_t cols, double* P) {
  softmax_rows(S, rows, cols, P);
  return kOk;
}
int oracle_sdpa(const double* Q, int64_t Mq, const double* K, const double* V, int64_t Mk, int64_t d, double scale,
                double* O, double* lse) {
  sdpa_head(Q, d, Mq, K, d, V, d, Mk, d, scale, O, d, lse);
  return kOk;
}
int oracle_attn_merge(const double* O_parts, const double* lse_parts, int nparts, int64_t M, int64_t d, double* O,
                      double* lse) {
  if (nparts < 1) return kBadShape;
  attn_merge(O_parts, lse_parts, nparts, M, d, O, lse);
  return kOk;
}
int oracle_reduce_partials(const double* parts, int T, int64_t M, int64_t N, const double* bias, double* Y) {
  reduce_partials(parts, T, M, N, bias, Y);
  return kOk;
}

int oracle_mlp_colwise_shard(const double* X, int64_t M, int64_t D, const double* W_up, const double* b_up, int64_t F,
                             int T, int r, int act, double* H) {
  return mlp_colwise_shard(X, M, D, W_up, b_up, F, T, r, act, H);
}
int oracle_mlp_rowwise_partial(const double* H, int64_t M, const double* W_down, int64_t D, int64_t F, int T, int r,
                               double* P) {
  return mlp_rowwise_partial(H, M, W_down, D, F, T, r, P);
}
int oracle_mlp_sharded_summed(const double* X, int64_t M, int64_t D, const double* W_up, const double* b_up,
                              int64_t F, const double* W_down, const double* b_down, int T, int act, double* Y) {
  return mlp_sharded_summed(X, M, D, W_up, b_up, F, W_down, b_down, T, act, Y);
}
int oracle_mlp_unsharded(const double* X, int64_t M, int64_t D, const double* W_up, const double* b_up, int64_t F,
                         const double* W_down, const double* b_down, int act, double* Y) {
  return mlp_unsharded(X, M, D, W_up, b_up, F, W_down, b_down, act, Y);
}
int oracle_swiglu_unsharded(const double* X, int64_t M, int64_t D, const double* W_in, const double* b_in, int64_t F,
                            const double* W_out, const double* b_out, double* Y) {
  return swiglu_unsharded(X, M, D, W_in, b_in, F, W_out, b_out, Y);
}
int oracle_swiglu_sharded_summed(const double* X, int64_t M, int64_t D, const double* W_in, const double* b_in,
                                 int64_t F, const double* W_out, const double* b_out, int T, double* Y) {
  return swiglu_sharded_summed(X, M, D, W_in, b_in, F, W_out, b_out, T, Y);
}
int oracle_rowwise_split_input(const double* X, int64_t M, int64_t K, const double* W, int64_t N, const double* b,
                               int T, double* Y) {
  return rowwise_split_input(X, M, K, W, N, b, T, Y);
}
int oracle_attn_unsharded(const double* X, int64_t M, int64_t D, const double* W_qkv, const double* W_o, int heads,
                          double* Y) {
  return attn_unsharded(X, M, D, W_qkv, W_o, heads, Y);
}
int oracle_attn_shard_output(const double* X, int64_t M, int64_t D, const double* W_qkv, int heads, int T, int r,
                             double* O_r) {
  return attn_shard_output_rows(X, M, D, W_qkv, heads, T, r, nullptr, 0, O_r);
}
int oracle_attn_rows(const double* X, int64_t M, int64_t D, const double* W_qkv, const double* W_o, int heads,
                     const int64_t* rows, int64_t nrows, int T, double* Y) {
  return attn_rows(X, M, D, W_qkv, W_o, heads, rows, nrows, T, Y);
}
int oracle_joint_attn_unsharded(const double* Xi, int64_t Mi, const double* Xt, int64_t Mt, int64_t D,
                                const double* Wqi, const double* Wqt, const double* Woi, const double* Wot, int heads,
                                double* Yi, double* Yt) {
  return joint_attn_unsharded(Xi, Mi, Xt, Mt, D, Wqi, Wqt, Woi, Wot, heads, Yi, Yt);
}
int oracle_joint_attn_rows(const double* Xi, int64_t Mi, const double* Xt, int64_t Mt, int64_t D, const double* Wqi,
                           const double* Wqt, const double* Woi, const double* Wot, int heads, const int64_t* ri,
                           int64_t ni, const int64_t* rt, int64_t nt, int T, double* Yi, double* Yt) {
  return joint_attn_rows(Xi, Mi, Xt, Mt, D, Wqi, Wqt, Woi, Wot, heads, ri, ni, rt, nt, T, Yi, Yt);
}

}  // extern "C"
