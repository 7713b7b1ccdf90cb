// rocs_oracle.cpp -- plain fp64 CPU oracle for IKBO-LCB and IKBO-DCA.
//
// TEST INFRASTRUCTURE ONLY.  This oracle is used by the tests, by the smoke check
// and by the CPU-baseline leg of the benchmark.  The CUDA product path never links,
// loads or calls it; it shares no code, header, table or helper with that path.
//
// What it computes follows "ROCS: Request-Oriented Compute Sharing for Efficient
// Large-Scale Recommendation" (arXiv:2607.27744), as read from the paper-archivist
// reading notes of that paper:
//   * LCB: the two-group ROCSified linear compression block, section 3.1.2, Eq. (5)
//     and its explicit two-group form Eq. (6):
//         [Y^R; Y^C] = [[W_RR, 0], [W_CR, W_CC]] . [X^R; X^C]
//     evaluated per candidate with the request-to-candidate broadcast MATERIALISED
//     (each candidate gets a fresh copy of its request's X^R) -- the plain
//     definition; the in-kernel broadcast of section 4 only reorders this sum.
//   * the request-output identity of section 3.1.5, Eq. (11): the request rows of
//     every candidate's full output equal the request output computed once; the
//     oracle checks this exactly on every candidate it evaluates.
//   * DCA: the candidate-group cross attention of section 3.2, Eq. (13),
//         A^C = Attn(Q^C, K, V) = softmax(scale . Q^C K^T) V,
//     non-causal, each candidate's query tokens over its own request's keys, with
//     the K/V broadcast MATERIALISED per candidate (section 4.3 describes the
//     dense implementation that copies K/V to the candidate batch).
//   * the chained block used by the chained workload: LCB -> bf16 -> linear query
//     projection -> bf16 -> DCA (section 3.2, Eq. (12): queries generated from the
//     LCB output; the projection is a plain linear map, no bias, no activation).
//
// Everything accumulates in double, in the index order written in the loops below.
// Inputs are widened to double exactly from their stored fp32 / bf16 bits.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

enum { ORC_OK = 0, ORC_INVALID = 1, ORC_BAD_OFFSETS = 2, ORC_ISOLATION = 10 };

// exact widening of a stored element (dtype 0: fp32, 1: bf16 bit pattern)
inline double widen(const void* base, int dtype, int64_t idx) {
  if (dtype == 0) return (double)static_cast<const float*>(base)[idx];
  uint32_t u = (uint32_t)static_cast<const uint16_t*>(base)[idx] << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

// Round a double to the nearest bf16 value (ties to even), returned as a double.
// bf16 = 8 significant bits, exponent range of binary32 (normal min 2^-126,
// subnormal quantum 2^-133).  Uses frexp + nearbyint (default rounding mode is
// round-half-even), i.e. a single rounding straight from double.
inline double round_bf16(double x) {
  if (!std::isfinite(x) || x == 0.0) return x;
  int e;
  double m = std::frexp(x, &e);  // x = m * 2^e, 0.5 <= |m| < 1
  int q = e - 8;                 // quantum exponent for 8 significant bits
  if (q < -133) q = -133;
  double r = std::nearbyint(std::ldexp(x, -q));
  double v = std::ldexp(r, q);
  if (std::fabs(v) >= std::ldexp(1.0, 128)) v = std::copysign(std::numeric_limits<double>::infinity(), x);
  return v;
}

// CSR check: off[0] == 0, non-decreasing, off[R] == total (total < 0: skip that test).
bool csr_ok(const int32_t* off, int64_t R, int64_t total) {
  if (R < 0 || off == nullptr) return false;
  if (off[0] != 0) return false;
  for (int64_t r = 0; r < R; ++r)
    if (off[r + 1] < off[r]) return false;
  return total < 0 || (int64_t)off[R] == total;
}

// candidate -> request map m, derived by a linear walk over the offsets (section 4.1)
std::vector<int64_t> index_map(const int32_t* off, int64_t R) {
  std::vector<int64_t> m((size_t)off[R]);
  for (int64_t r = 0; r < R; ++r)
    for (int64_t i = off[r]; i < off[r + 1]; ++i) m[(size_t)i] = r;
  return m;
}

// the process default thread count (all host cores unless OMP_NUM_THREADS says otherwise), taken before
// any call changes it
int default_threads() {
#ifdef _OPENMP
  static const int n = omp_get_max_threads();
  return n;
#else
  return 1;
#endif
}

// nthreads > 0: that many OpenMP threads for this call; 0: the process default, also after an earlier call
// asked for fewer
void set_threads(int nthreads) {
#ifdef _OPENMP
  omp_set_num_threads(nthreads > 0 ? nthreads : default_threads());
#else
  (void)nthreads;
#endif
}

// ---- LCB, one candidate: Eq. (6) with the broadcast materialised ------------------------
// y_full [(o_r+o_c) x d] = W_full [(o_r+o_c) x (n_r+n_c)] . X_full [(n_r+n_c) x d]
struct LcbDims {
  int64_t n_r, n_c, d, o_r, o_c;
};

void lcb_full_weight(const LcbDims& D, int dtype, const void* w_rr, const void* w_cr, const void* w_cc,
                     std::vector<double>& W) {
  const int64_t ni = D.n_r + D.n_c, no = D.o_r + D.o_c;
  W.assign((size_t)(no * ni), 0.0);
  for (int64_t o = 0; o < D.o_r; ++o) {
    for (int64_t j = 0; j < D.n_r; ++j) W[(size_t)(o * ni + j)] = widen(w_rr, dtype, o * D.n_r + j);
    for (int64_t j = 0; j < D.n_c; ++j) W[(size_t)(o * ni + D.n_r + j)] = 0.0;  // the masked block M_RC = 0
  }
  for (int64_t o = 0; o < D.o_c; ++o) {
    for (int64_t j = 0; j < D.n_r; ++j) W[(size_t)((D.o_r + o) * ni + j)] = widen(w_cr, dtype, o * D.n_r + j);
    for (int64_t j = 0; j < D.n_c; ++j) W[(size_t)((D.o_r + o) * ni + D.n_r + j)] = widen(w_cc, dtype, o * D.n_c + j);
  }
}

// Y^R_r = W_RR . X^R_r, j ascending
void lcb_request(const LcbDims& D, int dtype, const void* x_req, const std::vector<double>& W, int64_t r,
                 double* y /* [o_r x d] */) {
  const int64_t ni = D.n_r + D.n_c;
  for (int64_t o = 0; o < D.o_r; ++o)
    for (int64_t c = 0; c < D.d; ++c) {
      double acc = 0.0;
      for (int64_t j = 0; j < D.n_r; ++j) acc += W[(size_t)(o * ni + j)] * widen(x_req, dtype, (r * D.n_r + j) * D.d + c);
      y[o * D.d + c] = acc;
    }
}

// Full output of candidate i.  Returns false if the request rows differ from Y^R (Eq. 11).
bool lcb_candidate(const LcbDims& D, int dtype, const void* x_req, const void* x_cand, const std::vector<double>& W,
                   int64_t i, int64_t r, double* y_cand /* [o_c x d] */) {
  const int64_t ni = D.n_r + D.n_c, no = D.o_r + D.o_c;
  // the explicit broadcast: a fresh copy X_full = [X^R_r ; X^C_i]
  std::vector<double> X((size_t)(ni * D.d));
  for (int64_t j = 0; j < D.n_r; ++j)
    for (int64_t c = 0; c < D.d; ++c) X[(size_t)(j * D.d + c)] = widen(x_req, dtype, (r * D.n_r + j) * D.d + c);
  for (int64_t j = 0; j < D.n_c; ++j)
    for (int64_t c = 0; c < D.d; ++c) X[(size_t)((D.n_r + j) * D.d + c)] = widen(x_cand, dtype, (i * D.n_c + j) * D.d + c);
  std::vector<double> Y((size_t)(no * D.d));
  for (int64_t o = 0; o < no; ++o)
    for (int64_t c = 0; c < D.d; ++c) {
      double acc = 0.0;
      for (int64_t j = 0; j < ni; ++j) acc += W[(size_t)(o * ni + j)] * X[(size_t)(j * D.d + c)];
      Y[(size_t)(o * D.d + c)] = acc;
    }
  // Eq. (11): request rows of the full output == Y^R of the request, computed alone
  std::vector<double> yr((size_t)(D.o_r * D.d));
  lcb_request(D, dtype, x_req, W, r, yr.data());
  bool same = true;
  for (int64_t k = 0; k < D.o_r * D.d; ++k) same = same && (Y[(size_t)k] == yr[(size_t)k]);
  for (int64_t o = 0; o < D.o_c; ++o)
    for (int64_t c = 0; c < D.d; ++c) y_cand[o * D.d + c] = Y[(size_t)((D.o_r + o) * D.d + c)];
  return same;
}

// ---- DCA, one candidate: Eq. (13) with the K/V broadcast materialised ------------------
struct DcaDims {
  int64_t q, H, dh;
  double scale;
};

// o [q x H x dh], lse [q x H] for candidate i of request r with keys [s0, s1)
void dca_candidate(const DcaDims& D, const uint16_t* Q, const uint16_t* K, const uint16_t* V, int64_t i, int64_t s0,
                   int64_t s1, const double* q_override /* [q x H x dh] or null */, double* o, double* lse) {
  const int64_t L = s1 - s0, row = D.H * D.dh;
  // the explicit broadcast: fresh per-candidate copies of the request's K and V
  std::vector<double> Ki((size_t)(L * row)), Vi((size_t)(L * row));
  for (int64_t j = 0; j < L; ++j)
    for (int64_t e = 0; e < row; ++e) {
      Ki[(size_t)(j * row + e)] = widen(K, 1, (s0 + j) * row + e);
      Vi[(size_t)(j * row + e)] = widen(V, 1, (s0 + j) * row + e);
    }
  std::vector<double> s((size_t)L), p((size_t)L);
  for (int64_t t = 0; t < D.q; ++t)
    for (int64_t h = 0; h < D.H; ++h) {
      double* out = o + (t * D.H + h) * D.dh;
      if (L == 0) {  // empty key sequence: zero output, LSE = -inf
        for (int64_t c = 0; c < D.dh; ++c) out[c] = 0.0;
        lse[t * D.H + h] = -std::numeric_limits<double>::infinity();
        continue;
      }
      double m = -std::numeric_limits<double>::infinity();
      for (int64_t j = 0; j < L; ++j) {
        double acc = 0.0;
        for (int64_t c = 0; c < D.dh; ++c) {
          const double qv = q_override ? q_override[(t * D.H + h) * D.dh + c]
                                       : widen(Q, 1, ((i * D.q + t) * D.H + h) * D.dh + c);
          acc += qv * Ki[(size_t)(j * row + h * D.dh + c)];
        }
        s[(size_t)j] = D.scale * acc;
        if (s[(size_t)j] > m) m = s[(size_t)j];
      }
      double l = 0.0;
      for (int64_t j = 0; j < L; ++j) {
        p[(size_t)j] = std::exp(s[(size_t)j] - m);
        l += p[(size_t)j];
      }
      for (int64_t c = 0; c < D.dh; ++c) out[c] = 0.0;
      for (int64_t j = 0; j < L; ++j) {
        const double w = p[(size_t)j] / l;
        for (int64_t c = 0; c < D.dh; ++c) out[c] += w * Vi[(size_t)(j * row + h * D.dh + c)];
      }
      lse[t * D.H + h] = m + std::log(l);
    }
}

// ---- LCB block: bias, group-local norm and pointwise epilogue --------------------------
// One output group's epilogue (the fields mirror the ctypes structure in oracle/__init__.py).
//   bias     [o] fp32, per output row, broadcast over d: the GLM linear bias of section 3.1.2,
//            Eq. (4), applied on the row axis of the LCB (null = none)
//   residual bf16 rows of the group's output shape (null = none): a pointwise merge of an
//            aligned input of the same group, section 3.1.3, Eq. (8)
//   norm     0 none, 1 LayerNorm, 2 RMSNorm over the d entries of one output row, with the
//            group's own gamma/beta [d] (null = 1 / 0): the group-local norm of Eq. (7)
//   act      0 none, 1 ReLU, 2 SiLU, 3 GELU (erf form): a pointwise activation, Eq. (8)
// Order on one output row y: y = W x + b; y += residual; y = Norm(y); y = act(y).
struct OrcEpi {
  const float* bias;
  const uint16_t* residual;
  const float* gamma;
  const float* beta;
  double eps;
  int32_t norm;
  int32_t act;
};

double activation(int act, double x) {
  switch (act) {
    case 1: return x > 0.0 ? x : 0.0;
    case 2: return x / (1.0 + std::exp(-x));
    case 3: return 0.5 * x * (1.0 + std::erf(x / std::sqrt(2.0)));
    default: return x;
  }
}

// y [d]: one output row of a group; res_row = index of this row in the group's residual
void epilogue_row(const OrcEpi& e, int64_t d, int64_t res_row, double* y) {
  if (e.residual)
    for (int64_t c = 0; c < d; ++c) y[c] += widen(e.residual, 1, res_row * d + c);
  if (e.norm == 1 || e.norm == 2) {
    double mean = 0.0;
    if (e.norm == 1) {
      for (int64_t c = 0; c < d; ++c) mean += y[c];
      mean /= (double)d;
    }
    double var = 0.0;  // LayerNorm: population variance; RMSNorm: mean square
    for (int64_t c = 0; c < d; ++c) var += (y[c] - mean) * (y[c] - mean);
    var /= (double)d;
    const double inv = 1.0 / std::sqrt(var + e.eps);
    for (int64_t c = 0; c < d; ++c) {
      const double g = e.gamma ? (double)e.gamma[c] : 1.0, b = e.beta ? (double)e.beta[c] : 0.0;
      y[c] = (y[c] - mean) * inv * g + b;
    }
  }
  for (int64_t c = 0; c < d; ++c) y[c] = activation(e.act, y[c]);
}

bool epi_ok(const OrcEpi* e) {
  return e && e->norm >= 0 && e->norm <= 2 && e->act >= 0 && e->act <= 3 && e->eps >= 0.0;
}

// Y^R_r of the block: W_RR X^R_r + b^R, then the request epilogue
void lcb_block_request(const LcbDims& D, const void* x_req, const std::vector<double>& W, const OrcEpi& er,
                       int64_t r, double* y) {
  lcb_request(D, 1, x_req, W, r, y);
  for (int64_t o = 0; o < D.o_r; ++o) {
    double* row = y + o * D.d;
    if (er.bias)
      for (int64_t c = 0; c < D.d; ++c) row[c] += (double)er.bias[o];
    epilogue_row(er, D.d, r * D.o_r + o, row);
  }
}

}  // namespace

extern "C" {

int rocs_oracle_max_threads(void) { return default_threads(); }

// IKBO-LCB oracle.  dtype 0 = fp32 inputs, 1 = bf16 inputs (bit patterns).
// Computes Y^R for the requests listed in sel_req (y_req: [n_sel_req, o_r, d]) and
// Y^C for the candidates listed in sel_cand (y_cand: [n_sel_cand, o_c, d]).
int rocs_oracle_lcb(int64_t R, const int32_t* cand_off, int64_t n_r, int64_t n_c, int64_t d, int64_t o_r, int64_t o_c,
                    int dtype, const void* x_req, const void* x_cand, const void* w_rr, const void* w_cr,
                    const void* w_cc, int64_t n_sel_req, const int64_t* sel_req, double* y_req, int64_t n_sel_cand,
                    const int64_t* sel_cand, double* y_cand, int nthreads) {
  if (n_r < 0 || n_c < 0 || d < 0 || o_r < 0 || o_c < 0 || (dtype != 0 && dtype != 1)) return ORC_INVALID;
  if (!csr_ok(cand_off, R, -1)) return ORC_BAD_OFFSETS;
  set_threads(nthreads);
  const LcbDims D{n_r, n_c, d, o_r, o_c};
  const int64_t C = cand_off[R];
  std::vector<int64_t> m = index_map(cand_off, R);
  std::vector<double> W;
  lcb_full_weight(D, dtype, w_rr, w_cr, w_cc, W);
  for (int64_t k = 0; k < n_sel_req; ++k)
    if (sel_req[k] < 0 || sel_req[k] >= R) return ORC_INVALID;
  for (int64_t k = 0; k < n_sel_cand; ++k)
    if (sel_cand[k] < 0 || sel_cand[k] >= C) return ORC_INVALID;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t k = 0; k < n_sel_req; ++k) lcb_request(D, dtype, x_req, W, sel_req[k], y_req + k * o_r * d);
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t k = 0; k < n_sel_cand; ++k) {
    const int64_t i = sel_cand[k];
    if (!lcb_candidate(D, dtype, x_req, x_cand, W, i, m[(size_t)i], y_cand + k * o_c * d)) bad |= 1;
  }
  return bad ? ORC_ISOLATION : ORC_OK;
}

// IKBO-DCA oracle for the candidates in sel_cand: o [n_sel, q, H, dh], lse [n_sel, q, H].
int rocs_oracle_dca(int64_t R, const int32_t* cand_off, const int32_t* seq_off, int64_t q, int64_t H, int64_t dh,
                    double scale, const uint16_t* Q, const uint16_t* K, const uint16_t* V, int64_t n_sel,
                    const int64_t* sel_cand, double* o, double* lse, int nthreads) {
  if (q < 0 || H < 0 || dh < 0) return ORC_INVALID;
  if (!csr_ok(cand_off, R, -1) || !csr_ok(seq_off, R, -1)) return ORC_BAD_OFFSETS;
  set_threads(nthreads);
  const int64_t C = cand_off[R];
  for (int64_t k = 0; k < n_sel; ++k)
    if (sel_cand[k] < 0 || sel_cand[k] >= C) return ORC_INVALID;
  std::vector<int64_t> m = index_map(cand_off, R);
  const DcaDims D{q, H, dh, scale};
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t k = 0; k < n_sel; ++k) {
    const int64_t i = sel_cand[k], r = m[(size_t)i];
    dca_candidate(D, Q, K, V, i, seq_off[r], seq_off[r + 1], nullptr, o + k * q * H * dh, lse + k * q * H);
  }
  return ORC_OK;
}

// Linear query projection: q_out[k, n] = sum_j w_q[n, j] * y[k, j], j ascending.
// y is bf16 bit patterns [n_rows, n_in]; w_q bf16 [n_out, n_in]; q_out double [n_rows, n_out].
int rocs_oracle_proj(int64_t n_rows, int64_t n_in, int64_t n_out, const uint16_t* y, const uint16_t* w_q,
                     double* q_out, int nthreads) {
  if (n_rows < 0 || n_in < 0 || n_out < 0) return ORC_INVALID;
  set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t k = 0; k < n_rows; ++k)
    for (int64_t n = 0; n < n_out; ++n) {
      double acc = 0.0;
      for (int64_t j = 0; j < n_in; ++j) acc += widen(w_q, 1, n * n_in + j) * widen(y, 1, k * n_in + j);
      q_out[k * n_out + n] = acc;
    }
  return ORC_OK;
}

// Chained block for the candidates in sel_cand (q = 1 query token per candidate):
//   Y^C_i (LCB, Eq. 6) -> [round to bf16 if round_y] -> Q_i = W_q . vec(Y^C_i) -> round to bf16
//   -> DCA over request m_i's keys with H heads of size dh.
// round_y = 1: Y^C is stored in bf16 between the LCB and the projection (the unfused chain);
// round_y = 0: the projection consumes the exact LCB output (a chain that never stores Y^C).
// Outputs: y_cand [n_sel, o_c, d] (before rounding), q_out [n_sel, H*dh] (before rounding),
// o [n_sel, H, dh], lse [n_sel, H].
static int chain_impl(int64_t R, const int32_t* cand_off, int64_t n_r, int64_t n_c, int64_t d, int64_t o_r,
                      int64_t o_c, const uint16_t* x_req, const uint16_t* x_cand, const uint16_t* w_rr,
                      const uint16_t* w_cr, const uint16_t* w_cc, const uint16_t* w_q, const int32_t* seq_off,
                      int64_t H, int64_t dh, double scale, const uint16_t* K, const uint16_t* V, int64_t n_sel,
                      const int64_t* sel_cand, double* y_cand, double* q_out, double* o, double* lse, int round_y,
                      int nthreads) {
  if (!csr_ok(cand_off, R, -1) || !csr_ok(seq_off, R, -1)) return ORC_BAD_OFFSETS;
  set_threads(nthreads);
  const LcbDims D{n_r, n_c, d, o_r, o_c};
  const int64_t C = cand_off[R], n_in = o_c * d, n_out = H * dh;
  for (int64_t k = 0; k < n_sel; ++k)
    if (sel_cand[k] < 0 || sel_cand[k] >= C) return ORC_INVALID;
  std::vector<int64_t> m = index_map(cand_off, R);
  std::vector<double> W;
  lcb_full_weight(D, 1, w_rr, w_cr, w_cc, W);
  const DcaDims DD{1, H, dh, scale};
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t k = 0; k < n_sel; ++k) {
    const int64_t i = sel_cand[k], r = m[(size_t)i];
    double* yc = y_cand + k * n_in;
    if (!lcb_candidate(D, 1, x_req, x_cand, W, i, r, yc)) bad |= 1;
    std::vector<double> yb((size_t)n_in), qb((size_t)n_out);
    for (int64_t j = 0; j < n_in; ++j) yb[(size_t)j] = round_y ? round_bf16(yc[j]) : yc[j];
    for (int64_t n = 0; n < n_out; ++n) {
      double acc = 0.0;
      for (int64_t j = 0; j < n_in; ++j) acc += widen(w_q, 1, n * n_in + j) * yb[(size_t)j];
      q_out[k * n_out + n] = acc;
      qb[(size_t)n] = round_bf16(acc);
    }
    dca_candidate(DD, nullptr, K, V, i, seq_off[r], seq_off[r + 1], qb.data(), o + k * n_out, lse + k * H);
  }
  return bad ? ORC_ISOLATION : ORC_OK;
}

int rocs_oracle_chain(int64_t R, const int32_t* cand_off, int64_t n_r, int64_t n_c, int64_t d, int64_t o_r,
                      int64_t o_c, const uint16_t* x_req, const uint16_t* x_cand, const uint16_t* w_rr,
                      const uint16_t* w_cr, const uint16_t* w_cc, const uint16_t* w_q, const int32_t* seq_off,
                      int64_t H, int64_t dh, double scale, const uint16_t* K, const uint16_t* V, int64_t n_sel,
                      const int64_t* sel_cand, double* y_cand, double* q_out, double* o, double* lse, int nthreads) {
  return chain_impl(R, cand_off, n_r, n_c, d, o_r, o_c, x_req, x_cand, w_rr, w_cr, w_cc, w_q, seq_off, H, dh, scale,
                    K, V, n_sel, sel_cand, y_cand, q_out, o, lse, 1, nthreads);
}

int rocs_oracle_chain_exact(int64_t R, const int32_t* cand_off, int64_t n_r, int64_t n_c, int64_t d, int64_t o_r,
                            int64_t o_c, const uint16_t* x_req, const uint16_t* x_cand, const uint16_t* w_rr,
                            const uint16_t* w_cr, const uint16_t* w_cc, const uint16_t* w_q, const int32_t* seq_off,
                            int64_t H, int64_t dh, double scale, const uint16_t* K, const uint16_t* V, int64_t n_sel,
                            const int64_t* sel_cand, double* y_cand, double* q_out, double* o, double* lse,
                            int nthreads) {
  return chain_impl(R, cand_off, n_r, n_c, d, o_r, o_c, x_req, x_cand, w_rr, w_cr, w_cc, w_q, seq_off, H, dh, scale,
                    K, V, n_sel, sel_cand, y_cand, q_out, o, lse, 0, nthreads);
}

// The projection weight folded with W_CC (the linear maps compose):
//   W_q vec(W_CC X) = W_fold vec(X),   W_fold[k, n*d + c] = sum_o W_q[k, o*d + c] W_CC[o, n]
// w_q [n_out, o_c*d] bf16, w_cc [o_c, n_c] bf16 -> w_fold [n_out, n_c*d] in fp64.
int rocs_oracle_chain_fold(int64_t n_out, int64_t o_c, int64_t n_c, int64_t d, const uint16_t* w_q,
                           const uint16_t* w_cc, double* w_fold, int nthreads) {
  if (n_out < 0 || o_c < 0 || n_c < 0 || d < 0) return ORC_INVALID;
  set_threads(nthreads);
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < n_out; ++k)
    for (int64_t n = 0; n < n_c; ++n)
      for (int64_t c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int64_t o = 0; o < o_c; ++o) acc += widen(w_q, 1, k * o_c * d + o * d + c) * widen(w_cc, 1, o * n_c + n);
        w_fold[(k * n_c + n) * d + c] = acc;
      }
  return ORC_OK;
}

// DCA block (section 3.2, Eq. (13)), both query groups, for the selected requests / candidates.
// s_seq [T, d_s] bf16 request sequence representation (rows seq_off[r]..seq_off[r+1]-1 belong to r);
// w_kc, w_vc, w_kr, w_vr [H*dh, d_s] bf16; q_c [C*q, H, dh] and q_r [R*q_r, H, dh] bf16.
// Candidate group: for candidate i the request's sequence rows are copied (materialised broadcast),
// projected K_i = S_{m_i} W_K^C^T, V_i = S_{m_i} W_V^C^T in fp64, rounded to bf16 (the stored
// precision of projected K/V), and attended by the candidate's q tokens.  Request group: the same
// with W_K^R, W_V^R and request r's own q_r tokens.  Outputs o_c [n_sel_c, q, H, dh], lse_c
// [n_sel_c, q, H], o_r [n_sel_r, q_r, H, dh], lse_r [n_sel_r, q_r, H].
static void project_rows(const uint16_t* s_seq, int64_t s0, int64_t L, int64_t d_s, const uint16_t* w, int64_t n_out,
                         std::vector<uint16_t>& out) {
  out.assign((size_t)(L * n_out), 0);
  for (int64_t j = 0; j < L; ++j)
    for (int64_t n = 0; n < n_out; ++n) {
      double acc = 0.0;
      for (int64_t e = 0; e < d_s; ++e) acc += widen(s_seq, 1, (s0 + j) * d_s + e) * widen(w, 1, n * d_s + e);
      const float f = (float)round_bf16(acc);  // exact: a bf16 value
      uint32_t u;
      std::memcpy(&u, &f, 4);
      out[(size_t)(j * n_out + n)] = (uint16_t)(u >> 16);
    }
}

int rocs_oracle_dca_block(int64_t R, const int32_t* cand_off, const int32_t* seq_off, int64_t q, int64_t q_r,
                          int64_t H, int64_t dh, int64_t d_s, double scale, const uint16_t* s_seq, const uint16_t* w_kc,
                          const uint16_t* w_vc, const uint16_t* w_kr, const uint16_t* w_vr, const uint16_t* q_c,
                          const uint16_t* q_rq, int64_t n_sel_c, const int64_t* sel_c, double* o_c, double* lse_c,
                          int64_t n_sel_r, const int64_t* sel_r, double* o_r, double* lse_r, int nthreads) {
  if (q < 0 || q_r < 0 || H < 0 || dh < 0 || d_s < 0) return ORC_INVALID;
  if (!csr_ok(cand_off, R, -1) || !csr_ok(seq_off, R, -1)) return ORC_BAD_OFFSETS;
  set_threads(nthreads);
  const int64_t C = cand_off[R], n_out = H * dh;
  for (int64_t k = 0; k < n_sel_c; ++k)
    if (sel_c[k] < 0 || sel_c[k] >= C) return ORC_INVALID;
  for (int64_t k = 0; k < n_sel_r; ++k)
    if (sel_r[k] < 0 || sel_r[k] >= R) return ORC_INVALID;
  std::vector<int64_t> m = index_map(cand_off, R);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t k = 0; k < n_sel_c; ++k) {
    const int64_t i = sel_c[k], r = m[(size_t)i], s0 = seq_off[r], L = seq_off[r + 1] - s0;
    std::vector<uint16_t> Kp, Vp;  // this candidate's own copy of the projected request sequence
    project_rows(s_seq, s0, L, d_s, w_kc, n_out, Kp);
    project_rows(s_seq, s0, L, d_s, w_vc, n_out, Vp);
    const DcaDims D{q, H, dh, scale};
    dca_candidate(D, q_c, Kp.data(), Vp.data(), i, 0, L, nullptr, o_c + k * q * n_out, lse_c + k * q * H);
  }
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t k = 0; k < n_sel_r; ++k) {
    const int64_t r = sel_r[k], s0 = seq_off[r], L = seq_off[r + 1] - s0;
    std::vector<uint16_t> Kp, Vp;
    project_rows(s_seq, s0, L, d_s, w_kr, n_out, Kp);
    project_rows(s_seq, s0, L, d_s, w_vr, n_out, Vp);
    const DcaDims D{q_r, H, dh, scale};
    dca_candidate(D, q_rq, Kp.data(), Vp.data(), r, 0, L, nullptr, o_r + k * q_r * n_out, lse_r + k * q_r * H);
  }
  return ORC_OK;
}

// LCB block (section 3.1.2 Eq. (4)-(6) with the epilogues of section 3.1.3 Eq. (7)-(8)), bf16 inputs.
// Each selected candidate's full output [Y^R; Y^C] = W_full X_full + [b^R; b^C] is formed with the
// broadcast materialised (as rocs_oracle_lcb), then each output row gets its own group's epilogue
// (residual^R indexed by request row r*o_r+o, residual^C by candidate row i*o_c+o).  The request rows
// of every candidate's full output must equal Y^R of the request computed alone (Eq. (11)).
int rocs_oracle_lcb_block(int64_t R, const int32_t* cand_off, int64_t n_r, int64_t n_c, int64_t d, int64_t o_r,
                          int64_t o_c, const uint16_t* x_req, const uint16_t* x_cand, const uint16_t* w_rr,
                          const uint16_t* w_cr, const uint16_t* w_cc, const OrcEpi* epi_r, const OrcEpi* epi_c,
                          int64_t n_sel_req, const int64_t* sel_req, double* y_req, int64_t n_sel_cand,
                          const int64_t* sel_cand, double* y_cand, int nthreads) {
  if (n_r < 0 || n_c < 0 || d < 0 || o_r < 0 || o_c < 0 || !epi_ok(epi_r) || !epi_ok(epi_c)) return ORC_INVALID;
  if (!csr_ok(cand_off, R, -1)) return ORC_BAD_OFFSETS;
  set_threads(nthreads);
  const LcbDims D{n_r, n_c, d, o_r, o_c};
  const int64_t C = cand_off[R];
  for (int64_t k = 0; k < n_sel_req; ++k)
    if (sel_req[k] < 0 || sel_req[k] >= R) return ORC_INVALID;
  for (int64_t k = 0; k < n_sel_cand; ++k)
    if (sel_cand[k] < 0 || sel_cand[k] >= C) return ORC_INVALID;
  std::vector<int64_t> m = index_map(cand_off, R);
  std::vector<double> W;
  lcb_full_weight(D, 1, w_rr, w_cr, w_cc, W);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t k = 0; k < n_sel_req; ++k) lcb_block_request(D, x_req, W, *epi_r, sel_req[k], y_req + k * o_r * d);
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t k = 0; k < n_sel_cand; ++k) {
    const int64_t i = sel_cand[k], r = m[(size_t)i], ni = n_r + n_c, no = o_r + o_c;
    // the explicit broadcast: X_full = [X^R_r ; X^C_i]
    std::vector<double> X((size_t)(ni * d)), Y((size_t)(no * d));
    for (int64_t j = 0; j < n_r; ++j)
      for (int64_t c = 0; c < d; ++c) X[(size_t)(j * d + c)] = widen(x_req, 1, (r * n_r + j) * d + c);
    for (int64_t j = 0; j < n_c; ++j)
      for (int64_t c = 0; c < d; ++c) X[(size_t)((n_r + j) * d + c)] = widen(x_cand, 1, (i * n_c + j) * d + c);
    for (int64_t o = 0; o < no; ++o) {
      const double b = o < o_r ? (epi_r->bias ? (double)epi_r->bias[o] : 0.0)
                               : (epi_c->bias ? (double)epi_c->bias[o - o_r] : 0.0);
      for (int64_t c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int64_t j = 0; j < ni; ++j) acc += W[(size_t)(o * ni + j)] * X[(size_t)(j * d + c)];
        Y[(size_t)(o * d + c)] = acc + b;
      }
      if (o < o_r) epilogue_row(*epi_r, d, r * o_r + o, &Y[(size_t)(o * d)]);
      else epilogue_row(*epi_c, d, i * o_c + (o - o_r), &Y[(size_t)(o * d)]);
    }
    std::vector<double> yr((size_t)(o_r * d));
    lcb_block_request(D, x_req, W, *epi_r, r, yr.data());
    for (int64_t e = 0; e < o_r * d; ++e)
      if (Y[(size_t)e] != yr[(size_t)e]) bad |= 1;
    for (int64_t e = 0; e < o_c * d; ++e) y_cand[k * o_c * d + e] = Y[(size_t)(o_r * d + e)];
  }
  return bad ? ORC_ISOLATION : ORC_OK;
}

// GLM-masked factorization machine (section 3.1.4, Eq. (9)-(10)), bf16 inputs X^R [R, n_r, d],
// X^C [C, n_c, d].  For every selected candidate the full input [X^R_{m_i}; X^C_i] is copied (the
// materialised broadcast), its Gram matrix G = X_full X_full^T is formed in fp64, the block mask of
// Eq. (9) is applied (output group R keeps only its interactions with group R: the R-rows' C-columns
// are set to zero) and the candidate rows [n_r, n_r + n_c) are returned:
//     Y^C_i = [X^C_i X^R_{m_i}^T , X^C_i X^C_i^T]          y_cand [n_sel_c, n_c, n_r + n_c]
// Y^R_r = X^R_r X^R_r^T for the selected requests        y_req  [n_sel_r, n_r, n_r]
// The masked R-rows of each candidate's full output must equal Y^R of its request computed alone and
// hold exact zeros in the C-columns (Eq. (11)); otherwise ORC_ISOLATION.
static void fm_request(const uint16_t* x_req, int64_t n_r, int64_t d, int64_t r, double* y) {
  for (int64_t j = 0; j < n_r; ++j)
    for (int64_t k = 0; k < n_r; ++k) {
      double acc = 0.0;
      for (int64_t c = 0; c < d; ++c) acc += widen(x_req, 1, (r * n_r + j) * d + c) * widen(x_req, 1, (r * n_r + k) * d + c);
      y[j * n_r + k] = acc;
    }
}

int rocs_oracle_fm(int64_t R, const int32_t* cand_off, int64_t n_r, int64_t n_c, int64_t d, const uint16_t* x_req,
                   const uint16_t* x_cand, int64_t n_sel_r, const int64_t* sel_r, double* y_req, int64_t n_sel_c,
                   const int64_t* sel_c, double* y_cand, int nthreads) {
  if (n_r < 0 || n_c < 0 || d < 0) return ORC_INVALID;
  if (!csr_ok(cand_off, R, -1)) return ORC_BAD_OFFSETS;
  set_threads(nthreads);
  const int64_t C = cand_off[R], n = n_r + n_c;
  for (int64_t k = 0; k < n_sel_r; ++k)
    if (sel_r[k] < 0 || sel_r[k] >= R) return ORC_INVALID;
  for (int64_t k = 0; k < n_sel_c; ++k)
    if (sel_c[k] < 0 || sel_c[k] >= C) return ORC_INVALID;
  std::vector<int64_t> m = index_map(cand_off, R);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t k = 0; k < n_sel_r; ++k) fm_request(x_req, n_r, d, sel_r[k], y_req + k * n_r * n_r);
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t k = 0; k < n_sel_c; ++k) {
    const int64_t i = sel_c[k], r = m[(size_t)i];
    std::vector<double> X((size_t)(n * d)), G((size_t)(n * n));
    for (int64_t j = 0; j < n_r; ++j)
      for (int64_t c = 0; c < d; ++c) X[(size_t)(j * d + c)] = widen(x_req, 1, (r * n_r + j) * d + c);
    for (int64_t j = 0; j < n_c; ++j)
      for (int64_t c = 0; c < d; ++c) X[(size_t)((n_r + j) * d + c)] = widen(x_cand, 1, (i * n_c + j) * d + c);
    for (int64_t a = 0; a < n; ++a)
      for (int64_t b = 0; b < n; ++b) {
        double acc = 0.0;
        for (int64_t c = 0; c < d; ++c) acc += X[(size_t)(a * d + c)] * X[(size_t)(b * d + c)];
        const bool masked = a < n_r && b >= n_r;  // M_{R,C} = 0 (Eq. 9)
        G[(size_t)(a * n + b)] = masked ? 0.0 : acc;
      }
    std::vector<double> yr((size_t)(n_r * n_r));
    fm_request(x_req, n_r, d, r, yr.data());
    for (int64_t a = 0; a < n_r; ++a)
      for (int64_t b = 0; b < n; ++b) {
        const double want = b < n_r ? yr[(size_t)(a * n_r + b)] : 0.0;
        if (G[(size_t)(a * n + b)] != want) bad |= 1;
      }
    for (int64_t a = 0; a < n_c; ++a)
      for (int64_t b = 0; b < n; ++b) y_cand[(k * n_c + a) * n + b] = G[(size_t)((n_r + a) * n + b)];
  }
  return bad ? ORC_ISOLATION : ORC_OK;
}

// Exposed for the oracle's own tests of its bf16 rounding.
double rocs_oracle_round_bf16(double x) { return round_bf16(x); }

}  // extern "C"
