// expand.cu -- explicit-expand GPU baselines (ablation, NOT the method).
//
// The dense execution that "ROCS ..." (arXiv:2607.27744, section 4, opening paragraph; section
// 4.3) describes as the cost IKBO removes: request-side tensors are copied to the candidate
// batch size (the request-to-candidate broadcast is materialised in HBM) and the same GEMM /
// attention kernels then run with the identity map, every candidate its own "request".
//   LCB: X^R is expanded to [C, n_r, d]; Y^R and Z are recomputed per candidate.
//   DCA: each candidate's request K/V rows are copied into a per-candidate buffer, a chunk of
//        candidates at a time (the full expansion would exceed HBM for long histories).
#include <cstring>

#include "lcb_sm100.h"

namespace rocs {

// ------------------------------------------------------------------ device kernels
__device__ __forceinline__ int request_of(const int32_t* off, int R, int i) {
  int lo = 0, hi = R - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= i) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// out[k] = min(k, C) for k in [0, C + R]: C one-candidate items followed by R empty ones
__global__ void rocs_expand_ident_kernel(int32_t* out, int C, int n) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k <= n; k += gridDim.x * blockDim.x) out[k] = k < C ? k : C;
}

// item k < C copies request m_k's block, item k >= C copies request k - C's block
__global__ void rocs_expand_rows_kernel(const uint4* src, uint4* dst, const int32_t* cand_off, int R, int C,
                                        int64_t item_vec) {
  const int k = blockIdx.x;
  const int r = k < C ? request_of(cand_off, R, k) : k - C;
  const uint4* s = src + (int64_t)r * item_vec;
  uint4* d = dst + (int64_t)k * item_vec;
  for (int64_t e = threadIdx.x; e < item_vec; e += blockDim.x) d[e] = s[e];
}

// expanded key offsets of candidates [c0, c1): seq_out[k] = sum_{j<k} L_{m_{c0+j}}, cand_out = identity
__global__ void rocs_expand_kv_offsets_kernel(const int32_t* cand_off, const int32_t* seq_off, int R, int c0, int n,
                                              int32_t* cand_out, int32_t* seq_out) {
  __shared__ int s_part[1024];
  const int T = blockDim.x, t = threadIdx.x, per = (n + T - 1) / T;
  const int b0 = min(n, t * per), b1 = min(n, b0 + per);
  int sum = 0;
  for (int k = b0; k < b1; ++k) {
    const int r = request_of(cand_off, R, c0 + k);
    sum += seq_off[r + 1] - seq_off[r];
  }
  s_part[t] = sum;
  __syncthreads();
  for (int off = 1; off < T; off <<= 1) {
    const int v = t >= off ? s_part[t - off] : 0;
    __syncthreads();
    s_part[t] += v;
    __syncthreads();
  }
  int run = s_part[t] - sum;
  for (int k = b0; k < b1; ++k) {
    const int r = request_of(cand_off, R, c0 + k);
    seq_out[k] = run;
    cand_out[k] = k;
    run += seq_off[r + 1] - seq_off[r];
  }
  if (t == T - 1) {
    seq_out[n] = s_part[T - 1];
    cand_out[n] = n;
  }
}

__global__ void rocs_expand_kv_kernel(const uint4* k, const uint4* v, uint4* k_out, uint4* v_out,
                                      const int32_t* cand_off, const int32_t* seq_off, const int32_t* seq_out, int R,
                                      int c0, int64_t row_vec) {
  const int j = blockIdx.x;
  const int r = request_of(cand_off, R, c0 + j);
  const int64_t n = (int64_t)(seq_off[r + 1] - seq_off[r]) * row_vec;
  const int64_t src = (int64_t)seq_off[r] * row_vec, dst = (int64_t)seq_out[j] * row_vec;
  for (int64_t e = threadIdx.x; e < n; e += blockDim.x) {
    k_out[dst + e] = k[src + e];
    v_out[dst + e] = v[src + e];
  }
}

cudaError_t launch_ident(int32_t* out, int n, cudaStream_t st) {  // out[k] = k, k = 0..n
  rocs_expand_ident_kernel<<<(n + 256) / 256 < 4096 ? (n + 256) / 256 : 4096, 256, 0, st>>>(out, n, n);
  return cudaGetLastError();
}

cudaError_t launch_expand_rows(const void* src, void* dst, const int32_t* cand_off, int R, int C, int64_t row_bytes,
                               int64_t rows_per_item, cudaStream_t st) {
  const int64_t item_vec = row_bytes * rows_per_item / 16;
  if (C + R > 0)
    rocs_expand_rows_kernel<<<C + R, 256, 0, st>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst),
                                                   cand_off, R, C, item_vec);
  return cudaGetLastError();
}

}  // namespace rocs

using namespace rocs;

namespace rocs {
// defined in rocs_abi.cu
int lcb_validate_ext(const rocs_lcb_args* a, int64_t* C);
int lcb_run_ext(const rocs_lcb_args* a, int64_t C, WsHeader* hdr, uint8_t* body, cudaStream_t st, int* launches);
size_t lcb_body_bytes_ext(int64_t R, int64_t o_c, int64_t d);
int dca_validate_ext(const rocs_dca_args* a, int64_t* C, int64_t* T);
int dca_run_ext(const rocs_dca_args* a, int64_t C, int64_t T, int64_t n_units, WsHeader* hdr, uint8_t* body,
                cudaStream_t st, int* launches);
size_t dca_body_bytes_ext(int64_t R, int64_t n_units);
int dca_rows_per_unit();
void set_last_launches(int n);
}  // namespace rocs

namespace {
inline size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

struct LcbExpandLayout {
  size_t ident, xr, yr, inner, bytes;
};
LcbExpandLayout lcb_expand_layout(const rocs_lcb_args* a, int64_t C) {
  const int64_t n = C + a->R, es = a->dtype == ROCS_BF16 ? 2 : 4;
  LcbExpandLayout L;  // [WsHeader][identity CSR][X^R expanded][Y^R expanded][LCB body]
  L.ident = sizeof(WsHeader);
  L.xr = a256(L.ident + (size_t)(n + 1) * 4);
  L.yr = a256(L.xr + (size_t)n * a->n_r * a->d * es);
  L.inner = a256(L.yr + (size_t)n * a->o_r * a->d * es);
  L.bytes = L.inner + lcb_body_bytes_ext(n, a->o_c, a->d);
  return L;
}

struct DcaExpandLayout {
  size_t coff, soff, k, v, inner, bytes;
  int64_t max_rows, units_per_chunk;
};
DcaExpandLayout dca_expand_layout(const rocs_dca_args* a, int64_t C, int64_t chunk) {
  DcaExpandLayout L;
  // the largest number of expanded key rows any chunk needs
  int64_t best = 0;
  int64_t r = 0;
  for (int64_t c0 = 0; c0 < C; c0 += chunk) {
    const int64_t c1 = c0 + chunk < C ? c0 + chunk : C;
    int64_t rows = 0;
    for (int64_t i = c0; i < c1; ++i) {
      while (a->cand_off_host[r + 1] <= i) ++r;
      rows += a->seq_off_host[r + 1] - a->seq_off_host[r];
    }
    if (rows > best) best = rows;
    if (c1 == C) break;
  }
  const int rpu = dca_rows_per_unit();
  L.max_rows = best;
  L.units_per_chunk = chunk * a->H * ((a->q + rpu - 1) / rpu);
  const size_t row = (size_t)a->H * a->dh * 2;  // [WsHeader][cand CSR][key CSR][K exp][V exp][DCA body]
  L.coff = sizeof(WsHeader);
  L.soff = a256(L.coff + (size_t)(chunk + 1) * 4);
  L.k = a256(L.soff + (size_t)(chunk + 1) * 4);
  L.v = a256(L.k + (size_t)best * row);
  L.inner = a256(L.v + (size_t)best * row);
  L.bytes = L.inner + dca_body_bytes_ext(chunk, L.units_per_chunk);
  return L;
}
}  // namespace

extern "C" {

size_t rocs_lcb_expand_workspace_size(const rocs_lcb_args* a) {
  int64_t C;
  if (lcb_validate_ext(a, &C) != ROCS_OK) return 0;
  return lcb_expand_layout(a, C).bytes;
}

int rocs_lcb_forward_expand(const rocs_lcb_args* a, rocs_stream_t stream) {
  int64_t C = 0;
  int rc = lcb_validate_ext(a, &C);
  if (rc) return rc;
  const LcbExpandLayout L = lcb_expand_layout(a, C);
  if (!a->workspace || a->workspace_bytes < L.bytes || (reinterpret_cast<uintptr_t>(a->workspace) & 255))
    return ROCS_ERR_WORKSPACE;
  if (a->R == 0) return ROCS_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(a->workspace);
  const int64_t n = C + a->R, es = a->dtype == ROCS_BF16 ? 2 : 4;
  int32_t* ident = reinterpret_cast<int32_t*>(w + L.ident);
  rocs_expand_ident_kernel<<<(int)((n + 256) / 256 < 4096 ? (n + 256) / 256 : 4096), 256, 0, st>>>(ident, (int)C,
                                                                                                  (int)n);
  if (cudaGetLastError() != cudaSuccess) return ROCS_ERR_CUDA;
  if (launch_expand_rows(a->x_req, w + L.xr, a->cand_off_dev, (int)a->R, (int)C, a->d * es, a->n_r, st) !=
      cudaSuccess)
    return ROCS_ERR_CUDA;
  rocs_lcb_args e = *a;
  e.R = n;
  e.cand_off_dev = ident;
  e.cand_off_host = nullptr;  // not read by the launcher; the expanded CSR is the identity map
  e.x_req = w + L.xr;
  e.y_req = w + L.yr;
  int launches = 0;
  rc = lcb_run_ext(&e, C, reinterpret_cast<WsHeader*>(w), w + L.inner, st, &launches);
  if (rc) return rc;
  // Y^R of the R trailing (candidate-free) items are the request outputs
  if (cudaMemcpyAsync(a->y_req, w + L.yr + (size_t)C * a->o_r * a->d * es, (size_t)a->R * a->o_r * a->d * es,
                      cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return ROCS_ERR_CUDA;
  set_last_launches(launches + 2);
  return ROCS_OK;
}

size_t rocs_dca_expand_workspace_size(const rocs_dca_args* a, int64_t chunk) {
  int64_t C, T;
  if (chunk <= 0 || chunk > (1 << 20) || dca_validate_ext(a, &C, &T) != ROCS_OK) return 0;
  return dca_expand_layout(a, C, chunk).bytes;
}

int rocs_dca_forward_expand(const rocs_dca_args* a, int64_t chunk, rocs_stream_t stream) {
  int64_t C = 0, T = 0;
  if (chunk <= 0 || chunk > (1 << 20)) return ROCS_ERR_INVALID_ARG;
  int rc = dca_validate_ext(a, &C, &T);
  if (rc) return rc;
  if (a->kv_ld != 0 && a->kv_ld != a->H * a->dh) return ROCS_ERR_UNSUPPORTED;  // the copies assume dense rows
  const DcaExpandLayout L = dca_expand_layout(a, C, chunk);
  if (!a->workspace || a->workspace_bytes < L.bytes || (reinterpret_cast<uintptr_t>(a->workspace) & 255))
    return ROCS_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(a->workspace);
  int32_t* coff = reinterpret_cast<int32_t*>(w + L.coff);
  int32_t* soff = reinterpret_cast<int32_t*>(w + L.soff);
  const size_t qrow = (size_t)a->q * a->H * a->dh;
  int total = 0;
  int64_t r = 0;
  for (int64_t c0 = 0; c0 < C; c0 += chunk) {
    const int64_t c1 = c0 + chunk < C ? c0 + chunk : C, n = c1 - c0;
    int64_t rows = 0;
    for (int64_t i = c0; i < c1; ++i) {
      while (a->cand_off_host[r + 1] <= i) ++r;
      rows += a->seq_off_host[r + 1] - a->seq_off_host[r];
    }
    rocs_expand_kv_offsets_kernel<<<1, 1024, 0, st>>>(a->cand_off_dev, a->seq_off_dev, (int)a->R, (int)c0, (int)n,
                                                       coff, soff);
    rocs_expand_kv_kernel<<<(int)n, 256, 0, st>>>(
        static_cast<const uint4*>(a->k_ptr), static_cast<const uint4*>(a->v_ptr), reinterpret_cast<uint4*>(w + L.k),
        reinterpret_cast<uint4*>(w + L.v), a->cand_off_dev, a->seq_off_dev, soff, (int)a->R, (int)c0,
        (int64_t)a->H * a->dh * 2 / 16);
    if (cudaGetLastError() != cudaSuccess) return ROCS_ERR_CUDA;
    rocs_dca_args e = *a;
    e.R = n;
    e.cand_off_dev = coff;
    e.seq_off_dev = soff;
    e.cand_off_host = nullptr;
    e.seq_off_host = nullptr;
    e.q_ptr = static_cast<const uint8_t*>(a->q_ptr) + c0 * qrow * 2;
    e.o_ptr = static_cast<uint8_t*>(a->o_ptr) + c0 * qrow * 2;
    e.lse_ptr = a->lse_ptr ? a->lse_ptr + c0 * a->q * a->H : nullptr;
    e.k_ptr = w + L.k;
    e.v_ptr = w + L.v;
    int launches = 0;
    const int rpu = dca_rows_per_unit();
    rc = dca_run_ext(&e, n, rows, n * a->H * ((a->q + rpu - 1) / rpu), reinterpret_cast<WsHeader*>(w), w + L.inner,
                     st, &launches);
    if (rc) return rc;
    total += launches + 2;
  }
  set_last_launches(total);
  return ROCS_OK;
}

}  // extern "C"
