// host_pipeline.cu -- IKBO-LCB / IKBO-DCA on batches that live in (pinned) host memory.
//
// A batch is cut into chunks of whole requests (the CSR keeps a request's candidates, and its key
// sequence, contiguous, so a chunk's inputs and outputs are contiguous slices).  Two device staging
// slots alternate: while chunk c is computed in one slot, chunk c+1's inputs are copied in and chunk
// c-1's outputs copied out of the other, on three streams (copy-in, compute, copy-out) ordered by
// events.  Host-to-device and device-to-host copies run at the same time over the full-duplex link,
// so a PCIe-bound batch costs about max(input bytes, output bytes) instead of their sum.  The device
// kernels are the ones of rocs_lcb_forward / rocs_dca_forward, run per chunk on chunk-local CSR
// offsets (rebased on the device from the caller's device CSR).
//
// The three streams and their events are created once per device on first use and kept for the
// life of the process (like the caller's own CUDA context resources); every call enqueues only.
#include <algorithm>
#include <mutex>
#include <vector>

#include "lcb_sm100.h"

namespace rocs {
int lcb_validate_ext(const rocs_lcb_args* a, int64_t* C);
int lcb_run_ext(const rocs_lcb_args* a, int64_t C, WsHeader* hdr, uint8_t* body, cudaStream_t st, int* launches);
size_t lcb_body_bytes_ext(int64_t R, int64_t o_c, int64_t d);
int dca_validate_ext(const rocs_dca_args* a, int64_t* C, int64_t* T);
int dca_run_ext(const rocs_dca_args* a, int64_t C, int64_t T, int64_t n_units, WsHeader* hdr, uint8_t* body,
                cudaStream_t st, int* launches);
size_t dca_body_bytes_ext(int64_t R, int64_t n_units);
int64_t dca_units_ext(const rocs_dca_args* a);
void set_last_launches(int n);
}  // namespace rocs

using namespace rocs;

namespace {

inline size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

// dst[i] = src[r0 + i] - src[r0], i = 0..n  (chunk-local CSR offsets)
__global__ void rebase_offsets_kernel(const int32_t* __restrict__ src, int r0, int n, int32_t* __restrict__ dst) {
  const int32_t base = src[r0];
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= n; i += gridDim.x * blockDim.x) dst[i] = src[r0 + i] - base;
}

// keep the first device error of any chunk in the call's status header
__global__ void merge_status_kernel(const WsHeader* chunk, WsHeader* call) {
  if (threadIdx.x == 0 && chunk->code != 0 && call->code == 0) {
    call->code = chunk->code;
    call->detail = chunk->detail;
  }
}

struct Pipe {
  cudaStream_t s_in = nullptr, s_cmp = nullptr, s_out = nullptr;
  cudaEvent_t start = nullptr, in[2] = {}, cmp[2] = {}, out[2] = {};
  bool ok = false;
};

Pipe* pipe_for_current_device() {
  static std::mutex mu;
  static Pipe pipes[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  Pipe& p = pipes[dev];
  if (!p.ok) {
    bool ok = cudaStreamCreateWithFlags(&p.s_in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p.s_cmp, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p.s_out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&p.start, cudaEventDisableTiming) == cudaSuccess;
    for (int k = 0; ok && k < 2; ++k)
      ok = cudaEventCreateWithFlags(&p.in[k], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&p.cmp[k], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&p.out[k], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) return nullptr;
    p.ok = true;
  }
  return &p;
}

// Request ranges [b[k], b[k+1]) with about equal `weight` (weight(r) >= 0), at most `chunks` of them.
std::vector<int64_t> split_requests(int64_t R, int64_t chunks, const std::vector<int64_t>& weight) {
  int64_t total = 0;
  for (int64_t r = 0; r < R; ++r) total += weight[(size_t)r];
  std::vector<int64_t> b{0};
  int64_t acc = 0;
  for (int64_t r = 0; r < R; ++r) {
    acc += weight[(size_t)r];
    const int64_t k = (int64_t)b.size();  // chunk boundaries placed so far
    if (k < chunks && r + 1 < R && acc * chunks >= total * k) b.push_back(r + 1);
  }
  b.push_back(R);
  return b;
}

// ---------------------------------------------------------------- LCB
struct LcbPlan {
  std::vector<int64_t> b;  // request boundaries of the chunks
  int64_t R_max = 0, C_max = 0;
  size_t ws, csr, xr, xc, yr, yc, slot;  // byte offsets inside one slot, slot size
};

LcbPlan lcb_plan(const rocs_lcb_args* a, int64_t chunks) {
  LcbPlan P;
  std::vector<int64_t> w((size_t)a->R);
  for (int64_t r = 0; r < a->R; ++r)  // bytes moved for request r
    w[(size_t)r] = a->n_r * a->d + a->o_r * a->d + (int64_t)(a->cand_off_host[r + 1] - a->cand_off_host[r]) *
                                                     (a->n_c + a->o_c) * a->d;
  P.b = split_requests(a->R, chunks, w);
  for (size_t k = 0; k + 1 < P.b.size(); ++k) {
    P.R_max = std::max(P.R_max, P.b[k + 1] - P.b[k]);
    P.C_max = std::max<int64_t>(P.C_max, a->cand_off_host[P.b[k + 1]] - a->cand_off_host[P.b[k]]);
  }
  const size_t es = a->dtype == ROCS_BF16 ? 2 : 4;
  P.ws = 0;
  P.csr = a256(sizeof(WsHeader) + lcb_body_bytes_ext(P.R_max, a->o_c, a->d));
  P.xr = P.csr + a256((size_t)(P.R_max + 1) * sizeof(int32_t));
  P.xc = P.xr + a256((size_t)P.R_max * a->n_r * a->d * es);
  P.yr = P.xc + a256((size_t)P.C_max * a->n_c * a->d * es);
  P.yc = P.yr + a256((size_t)P.R_max * a->o_r * a->d * es);
  P.slot = P.yc + a256((size_t)P.C_max * a->o_c * a->d * es);
  return P;
}

// ---------------------------------------------------------------- DCA
struct DcaPlan {
  std::vector<int64_t> b;
  int64_t R_max = 0, C_max = 0, T_max = 0, U_max = 0;
  size_t ws, csr_c, csr_s, q, k, v, o, lse, slot;
};

// the chunk's arguments with host offsets rebased into `oc` / `os` (device pointers left to the caller)
rocs_dca_args dca_chunk_args(const rocs_dca_args* a, int64_t r0, int64_t r1, std::vector<int32_t>& oc,
                             std::vector<int32_t>& os) {
  rocs_dca_args ca = *a;
  ca.R = r1 - r0;
  oc.assign((size_t)ca.R + 1, 0);
  os.assign((size_t)ca.R + 1, 0);
  for (int64_t r = 0; r <= ca.R; ++r) {
    oc[(size_t)r] = a->cand_off_host[r0 + r] - a->cand_off_host[r0];
    os[(size_t)r] = a->seq_off_host[r0 + r] - a->seq_off_host[r0];
  }
  ca.cand_off_host = oc.data();
  ca.seq_off_host = os.data();
  return ca;
}

DcaPlan dca_plan(const rocs_dca_args* a, int64_t chunks) {
  DcaPlan P;
  const int64_t hd = a->H * a->dh;
  std::vector<int64_t> w((size_t)a->R);
  for (int64_t r = 0; r < a->R; ++r)
    w[(size_t)r] = 2 * a->q * (int64_t)(a->cand_off_host[r + 1] - a->cand_off_host[r]) * hd +
                   2 * (int64_t)(a->seq_off_host[r + 1] - a->seq_off_host[r]) * hd;
  P.b = split_requests(a->R, chunks, w);
  std::vector<int32_t> oc, os;
  for (size_t k = 0; k + 1 < P.b.size(); ++k) {
    const int64_t r0 = P.b[k], r1 = P.b[k + 1];
    P.R_max = std::max(P.R_max, r1 - r0);
    P.C_max = std::max<int64_t>(P.C_max, a->cand_off_host[r1] - a->cand_off_host[r0]);
    P.T_max = std::max<int64_t>(P.T_max, a->seq_off_host[r1] - a->seq_off_host[r0]);
    rocs_dca_args ca = dca_chunk_args(a, r0, r1, oc, os);
    P.U_max = std::max(P.U_max, dca_units_ext(&ca));
  }
  P.ws = 0;
  P.csr_c = a256(sizeof(WsHeader) + dca_body_bytes_ext(P.R_max, P.U_max));
  P.csr_s = P.csr_c + a256((size_t)(P.R_max + 1) * sizeof(int32_t));
  P.q = P.csr_s + a256((size_t)(P.R_max + 1) * sizeof(int32_t));
  P.k = P.q + a256((size_t)P.C_max * a->q * hd * 2);
  P.v = P.k + a256((size_t)P.T_max * hd * 2);
  P.o = P.v + a256((size_t)P.T_max * hd * 2);
  P.lse = P.o + a256((size_t)P.C_max * a->q * hd * 2);
  P.slot = P.lse + a256(a->lse_ptr ? (size_t)P.C_max * a->q * a->H * sizeof(float) : 0);
  return P;
}

}  // namespace

extern "C" {

size_t rocs_lcb_host_staging_size(const rocs_lcb_args* a, int64_t chunks) {
  int64_t C;
  if (chunks < 1 || lcb_validate_ext(a, &C) != ROCS_OK) return 0;
  return 256 + 2 * lcb_plan(a, chunks).slot;
}

int rocs_lcb_forward_host(const rocs_lcb_args* a, int64_t chunks, void* staging, size_t staging_bytes,
                          rocs_stream_t stream) {
  int64_t C = 0;
  int rc = lcb_validate_ext(a, &C);
  if (rc) return rc;
  if (chunks < 1) return ROCS_ERR_INVALID_ARG;
  const LcbPlan P = lcb_plan(a, chunks);
  if (!staging || staging_bytes < 256 + 2 * P.slot || (reinterpret_cast<uintptr_t>(staging) & 255))
    return ROCS_ERR_WORKSPACE;
  Pipe* pp = pipe_for_current_device();
  if (!pp) return ROCS_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  WsHeader* call_hdr = static_cast<WsHeader*>(staging);
  uint8_t* slots = static_cast<uint8_t*>(staging) + 256;
  const size_t es = a->dtype == ROCS_BF16 ? 2 : 4;
  if (cudaEventRecord(pp->start, st) != cudaSuccess || cudaStreamWaitEvent(pp->s_in, pp->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(pp->s_cmp, pp->start, 0) != cudaSuccess ||
      cudaMemsetAsync(call_hdr, 0, sizeof(WsHeader), pp->s_cmp) != cudaSuccess)
    return ROCS_ERR_CUDA;
  int launches = 0;
  const int n_chunks = (int)P.b.size() - 1;
  std::vector<int32_t> off_local;
  for (int c = 0; c < n_chunks; ++c) {
    const int k = c & 1;
    uint8_t* s = slots + (size_t)k * P.slot;
    const int64_t r0 = P.b[c], r1 = P.b[c + 1], Rc = r1 - r0;
    const int64_t c0 = a->cand_off_host[r0], c1 = a->cand_off_host[r1], Cc = c1 - c0;
    // copy in (after the copy-out that last used this slot)
    if (c >= 2 && cudaStreamWaitEvent(pp->s_in, pp->out[k], 0) != cudaSuccess) return ROCS_ERR_CUDA;
    const size_t xr_b = (size_t)Rc * a->n_r * a->d * es, xc_b = (size_t)Cc * a->n_c * a->d * es;
    if ((xr_b && cudaMemcpyAsync(s + P.xr, static_cast<const uint8_t*>(a->x_req) + (size_t)r0 * a->n_r * a->d * es,
                                 xr_b, cudaMemcpyHostToDevice, pp->s_in) != cudaSuccess) ||
        (xc_b && cudaMemcpyAsync(s + P.xc, static_cast<const uint8_t*>(a->x_cand) + (size_t)c0 * a->n_c * a->d * es,
                                 xc_b, cudaMemcpyHostToDevice, pp->s_in) != cudaSuccess) ||
        cudaEventRecord(pp->in[k], pp->s_in) != cudaSuccess)
      return ROCS_ERR_CUDA;
    // compute on chunk-local offsets
    if (cudaStreamWaitEvent(pp->s_cmp, pp->in[k], 0) != cudaSuccess) return ROCS_ERR_CUDA;
    int32_t* csr = reinterpret_cast<int32_t*>(s + P.csr);
    rebase_offsets_kernel<<<1, 256, 0, pp->s_cmp>>>(a->cand_off_dev, (int)r0, (int)Rc, csr);
    if (cudaGetLastError() != cudaSuccess) return ROCS_ERR_CUDA;
    off_local.assign((size_t)Rc + 1, 0);
    for (int64_t r = 0; r <= Rc; ++r) off_local[(size_t)r] = a->cand_off_host[r0 + r] - (int32_t)c0;
    rocs_lcb_args ca = *a;
    ca.R = Rc;
    ca.cand_off_dev = csr;
    ca.cand_off_host = off_local.data();
    ca.x_req = s + P.xr;
    ca.x_cand = Cc ? s + P.xc : nullptr;
    ca.y_req = s + P.yr;
    ca.y_cand = Cc ? s + P.yc : nullptr;
    WsHeader* hdr = reinterpret_cast<WsHeader*>(s + P.ws);
    int l = 0;
    rc = lcb_run_ext(&ca, Cc, hdr, reinterpret_cast<uint8_t*>(hdr + 1), pp->s_cmp, &l);
    if (rc) return rc;
    merge_status_kernel<<<1, 32, 0, pp->s_cmp>>>(hdr, call_hdr);
    if (cudaGetLastError() != cudaSuccess || cudaEventRecord(pp->cmp[k], pp->s_cmp) != cudaSuccess) return ROCS_ERR_CUDA;
    launches += l + 2;
    // copy out
    const size_t yr_b = (size_t)Rc * a->o_r * a->d * es, yc_b = (size_t)Cc * a->o_c * a->d * es;
    if (cudaStreamWaitEvent(pp->s_out, pp->cmp[k], 0) != cudaSuccess ||
        (yr_b && cudaMemcpyAsync(static_cast<uint8_t*>(a->y_req) + (size_t)r0 * a->o_r * a->d * es, s + P.yr, yr_b,
                                 cudaMemcpyDeviceToHost, pp->s_out) != cudaSuccess) ||
        (yc_b && cudaMemcpyAsync(static_cast<uint8_t*>(a->y_cand) + (size_t)c0 * a->o_c * a->d * es, s + P.yc, yc_b,
                                 cudaMemcpyDeviceToHost, pp->s_out) != cudaSuccess) ||
        cudaEventRecord(pp->out[k], pp->s_out) != cudaSuccess)
      return ROCS_ERR_CUDA;
  }
  // the caller's stream continues once every chunk's outputs have landed
  for (int k = 0; k < std::min(2, n_chunks); ++k)
    if (cudaStreamWaitEvent(st, pp->out[k], 0) != cudaSuccess) return ROCS_ERR_CUDA;
  set_last_launches(launches);
  return ROCS_OK;
}

}  // extern "C"

extern "C" {

size_t rocs_dca_host_staging_size(const rocs_dca_args* a, int64_t chunks) {
  int64_t C, T;
  if (chunks < 1 || dca_validate_ext(a, &C, &T) != ROCS_OK || (a->kv_ld != 0 && a->kv_ld != a->H * a->dh)) return 0;
  return 256 + 2 * dca_plan(a, chunks).slot;
}

int rocs_dca_forward_host(const rocs_dca_args* a, int64_t chunks, void* staging, size_t staging_bytes,
                          rocs_stream_t stream) {
  int64_t C = 0, T = 0;
  int rc = dca_validate_ext(a, &C, &T);
  if (rc) return rc;
  if (chunks < 1) return ROCS_ERR_INVALID_ARG;
  if (a->kv_ld != 0 && a->kv_ld != a->H * a->dh) return ROCS_ERR_UNSUPPORTED;  // host K/V rows are contiguous
  const DcaPlan P = dca_plan(a, chunks);
  if (!staging || staging_bytes < 256 + 2 * P.slot || (reinterpret_cast<uintptr_t>(staging) & 255))
    return ROCS_ERR_WORKSPACE;
  Pipe* pp = pipe_for_current_device();
  if (!pp) return ROCS_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  WsHeader* call_hdr = static_cast<WsHeader*>(staging);
  uint8_t* slots = static_cast<uint8_t*>(staging) + 256;
  const size_t hd = (size_t)(a->H * a->dh), qrow = (size_t)a->q * hd * 2, kvrow = hd * 2,
               lrow = (size_t)a->q * a->H * sizeof(float);
  if (cudaEventRecord(pp->start, st) != cudaSuccess || cudaStreamWaitEvent(pp->s_in, pp->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(pp->s_cmp, pp->start, 0) != cudaSuccess ||
      cudaMemsetAsync(call_hdr, 0, sizeof(WsHeader), pp->s_cmp) != cudaSuccess)
    return ROCS_ERR_CUDA;
  int launches = 0;
  const int n_chunks = (int)P.b.size() - 1;
  std::vector<int32_t> oc, os;
  for (int c = 0; c < n_chunks; ++c) {
    const int k = c & 1;
    uint8_t* s = slots + (size_t)k * P.slot;
    const int64_t r0 = P.b[c], r1 = P.b[c + 1];
    const int64_t c0 = a->cand_off_host[r0], Cc = a->cand_off_host[r1] - c0;
    const int64_t s0 = a->seq_off_host[r0], Tc = a->seq_off_host[r1] - s0;
    if (c >= 2 && cudaStreamWaitEvent(pp->s_in, pp->out[k], 0) != cudaSuccess) return ROCS_ERR_CUDA;
    if ((Cc && cudaMemcpyAsync(s + P.q, static_cast<const uint8_t*>(a->q_ptr) + (size_t)c0 * qrow, (size_t)Cc * qrow,
                               cudaMemcpyHostToDevice, pp->s_in) != cudaSuccess) ||
        (Tc && cudaMemcpyAsync(s + P.k, static_cast<const uint8_t*>(a->k_ptr) + (size_t)s0 * kvrow, (size_t)Tc * kvrow,
                               cudaMemcpyHostToDevice, pp->s_in) != cudaSuccess) ||
        (Tc && cudaMemcpyAsync(s + P.v, static_cast<const uint8_t*>(a->v_ptr) + (size_t)s0 * kvrow, (size_t)Tc * kvrow,
                               cudaMemcpyHostToDevice, pp->s_in) != cudaSuccess) ||
        cudaEventRecord(pp->in[k], pp->s_in) != cudaSuccess)
      return ROCS_ERR_CUDA;
    if (cudaStreamWaitEvent(pp->s_cmp, pp->in[k], 0) != cudaSuccess) return ROCS_ERR_CUDA;
    int32_t* csr_c = reinterpret_cast<int32_t*>(s + P.csr_c);
    int32_t* csr_s = reinterpret_cast<int32_t*>(s + P.csr_s);
    rebase_offsets_kernel<<<1, 256, 0, pp->s_cmp>>>(a->cand_off_dev, (int)r0, (int)(r1 - r0), csr_c);
    rebase_offsets_kernel<<<1, 256, 0, pp->s_cmp>>>(a->seq_off_dev, (int)r0, (int)(r1 - r0), csr_s);
    if (cudaGetLastError() != cudaSuccess) return ROCS_ERR_CUDA;
    rocs_dca_args ca = dca_chunk_args(a, r0, r1, oc, os);
    ca.cand_off_dev = csr_c;
    ca.seq_off_dev = csr_s;
    ca.q_ptr = Cc ? s + P.q : nullptr;
    ca.k_ptr = Tc ? s + P.k : nullptr;
    ca.v_ptr = Tc ? s + P.v : nullptr;
    ca.o_ptr = Cc ? s + P.o : nullptr;
    ca.lse_ptr = a->lse_ptr ? reinterpret_cast<float*>(s + P.lse) : nullptr;
    ca.kv_ld = 0;
    WsHeader* hdr = reinterpret_cast<WsHeader*>(s + P.ws);
    int l = 0;
    rc = dca_run_ext(&ca, Cc, Tc, dca_units_ext(&ca), hdr, reinterpret_cast<uint8_t*>(hdr + 1), pp->s_cmp, &l);
    if (rc) return rc;
    merge_status_kernel<<<1, 32, 0, pp->s_cmp>>>(hdr, call_hdr);
    if (cudaGetLastError() != cudaSuccess || cudaEventRecord(pp->cmp[k], pp->s_cmp) != cudaSuccess) return ROCS_ERR_CUDA;
    launches += l + 3;
    if (cudaStreamWaitEvent(pp->s_out, pp->cmp[k], 0) != cudaSuccess ||
        (Cc && cudaMemcpyAsync(static_cast<uint8_t*>(a->o_ptr) + (size_t)c0 * qrow, s + P.o, (size_t)Cc * qrow,
                               cudaMemcpyDeviceToHost, pp->s_out) != cudaSuccess) ||
        (Cc && a->lse_ptr &&
         cudaMemcpyAsync(reinterpret_cast<uint8_t*>(a->lse_ptr) + (size_t)c0 * lrow, s + P.lse, (size_t)Cc * lrow,
                         cudaMemcpyDeviceToHost, pp->s_out) != cudaSuccess) ||
        cudaEventRecord(pp->out[k], pp->s_out) != cudaSuccess)
      return ROCS_ERR_CUDA;
  }
  for (int k = 0; k < std::min(2, n_chunks); ++k)
    if (cudaStreamWaitEvent(st, pp->out[k], 0) != cudaSuccess) return ROCS_ERR_CUDA;
  set_last_launches(launches);
  return ROCS_OK;
}

}  // extern "C"
