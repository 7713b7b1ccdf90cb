// lcb_f32.cu -- IKBO-LCB in fp32 on the CUDA cores (the fp32 configuration: tensor-core
// TF32 would not meet an fp32 error budget).  Same decomposition as the bf16 kernel
// ("ROCS ...", arXiv:2607.27744, section 4.1, Eq. (14)):
//   launch 1, one block per (request, output-row group):  Y^R_r = W_RR X^R_r,  Z_r = W_CR X^R_r
//   launch 2, one block per candidate:                     Y^C_i = W_CC X^C_i + Z_{m_i}
// with m_i resolved inside the kernel from the CSR offsets (section 4.3.1's in-kernel
// lookup, here a binary search) -- the request tensors are never expanded per candidate.
#include "lcb_sm100.h"

namespace rocs {

__global__ void rocs_lcb_f32_request_kernel(const LcbF32Params p) {
  const int r = blockIdx.x;
  const int rows = p.o_r + p.o_c;
  const float* xr = p.x_req + (size_t)r * p.n_r * p.d;
  for (int e = threadIdx.x; e < rows * p.d; e += blockDim.x) {
    const int o = e / p.d, c = e % p.d;
    const float* w = o < p.o_r ? p.w_rr + (size_t)o * p.n_r : p.w_cr + (size_t)(o - p.o_r) * p.n_r;
    float acc = 0.f;
    for (int j = 0; j < p.n_r; ++j) acc = fmaf(w[j], xr[(size_t)j * p.d + c], acc);
    if (o < p.o_r) p.y_req[((size_t)r * p.o_r + o) * p.d + c] = acc;
    else p.z[((size_t)r * p.o_c + (o - p.o_r)) * p.d + c] = acc;
  }
}

__global__ void rocs_lcb_f32_candidate_kernel(const LcbF32Params p) {
  const int i = blockIdx.x;
  __shared__ int s_r;
  if (threadIdx.x == 0) {
    int lo = 0, hi = p.R - 1;  // last r with cand_off[r] <= i
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.cand_off[mid] <= i) lo = mid; else hi = mid - 1;
    }
    if (!(p.cand_off[lo] <= i && i < p.cand_off[lo + 1])) {
      record_error(p.ws, ROCS_ERR_DEVICE_INDEX, 401);
      lo = -1;
    }
    s_r = lo;
  }
  __syncthreads();
  const int r = s_r;
  if (r < 0) return;
  const float* xc = p.x_cand + (size_t)i * p.n_c * p.d;
  const float* z = p.z + (size_t)r * p.o_c * p.d;
  for (int e = threadIdx.x; e < p.o_c * p.d; e += blockDim.x) {
    const int o = e / p.d, c = e % p.d;
    const float* w = p.w_cc + (size_t)o * p.n_c;
    float acc = 0.f;
    for (int j = 0; j < p.n_c; ++j) acc = fmaf(w[j], xc[(size_t)j * p.d + c], acc);
    p.y_cand[(size_t)i * p.o_c * p.d + e] = acc + z[e];
  }
}

cudaError_t launch_lcb_f32(const LcbF32Params& p, cudaStream_t st) {
  if (p.R > 0) rocs_lcb_f32_request_kernel<<<p.R, 256, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (p.C > 0) rocs_lcb_f32_candidate_kernel<<<p.C, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace rocs
