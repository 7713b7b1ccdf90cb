// lcb_sm100.h -- launch parameters of the IKBO kernels (internal to the library).
#pragma once
#include "epilogue.cuh"

namespace rocs {

// Persistent IKBO-LCB kernel (bf16 in, fp32 accumulate, bf16 out).
struct LcbParams {
  CUtensorMap tm_xc;   // X^C  viewed as [C*n_c, d],  box {64, n_c}
  CUtensorMap tm_xr;   // X^R  viewed as [R*n_r, d],  box {64, 64}
  CUtensorMap tm_wcc;  // W_CC [o_c, n_c],            box {64, 128}
  CUtensorMap tm_wrr;  // W_RR [o_r, n_r],            box {64, 128}
  CUtensorMap tm_wcr;  // W_CR [o_c, n_r],            box {64, 128}
  CUtensorMap tm_yc;   // Y^C  viewed as [C*o_c, d],  box {64, 32}  (stores)
  CUtensorMap tm_yr;   // Y^R  viewed as [R*o_r, d],  box {64, 32}  (stores)
  const int32_t* cand_off;  // [R+1]
  float* zws;               // Z fp32, [R][d/4][o_c][4]
  int* flags;               // [R], incremented by each epilogue warp of the Z tile
  WsHeader* ws;
  int R, C, n_r, o_r;
  long long wait_limit_ns;  // limit of every wait in the kernel
  int skip_release;         // fault injection: the Z tile of this request never releases its flag (-1: none)
  // LCB block epilogue (used by the epilogue instantiation only)
  CUtensorMap tm_res_r;     // residual of Y^R viewed as [R*o_r, d], box {64, 32} (loads)
  CUtensorMap tm_res_c;     // residual of Y^C viewed as [C*o_c, d], box {64, 32} (loads)
  CUtensorMap tm_res_cb;    // the same, box {64, 128}: one candidate's whole residual tile (B operand loads)
  EpiGroup epi_r, epi_c;
};
// Zeroes a[0:na] and b[0:nb] (the workspace header and the request ready flags) and lets the LCB kernel that
// follows on the stream start its set-up before it finishes (programmatic dependent launch).
cudaError_t launch_zero_ints(int* a, int na, int* b, int nb, cudaStream_t st);
cudaError_t launch_lcb_sm100(const LcbParams& p, int d, int n_c, bool epilogue, int grid, cudaStream_t st);

// fp32 CUDA-core IKBO-LCB (two launches: request GEMM, then candidate GEMM + fused Z add).
struct LcbF32Params {
  const float *x_req, *x_cand, *w_rr, *w_cr, *w_cc;
  float *y_req, *y_cand, *z;  // z: [R, o_c, d]
  const int32_t* cand_off;
  WsHeader* ws;
  int R, C, n_r, n_c, d, o_r, o_c;
};
cudaError_t launch_lcb_f32(const LcbF32Params& p, cudaStream_t st);

// Persistent IKBO-DCA kernel.
struct DcaParams {
  CUtensorMap tm_q;  // Q viewed as [C*q, H*dh], box {64, 128}
  CUtensorMap tm_k;  // K viewed as [T, H*dh],   box {64, 128}
  CUtensorMap tm_v;  // V viewed as [T, H*dh],   box {64, 128}
  CUtensorMap tm_o;  // O viewed as [C*q, H*dh], box {64, 32}   (stores)
  const int32_t* cand_off;
  const int32_t* seq_off;
  const int4* units;  // work-unit table {r, h, row0, w}: w = (split slot << 3) | (head pair << 2) | half (0 whole, 1, 2)
  int* ticket;        // work-unit counter (zeroed by the schedule kernel)
  float* split_buf;   // split units: per slot, half, tile, warp: unnormalised O [dh/4][32][4], m [32], l [32]
  int* split_cnt;     // split units: per slot, tile and warp, halves finished (zeroed by the schedule kernel)
  __nv_bfloat16* o;
  float* lse;
  WsHeader* ws;
  int R, q, H, n_units;
  float scale_log2;  // softmax scale * log2(e)
  long long wait_limit_ns;
};
cudaError_t launch_dca_sm100(const DcaParams& p, int dh, int grid, cudaStream_t st);

struct DcaSchedParams {
  const int32_t* cand_off;
  const int32_t* seq_off;
  int* scratch;  // 3R+1 ints
  int4* units;
  WsHeader* ws;
  int* ticket;     // the counter the attention kernel claims units from (zeroed here)
  int* split_cnt;  // [n_split * 8], zeroed here
  int R, q, H, rows_per_unit, max_units;
  int n_split;     // the last n_split units in claim order are split in two along the keys
  int pair_heads;  // a request's last chunk of <= 128 rows is one unit per head pair
};
cudaError_t launch_dca_schedule(const DcaSchedParams& p, cudaStream_t st);

// Dense projection GEMM  out[M, N] = in[M, K] . W[N, K]^T  (bf16 in/out, fp32 accumulate).
struct ProjParams {
  CUtensorMap tm_a;    // in  [M, K] (row stride lda), box {64, 128}
  CUtensorMap tm_b;    // W   [N, K], box {64, 256}
  __nv_bfloat16* out;  // [M, N] bf16, or null when out_f32 is given
  float* out_f32;      // [M, N] fp32 output instead of bf16 (or null)
  const float* add;    // IKBO broadcast-add: out[i, :] += add[m_i, :] with m_i from add_off (or null)
  const int32_t* add_off;  // [add_R + 1] CSR: rows add_off[r] .. add_off[r+1]-1 belong to r
  WsHeader* ws;
  int M, N, K, add_R;
  long long wait_limit_ns;
};
// W_fold[k, n*d + c] = sum_o W_q[k, o*d + c] W_CC[o, n]  (fp32 accumulate, bf16 out)
cudaError_t launch_chain_fold(const __nv_bfloat16* w_q, const __nv_bfloat16* w_cc, __nv_bfloat16* w_fold, int n_out,
                              int o_c, int n_c, int d, cudaStream_t st);
cudaError_t launch_proj_sm100(const ProjParams& p, int grid, cudaStream_t st);

// IKBO masked factorization machine (bf16 in, fp32 accumulate, bf16 out in aligned rows).
struct FmParams {
  CUtensorMap tm_xr;   // X^R as [R][n_r][d], box {64, 128, 1}   (A of request tiles; rows past n_r read 0)
  CUtensorMap tm_xrb;  // X^R as [R][n_r][d], box {64, n_b, 1}   (the resident B operand)
  CUtensorMap tm_xc;   // X^C as [C*n_c, d],  box {64, 128}      (A of candidate tiles)
  CUtensorMap tm_yr;   // Y^R as [R][n_r][ld_req], box {64, 32, 1} (stores)
  CUtensorMap tm_yc;   // Y^C as [C*n_c, ld_cand], box {64, 32}   (stores)
  const int32_t* cand_off;  // [R+1]
  const int32_t* unit_off;  // [R+1], from the schedule kernel
  WsHeader* ws;
  int R, n_r, n_c, n_b, ld_req, ld_cand, n_units, req_tiles;
  long long wait_limit_ns;
};
cudaError_t launch_fm_schedule(const int32_t* cand_off, int32_t* unit_off, int R, int n_c, int req_tiles,
                               cudaStream_t st);
cudaError_t launch_fm_sm100(const FmParams& p, int d, int grid, cudaStream_t st);
cudaError_t launch_pad_cols(const void* in, int64_t rows, int64_t cols, int64_t ld_in, void* out, int64_t ld_out,
                            int es, int grid, cudaStream_t st);

// out[k] = k for k = 0..n (the identity candidate map: every request its own single candidate).
cudaError_t launch_ident(int32_t* out, int n, cudaStream_t st);

// Explicit-expand baseline helpers.
cudaError_t launch_expand_rows(const void* src, void* dst, const int32_t* cand_off, int R, int C, int64_t row_bytes,
                               int64_t rows_per_item, cudaStream_t st);
cudaError_t launch_expand_kv(const void* k, const void* v, void* k_out, void* v_out, const int32_t* cand_off,
                             const int32_t* seq_off, int32_t* seq_off_out, int R, int c0, int c1, int64_t row_bytes,
                             cudaStream_t st);

}  // namespace rocs
