// rocs_abi.cu -- host side of the C ABI declared in include/rocs_ikbo.h: argument and CSR
// validation, workspace layout, TMA tensor-map construction and kernel launches.
// No entry point allocates or frees memory or synchronises a stream (except
// rocs_read_status, whose job is to synchronise and read).
#include <atomic>
#include <cmath>
#include <mutex>
#include <cstring>

#include "lcb_sm100.h"

namespace rocs {
int dca_rows_per_unit();
}

using namespace rocs;

namespace {

thread_local int g_last_launches = 0;

// A second stream per device (created on first use, kept for the process) with a fork and a join
// event, for launches that run beside the caller's stream inside one call.
struct AuxStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  bool ok = false;
};
AuxStream* aux_stream_for_current_device() {
  static std::mutex mu;
  static AuxStream aux[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  AuxStream& x = aux[dev];
  if (!x.ok) {
    if (cudaStreamCreateWithFlags(&x.s, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&x.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&x.join, cudaEventDisableTiming) != cudaSuccess)
      return nullptr;
    x.ok = true;
  }
  return &x;
}

// SM count of the calling thread's current device, cached per device (threads that race on a first call
// store the same value).
int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return n;
  static std::atomic<int> cache[64] = {};
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c) return c;
  }
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2-D bf16 tensor map [outer rows, inner cols] with a row pitch, 128-byte swizzle.
bool tmap_bf16(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_in,
               uint32_t box_out) {
  EncodeTiledFn f = encode_fn();
  if (!f || !base || inner == 0 || outer == 0) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_in, box_out};
  cuuint32_t es[2] = {1, 1};
  return f(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D view [outer2][outer1][inner] with rows of row_bytes and planes of plane_bytes
bool tmap_bf16_3d(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer1, uint64_t outer2,
                  uint64_t row_bytes, uint64_t plane_bytes, uint32_t box_in, uint32_t box_1) {
  EncodeTiledFn f = encode_fn();
  if (!f || !base || inner == 0 || outer1 == 0 || outer2 == 0) return false;
  cuuint64_t dims[3] = {inner, outer1, outer2};
  cuuint64_t strides[2] = {row_bytes, plane_bytes};
  cuuint32_t box[3] = {box_in, box_1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return f(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline size_t a256(size_t x) { return (x + 255) & ~size_t(255); }
inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// off[0] == 0, non-decreasing; *total = off[R]
int check_csr(const int32_t* off, int64_t R, int64_t* total) {
  if (!off) return ROCS_ERR_INVALID_ARG;
  if (off[0] != 0) return ROCS_ERR_BAD_OFFSETS;
  for (int64_t r = 0; r < R; ++r)
    if (off[r + 1] < off[r]) return ROCS_ERR_BAD_OFFSETS;
  *total = off[R];
  return ROCS_OK;
}

// ---------------------------------------------------------------- LCB
// workspace = [WsHeader][body]; body = [flags: R ints][Z: R * o_c * d fp32]
struct LcbLayout {
  size_t flags, z, body;
};
LcbLayout lcb_body(int64_t R, int64_t o_c, int64_t d) {
  LcbLayout L;
  L.flags = 0;
  L.z = a256((size_t)R * sizeof(int));
  L.body = L.z + (size_t)R * o_c * d * sizeof(float);
  return L;
}
size_t lcb_bytes(const rocs_lcb_args* a) { return sizeof(WsHeader) + lcb_body(a->R, a->o_c, a->d).body; }

int lcb_validate(const rocs_lcb_args* a, int64_t* C) {
  if (!a) return ROCS_ERR_INVALID_ARG;
  if (a->R < 0 || a->n_r <= 0 || a->n_c <= 0 || a->d <= 0 || a->o_r <= 0 || a->o_c <= 0) return ROCS_ERR_INVALID_ARG;
  if (a->R > (1 << 30)) return ROCS_ERR_UNSUPPORTED;
  if (a->dtype != ROCS_F32 && a->dtype != ROCS_BF16) return ROCS_ERR_INVALID_ARG;
  int rc = check_csr(a->cand_off_host, a->R, C);
  if (rc) return rc;
  if (a->R > 0 && !a->cand_off_dev) return ROCS_ERR_INVALID_ARG;
  const int64_t es = a->dtype == ROCS_BF16 ? 2 : 4;
  if ((a->d * es) % 16 != 0) return ROCS_ERR_UNSUPPORTED;  // row alignment contract
  if (a->R > 0 && (!a->x_req || !a->w_rr || !a->w_cr || !a->w_cc || !a->y_req)) return ROCS_ERR_INVALID_ARG;
  if (*C > 0 && (!a->x_cand || !a->y_cand)) return ROCS_ERR_INVALID_ARG;
  const void* ptrs[] = {a->x_req, a->x_cand, a->w_rr, a->w_cr, a->w_cc, a->y_req, a->y_cand};
  for (const void* p : ptrs)
    if (p && !al16(p)) return ROCS_ERR_INVALID_ARG;
  if (a->dtype == ROCS_BF16) {
    if (a->n_r % 64 || (a->n_c != 64 && a->n_c != 128) || (a->d != 64 && a->d != 128) || a->o_r % 128 ||
        a->o_c != 128)
      return ROCS_ERR_UNSUPPORTED;
    if ((a->n_r * 2) % 16 || (a->n_c * 2) % 16) return ROCS_ERR_UNSUPPORTED;
    if (*C * a->o_c >= (int64_t(1) << 31) || a->R * a->n_r >= (int64_t(1) << 31) || *C * a->n_c >= (int64_t(1) << 31))
      return ROCS_ERR_UNSUPPORTED;  // TMA coordinates are 32-bit
  } else {
    if (a->n_r > 1024 || a->n_c > 1024 || a->d > 1024) return ROCS_ERR_UNSUPPORTED;
  }
  return ROCS_OK;
}

struct LcbOpts {
  long long wait_ns = kDefaultWaitLimitNs;
  int skip_release = -1;  // fault injection only
  bool block = false;     // LCB block: fused per-group epilogue
  const rocs_lcb_epilogue* epi_r = nullptr;
  const rocs_lcb_epilogue* epi_c = nullptr;
};

int epi_validate(const rocs_lcb_epilogue* e) {
  if (!e) return ROCS_OK;
  if (e->norm < ROCS_NORM_NONE || e->norm > ROCS_NORM_RMS || e->act < ROCS_ACT_NONE || e->act > ROCS_ACT_GELU)
    return ROCS_ERR_INVALID_ARG;
  if (!(e->eps >= 0.0f) || !std::isfinite(e->eps)) return ROCS_ERR_INVALID_ARG;
  if ((e->residual && !al16(e->residual)) || (e->gamma && !al16(e->gamma)) || (e->beta && !al16(e->beta)))
    return ROCS_ERR_INVALID_ARG;  // residual by TMA, gamma/beta as float4
  if (e->bias && (reinterpret_cast<uintptr_t>(e->bias) & 3u)) return ROCS_ERR_INVALID_ARG;
  return ROCS_OK;
}

EpiGroup epi_group(const rocs_lcb_epilogue* e) {
  EpiGroup g;
  std::memset(&g, 0, sizeof(g));
  if (!e) return g;
  g.bias = e->bias;
  g.gamma = e->gamma;
  g.beta = e->beta;
  g.eps = e->eps;
  g.norm = e->norm;
  g.act = e->act;
  g.has_residual = e->residual != nullptr;
  return g;
}

int lcb_run(const rocs_lcb_args* a, int64_t C, WsHeader* hdr, uint8_t* w, cudaStream_t st, int* launches,
            const LcbOpts& opts = LcbOpts()) {
  const LcbLayout L = lcb_body(a->R, a->o_c, a->d);
  static_assert(sizeof(WsHeader) % sizeof(int) == 0, "header zeroed as ints");
  if (launch_zero_ints(reinterpret_cast<int*>(hdr), (int)(sizeof(WsHeader) / sizeof(int)), reinterpret_cast<int*>(w + L.flags),
                       (int)a->R, st) != cudaSuccess)
    return ROCS_ERR_CUDA;
  *launches = 1;  // the zeroing kernel
  if (a->R == 0) return ROCS_OK;
  if (a->dtype == ROCS_F32) {
    LcbF32Params p;
    p.x_req = static_cast<const float*>(a->x_req);
    p.x_cand = static_cast<const float*>(a->x_cand);
    p.w_rr = static_cast<const float*>(a->w_rr);
    p.w_cr = static_cast<const float*>(a->w_cr);
    p.w_cc = static_cast<const float*>(a->w_cc);
    p.y_req = static_cast<float*>(a->y_req);
    p.y_cand = static_cast<float*>(a->y_cand);
    p.z = reinterpret_cast<float*>(w + L.z);
    p.cand_off = a->cand_off_dev;
    p.ws = hdr;
    p.R = (int)a->R;
    p.C = (int)C;
    p.n_r = (int)a->n_r;
    p.n_c = (int)a->n_c;
    p.d = (int)a->d;
    p.o_r = (int)a->o_r;
    p.o_c = (int)a->o_c;
    if (launch_lcb_f32(p, st) != cudaSuccess) return ROCS_ERR_CUDA;
    *launches = 1 + (C > 0 ? 2 : 1);
    return ROCS_OK;
  }
  LcbParams p;
  std::memset(&p, 0, sizeof(p));
  const uint64_t d = a->d, rb = d * 2;
  bool ok = true;
  if (C > 0) {
    ok &= tmap_bf16(&p.tm_xc, a->x_cand, d, (uint64_t)C * a->n_c, rb, 64, (uint32_t)a->n_c);
    ok &= tmap_bf16(&p.tm_yc, a->y_cand, d, (uint64_t)C * a->o_c, rb, 64, 32);
    ok &= tmap_bf16(&p.tm_wcc, a->w_cc, a->n_c, a->o_c, a->n_c * 2, 64, 128);
  }
  ok &= tmap_bf16(&p.tm_xr, a->x_req, d, (uint64_t)a->R * a->n_r, rb, 64, 64);
  ok &= tmap_bf16(&p.tm_wrr, a->w_rr, a->n_r, a->o_r, a->n_r * 2, 64, 128);
  ok &= tmap_bf16(&p.tm_wcr, a->w_cr, a->n_r, a->o_c, a->n_r * 2, 64, 128);
  ok &= tmap_bf16(&p.tm_yr, a->y_req, d, (uint64_t)a->R * a->o_r, rb, 64, 32);
  if (opts.block) {
    p.epi_r = epi_group(opts.epi_r);
    p.epi_c = epi_group(opts.epi_c);
    // residual maps: the same boxes as the output stores (unused maps get any valid descriptor)
    p.tm_res_r = p.tm_yr;
    p.tm_res_c = p.tm_yr;
    p.tm_res_cb = p.tm_yr;
    if (p.epi_r.has_residual)
      ok &= tmap_bf16(&p.tm_res_r, opts.epi_r->residual, d, (uint64_t)a->R * a->o_r, rb, 64, 32);
    if (p.epi_c.has_residual && C > 0) {
      ok &= tmap_bf16(&p.tm_res_c, opts.epi_c->residual, d, (uint64_t)C * a->o_c, rb, 64, 32);
      ok &= tmap_bf16(&p.tm_res_cb, opts.epi_c->residual, d, (uint64_t)C * a->o_c, rb, 64, 128);
    }
  }
  if (!ok) return ROCS_ERR_CUDA;
  p.cand_off = a->cand_off_dev;
  p.zws = reinterpret_cast<float*>(w + L.z);
  p.flags = reinterpret_cast<int*>(w + L.flags);
  p.ws = hdr;
  p.R = (int)a->R;
  p.C = (int)C;
  p.n_r = (int)a->n_r;
  p.o_r = (int)a->o_r;
  p.wait_limit_ns = opts.wait_ns;
  p.skip_release = opts.skip_release;
  const int64_t n_req_tiles = a->R * (1 + a->o_r / 128);
  int64_t grid = C > n_req_tiles ? C : n_req_tiles;
  if (grid > sm_count()) grid = sm_count();
  if (grid < 1) grid = 1;
  if (launch_lcb_sm100(p, (int)a->d, (int)a->n_c, opts.block, (int)grid, st) != cudaSuccess) return ROCS_ERR_CUDA;
  *launches = 2;  // zeroing kernel + LCB kernel
  return ROCS_OK;
}

// ---------------------------------------------------------------- DCA
// workspace = [WsHeader][body]; body = [scratch: 3R+1 ints][work units: n_units int4]
// Work units: per request and head, chunks of 256 query rows (two 128-row tiles).  pair_heads: a request's last
// chunk of at most 128 rows is one unit for two heads (tile B = the next head), as the schedule kernel builds it.
int64_t dca_units(const rocs_dca_args* a, bool pair_heads = false) {
  const int rpu = dca_rows_per_unit();
  int64_t n = 0;
  for (int64_t r = 0; r < a->R; ++r) {
    const int64_t rows = a->q * (int64_t)(a->cand_off_host[r + 1] - a->cand_off_host[r]);
    const int64_t nb = (rows + rpu - 1) / rpu;
    if (pair_heads && a->H >= 2 && nb > 0 && rows - (nb - 1) * rpu <= rpu / 2)
      n += a->H * (nb - 1) + (a->H + 1) / 2;
    else
      n += a->H * nb;
  }
  return n;
}
// Head pairs are formed where both heads' K/V tiles fit the ring: dh = 64
bool dca_pair_heads(const rocs_dca_args* a) { return a->dh == 64; }
struct DcaLayout {
  size_t scratch, units, split_cnt, split_buf, body;
};
// n_units: work-table entries (a split unit counts twice); n_split: units split in two along the keys
DcaLayout dca_body(int64_t R, int64_t n_units, int64_t n_split = 0, int64_t dh = 128) {
  DcaLayout L;
  L.scratch = 0;
  L.units = a256((size_t)(3 * R + 1) * sizeof(int));
  L.split_cnt = a256(L.units + (size_t)n_units * sizeof(int4));
  L.split_buf = a256(L.split_cnt + (size_t)n_split * 8 * sizeof(int));
  // per split unit: 2 halves x 2 tiles x 4 warps x 32 rows x (dh O values + max + sum), fp32
  L.body = n_split ? L.split_buf + (size_t)n_split * 2 * 2 * 4 * 32 * (dh + 2) * sizeof(float) : L.units + (size_t)n_units * sizeof(int4);
  return L;
}
// Units split along the keys: the persistent grid claims units longest first, so with U units of equal
// length on G CTAs the last U mod G of them form a partial wave of full-length units.  Those are split in
// two, making the tail a wave of half-length work.  Only when every request with candidates has the same
// number of K/V tiles, at least two (each half then has keys): with ragged key lengths the longest-first
// claim order already evens out the tail, and splitting measured slower (merge and per-unit costs).
int64_t dca_split_count(const rocs_dca_args* a, int64_t n_units) {
  const int64_t G = sm_count();
  if (n_units <= G || n_units % G == 0) return 0;
  int64_t nkv = -1;
  for (int64_t r = 0; r < a->R; ++r) {
    if (a->cand_off_host[r + 1] == a->cand_off_host[r]) continue;
    const int64_t t = (a->seq_off_host[r + 1] - a->seq_off_host[r] + 127) / 128;
    if (t < 2 || (nkv >= 0 && t != nkv)) return 0;
    nkv = t;
  }
  return n_units % G;
}

int dca_validate(const rocs_dca_args* a, int64_t* C, int64_t* T) {
  if (!a) return ROCS_ERR_INVALID_ARG;
  if (a->R < 0 || a->q <= 0 || a->H <= 0 || a->dh <= 0) return ROCS_ERR_INVALID_ARG;
  if (a->dh != 64 && a->dh != 128) return ROCS_ERR_UNSUPPORTED;
  if (a->R > (1 << 28)) return ROCS_ERR_UNSUPPORTED;
  int rc = check_csr(a->cand_off_host, a->R, C);
  if (rc) return rc;
  rc = check_csr(a->seq_off_host, a->R, T);
  if (rc) return rc;
  if (a->R > 0 && (!a->cand_off_dev || !a->seq_off_dev)) return ROCS_ERR_INVALID_ARG;
  if (*C > 0 && (!a->q_ptr || !a->o_ptr)) return ROCS_ERR_INVALID_ARG;
  if (*T > 0 && (!a->k_ptr || !a->v_ptr)) return ROCS_ERR_INVALID_ARG;
  const void* ptrs[] = {a->q_ptr, a->k_ptr, a->v_ptr, a->o_ptr};
  for (const void* p : ptrs)
    if (p && !al16(p)) return ROCS_ERR_INVALID_ARG;
  if (a->lse_ptr && (reinterpret_cast<uintptr_t>(a->lse_ptr) & 3u)) return ROCS_ERR_INVALID_ARG;
  if (a->kv_ld != 0 && (a->kv_ld < a->H * a->dh || (a->kv_ld * 2) % 16)) return ROCS_ERR_UNSUPPORTED;
  if (*C * a->q >= (int64_t(1) << 31) || *T >= (int64_t(1) << 31) || a->H * a->dh >= (int64_t(1) << 20))
    return ROCS_ERR_UNSUPPORTED;
  return ROCS_OK;
}

// ticket: the work counter of this launch (default: the header's); two launches that run at the same
// time on one header use different counters
int dca_run(const rocs_dca_args* a, int64_t C, int64_t T, int64_t n_units, WsHeader* hdr, uint8_t* w,
            cudaStream_t st, int* launches, bool reset_header = true, int* ticket = nullptr, int64_t n_split = 0,
            bool pair_heads = false) {
  const DcaLayout L = dca_body(a->R, n_units + n_split, n_split, a->dh);
  if (n_units >= (int64_t(1) << 31)) return ROCS_ERR_UNSUPPORTED;
  if (reset_header && cudaMemsetAsync(hdr, 0, sizeof(WsHeader), st) != cudaSuccess) return ROCS_ERR_CUDA;
  if (n_units == 0) return ROCS_OK;
  DcaSchedParams sp;
  sp.cand_off = a->cand_off_dev;
  sp.seq_off = a->seq_off_dev;
  sp.scratch = reinterpret_cast<int*>(w + L.scratch);
  sp.units = reinterpret_cast<int4*>(w + L.units);
  sp.ws = hdr;
  sp.ticket = ticket ? ticket : &hdr->counter;
  sp.R = (int)a->R;
  sp.q = (int)a->q;
  sp.H = (int)a->H;
  sp.rows_per_unit = dca_rows_per_unit();
  sp.max_units = (int)(n_units + n_split);
  sp.n_split = (int)n_split;
  sp.pair_heads = pair_heads ? 1 : 0;
  sp.split_cnt = reinterpret_cast<int*>(w + L.split_cnt);
  if (launch_dca_schedule(sp, st) != cudaSuccess) return ROCS_ERR_CUDA;
  DcaParams p;
  std::memset(&p, 0, sizeof(p));
  const uint64_t hd = a->H * a->dh, rb = hd * 2, kvb = (a->kv_ld ? a->kv_ld : hd) * 2;
  bool ok = tmap_bf16(&p.tm_q, a->q_ptr, hd, (uint64_t)C * a->q, rb, 64, 128);
  ok &= tmap_bf16(&p.tm_o, a->o_ptr, hd, (uint64_t)C * a->q, rb, 64, 32);
  if (T > 0) {
    ok &= tmap_bf16(&p.tm_k, a->k_ptr, hd, (uint64_t)T, kvb, 64, 128);
    ok &= tmap_bf16(&p.tm_v, a->v_ptr, hd, (uint64_t)T, kvb, 64, 128);
  } else {  // never loaded (every request has zero keys); any valid descriptor will do
    p.tm_k = p.tm_q;
    p.tm_v = p.tm_q;
  }
  if (!ok) return ROCS_ERR_CUDA;
  p.cand_off = a->cand_off_dev;
  p.seq_off = a->seq_off_dev;
  p.units = sp.units;
  p.split_cnt = sp.split_cnt;
  p.split_buf = reinterpret_cast<float*>(w + L.split_buf);
  p.o = static_cast<__nv_bfloat16*>(a->o_ptr);
  p.lse = a->lse_ptr;
  p.ws = sp.ws;
  p.ticket = sp.ticket;
  p.R = (int)a->R;
  p.q = (int)a->q;
  p.H = (int)a->H;
  p.n_units = (int)(n_units + n_split);
  p.scale_log2 = a->scale * 1.4426950408889634f;
  p.wait_limit_ns = kDefaultWaitLimitNs;
  int64_t grid = n_units + n_split < sm_count() ? n_units + n_split : sm_count();
  if (launch_dca_sm100(p, (int)a->dh, (int)grid, st) != cudaSuccess) return ROCS_ERR_CUDA;
  *launches = 2;
  return ROCS_OK;
}

}  // namespace

namespace rocs {
int lcb_validate_ext(const rocs_lcb_args* a, int64_t* C) { return lcb_validate(a, C); }
int lcb_run_ext(const rocs_lcb_args* a, int64_t C, WsHeader* hdr, uint8_t* body, cudaStream_t st, int* launches) {
  return lcb_run(a, C, hdr, body, st, launches);
}
size_t lcb_body_bytes_ext(int64_t R, int64_t o_c, int64_t d) { return lcb_body(R, o_c, d).body; }
int dca_validate_ext(const rocs_dca_args* a, int64_t* C, int64_t* T) { return dca_validate(a, C, T); }
int dca_run_ext(const rocs_dca_args* a, int64_t C, int64_t T, int64_t n_units, WsHeader* hdr, uint8_t* body,
                cudaStream_t st, int* launches) {
  return dca_run(a, C, T, n_units, hdr, body, st, launches);
}
size_t dca_body_bytes_ext(int64_t R, int64_t n_units) { return dca_body(R, n_units).body; }
int64_t dca_units_ext(const rocs_dca_args* a) { return dca_units(a); }
void set_last_launches(int n) { g_last_launches = n; }
std::atomic<uint64_t>& configured_device_mask_ref() {
  static std::atomic<uint64_t> mask{0};
  return mask;
}
}  // namespace rocs

extern "C" {

size_t rocs_lcb_workspace_size(const rocs_lcb_args* a) {
  int64_t C;
  if (lcb_validate(a, &C) != ROCS_OK) return 0;
  return lcb_bytes(a);
}

int rocs_lcb_forward(const rocs_lcb_args* a, rocs_stream_t stream) {
  int64_t C = 0;
  int rc = lcb_validate(a, &C);
  if (rc) return rc;
  if (!a->workspace || a->workspace_bytes < lcb_bytes(a) || (reinterpret_cast<uintptr_t>(a->workspace) & 255))
    return ROCS_ERR_WORKSPACE;
  int launches = 0;
  WsHeader* hdr = static_cast<WsHeader*>(a->workspace);
  rc = lcb_run(a, C, hdr, reinterpret_cast<uint8_t*>(hdr + 1), reinterpret_cast<cudaStream_t>(stream), &launches);
  if (rc == ROCS_OK) g_last_launches = launches;
  return rc;
}

int rocs_lcb_forward_fault_injection(const rocs_lcb_args* a, rocs_stream_t stream, int64_t skip_release_request,
                                     int64_t wait_limit_ns) {
  int64_t C = 0;
  int rc = lcb_validate(a, &C);
  if (rc) return rc;
  if (a->dtype != ROCS_BF16) return ROCS_ERR_UNSUPPORTED;  // the ready flags exist in the bf16 kernel only
  if (skip_release_request < -1 || skip_release_request >= a->R) return ROCS_ERR_INVALID_ARG;
  if (wait_limit_ns < 1000000 || wait_limit_ns > 10000000000ll) return ROCS_ERR_INVALID_ARG;
  if (!a->workspace || a->workspace_bytes < lcb_bytes(a) || (reinterpret_cast<uintptr_t>(a->workspace) & 255))
    return ROCS_ERR_WORKSPACE;
  LcbOpts o;
  o.wait_ns = wait_limit_ns;
  o.skip_release = (int)skip_release_request;
  int launches = 0;
  WsHeader* hdr = static_cast<WsHeader*>(a->workspace);
  rc = lcb_run(a, C, hdr, reinterpret_cast<uint8_t*>(hdr + 1), reinterpret_cast<cudaStream_t>(stream), &launches, o);
  if (rc == ROCS_OK) g_last_launches = launches;
  return rc;
}

int rocs_lcb_block_forward_fault_injection(const rocs_lcb_args* a, const rocs_lcb_epilogue* epi_req,
                                           const rocs_lcb_epilogue* epi_cand, rocs_stream_t stream,
                                           int64_t skip_release_request, int64_t wait_limit_ns) {
  int64_t C = 0;
  int rc = lcb_validate(a, &C);
  if (rc) return rc;
  if (a->dtype != ROCS_BF16) return ROCS_ERR_UNSUPPORTED;
  if ((rc = epi_validate(epi_req)) || (rc = epi_validate(epi_cand))) return rc;
  if (skip_release_request < -1 || skip_release_request >= a->R) return ROCS_ERR_INVALID_ARG;
  if (wait_limit_ns < 1000000 || wait_limit_ns > 10000000000ll) return ROCS_ERR_INVALID_ARG;
  if (!a->workspace || a->workspace_bytes < lcb_bytes(a) || (reinterpret_cast<uintptr_t>(a->workspace) & 255))
    return ROCS_ERR_WORKSPACE;
  LcbOpts o;
  o.block = true;
  o.epi_r = epi_req;
  o.epi_c = epi_cand;
  o.wait_ns = wait_limit_ns;
  o.skip_release = (int)skip_release_request;
  int launches = 0;
  WsHeader* hdr = static_cast<WsHeader*>(a->workspace);
  rc = lcb_run(a, C, hdr, reinterpret_cast<uint8_t*>(hdr + 1), reinterpret_cast<cudaStream_t>(stream), &launches, o);
  if (rc == ROCS_OK) g_last_launches = launches;
  return rc;
}

int rocs_lcb_block_forward(const rocs_lcb_args* a, const rocs_lcb_epilogue* epi_req,
                           const rocs_lcb_epilogue* epi_cand, rocs_stream_t stream) {
  int64_t C = 0;
  int rc = lcb_validate(a, &C);
  if (rc) return rc;
  if (a->dtype != ROCS_BF16) return ROCS_ERR_UNSUPPORTED;  // the epilogue lives in the bf16 kernel
  if ((rc = epi_validate(epi_req)) || (rc = epi_validate(epi_cand))) return rc;
  if (!a->workspace || a->workspace_bytes < lcb_bytes(a) || (reinterpret_cast<uintptr_t>(a->workspace) & 255))
    return ROCS_ERR_WORKSPACE;
  LcbOpts o;
  o.block = true;
  o.epi_r = epi_req;
  o.epi_c = epi_cand;
  int launches = 0;
  WsHeader* hdr = static_cast<WsHeader*>(a->workspace);
  rc = lcb_run(a, C, hdr, reinterpret_cast<uint8_t*>(hdr + 1), reinterpret_cast<cudaStream_t>(stream), &launches, o);
  if (rc == ROCS_OK) g_last_launches = launches;
  return rc;
}

size_t rocs_dca_workspace_size(const rocs_dca_args* a) {
  int64_t C, T;
  if (dca_validate(a, &C, &T) != ROCS_OK) return 0;
  const int64_t n_units = dca_units(a, dca_pair_heads(a)), n_split = dca_split_count(a, n_units);
  return sizeof(WsHeader) + dca_body(a->R, n_units + n_split, n_split, a->dh).body;
}

int rocs_dca_forward(const rocs_dca_args* a, rocs_stream_t stream) {
  int64_t C = 0, T = 0;
  int rc = dca_validate(a, &C, &T);
  if (rc) return rc;
  const bool pair = dca_pair_heads(a);
  const int64_t n_units = dca_units(a, pair), n_split = dca_split_count(a, n_units);
  if (!a->workspace ||
      a->workspace_bytes < sizeof(WsHeader) + dca_body(a->R, n_units + n_split, n_split, a->dh).body ||
      (reinterpret_cast<uintptr_t>(a->workspace) & 255))
    return ROCS_ERR_WORKSPACE;
  int launches = 0;
  WsHeader* hdr = static_cast<WsHeader*>(a->workspace);
  rc = dca_run(a, C, T, n_units, hdr, reinterpret_cast<uint8_t*>(hdr + 1), reinterpret_cast<cudaStream_t>(stream),
               &launches, true, nullptr, n_split, pair);
  if (rc == ROCS_OK) g_last_launches = launches;
  return rc;
}

// ---- DCA block: projection GEMM + candidate-group and request-group attention
namespace {
struct BlockLayout {
  size_t ident, kv, body_c, body_r, bytes;
  int64_t C, T, units_c, units_r;
};
int block_layout(const rocs_dca_block_args* a, BlockLayout* L) {
  if (!a || a->R < 0 || a->q <= 0 || a->q_req <= 0 || a->H <= 0 || a->d_s <= 0) return ROCS_ERR_INVALID_ARG;
  if ((a->dh != 64 && a->dh != 128) || a->d_s % 64) return ROCS_ERR_UNSUPPORTED;
  int rc = check_csr(a->cand_off_host, a->R, &L->C);
  if (rc) return rc;
  rc = check_csr(a->seq_off_host, a->R, &L->T);
  if (rc) return rc;
  const int64_t hd = a->H * a->dh, rpu = dca_rows_per_unit();
  if (L->T * 4 * hd >= (int64_t(1) << 31) || L->C * a->q >= (int64_t(1) << 31)) return ROCS_ERR_UNSUPPORTED;
  L->units_c = 0;
  for (int64_t r = 0; r < a->R; ++r)
    L->units_c += a->H * ((a->q * (int64_t)(a->cand_off_host[r + 1] - a->cand_off_host[r]) + rpu - 1) / rpu);
  L->units_r = a->R * a->H * ((a->q_req + rpu - 1) / rpu);
  L->ident = sizeof(WsHeader);
  L->kv = a256(L->ident + (size_t)(a->R + 1) * 4);
  L->body_c = a256(L->kv + (size_t)L->T * 4 * hd * 2);
  L->body_r = a256(L->body_c + dca_body(a->R, L->units_c).body);
  L->bytes = L->body_r + dca_body(a->R, L->units_r).body;
  return ROCS_OK;
}
}  // namespace

extern "C" size_t rocs_dca_block_workspace_size(const rocs_dca_block_args* a) {
  BlockLayout L;
  return block_layout(a, &L) == ROCS_OK ? L.bytes : 0;
}

extern "C" int rocs_dca_block_forward(const rocs_dca_block_args* a, rocs_stream_t stream) {
  BlockLayout L;
  int rc = block_layout(a, &L);
  if (rc) return rc;
  if (!a->workspace || a->workspace_bytes < L.bytes || (reinterpret_cast<uintptr_t>(a->workspace) & 255))
    return ROCS_ERR_WORKSPACE;
  const void* ptrs[] = {a->s_seq, a->w_kv, a->q_c, a->q_r, a->o_c, a->o_r};
  for (const void* p : ptrs)
    if (p && !al16(p)) return ROCS_ERR_INVALID_ARG;
  if (a->R > 0 && (!a->cand_off_dev || !a->seq_off_dev || !a->w_kv || !a->q_r || !a->o_r)) return ROCS_ERR_INVALID_ARG;
  if (L.C > 0 && (!a->q_c || !a->o_c)) return ROCS_ERR_INVALID_ARG;
  if (L.T > 0 && !a->s_seq) return ROCS_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(a->workspace);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(w);
  if (cudaMemsetAsync(hdr, 0, sizeof(WsHeader), st) != cudaSuccess) return ROCS_ERR_CUDA;
  if (a->R == 0) return ROCS_OK;
  int launches = 0;
  const int64_t hd = a->H * a->dh;
  uint8_t* kv = w + L.kv;
  if (L.T > 0) {  // [K^C | V^C | K^R | V^R] = S . W_kv^T, once per request sequence row
    ProjParams pp;
    std::memset(&pp, 0, sizeof(pp));
    bool ok = tmap_bf16(&pp.tm_a, a->s_seq, a->d_s, L.T, a->d_s * 2, 64, 128);
    ok &= tmap_bf16(&pp.tm_b, a->w_kv, a->d_s, 4 * hd, a->d_s * 2, 64, 256);
    if (!ok) return ROCS_ERR_CUDA;
    pp.out = reinterpret_cast<__nv_bfloat16*>(kv);
    pp.ws = hdr;
    pp.M = (int)L.T;
    pp.N = (int)(4 * hd);
    pp.K = (int)a->d_s;
    pp.wait_limit_ns = kDefaultWaitLimitNs;
    const int64_t tiles = ((L.T + 127) / 128) * (4 * hd / 256);
    if (launch_proj_sm100(pp, (int)(tiles < sm_count() ? tiles : sm_count()), st) != cudaSuccess) return ROCS_ERR_CUDA;
    ++launches;
  }
  int32_t* ident = reinterpret_cast<int32_t*>(w + L.ident);
  if (launch_ident(ident, (int)a->R, st) != cudaSuccess) return ROCS_ERR_CUDA;
  ++launches;
  // The request group (one unit per request and head, few of them, each as long as a request's key
  // sequence) runs on a second stream at the same time as the candidate group: launched first, it
  // takes its SMs before the persistent candidate kernel fills the rest, instead of forming a tail.
  AuxStream* aux = aux_stream_for_current_device();
  if (!aux || cudaEventRecord(aux->fork, st) != cudaSuccess || cudaStreamWaitEvent(aux->s, aux->fork, 0) != cudaSuccess)
    return ROCS_ERR_CUDA;
  rocs_dca_args d;
  std::memset(&d, 0, sizeof(d));
  d.R = a->R;
  d.H = a->H;
  d.dh = a->dh;
  d.scale = a->scale;
  d.seq_off_dev = a->seq_off_dev;
  d.seq_off_host = a->seq_off_host;
  d.kv_ld = 4 * hd;
  d.q = a->q;
  d.cand_off_dev = a->cand_off_dev;
  d.cand_off_host = a->cand_off_host;
  d.q_ptr = a->q_c;
  d.k_ptr = kv;
  d.v_ptr = kv + hd * 2;
  d.o_ptr = a->o_c;
  d.lse_ptr = a->lse_c;
  int n = 0;
  // request group: every request is its own single "candidate" with q_r query tokens
  rocs_dca_args dr = d;
  dr.q = a->q_req;
  dr.cand_off_dev = ident;
  dr.cand_off_host = nullptr;
  dr.q_ptr = a->q_r;
  dr.k_ptr = kv + 2 * hd * 2;
  dr.v_ptr = kv + 3 * hd * 2;
  dr.o_ptr = a->o_r;
  dr.lse_ptr = a->lse_r;
  rc = dca_run(&dr, a->R, L.T, L.units_r, hdr, w + L.body_r, aux->s, &n, false, &hdr->counter2);
  if (rc) return rc;
  launches += n;
  if (cudaEventRecord(aux->join, aux->s) != cudaSuccess) return ROCS_ERR_CUDA;
  // candidate group (IKBO: K/V at batch B_r, m_i resolved in the kernel)
  if (L.C > 0) {
    rc = dca_run(&d, L.C, L.T, L.units_c, hdr, w + L.body_c, st, &n, false);
    if (rc) return rc;
    launches += n;
  }
  if (cudaStreamWaitEvent(st, aux->join, 0) != cudaSuccess) return ROCS_ERR_CUDA;
  g_last_launches = launches;
  return ROCS_OK;
}

// ---------------------------------------------------------------- masked FM + alignment transform
int64_t rocs_align_cols(int64_t cols, int64_t elem_bytes) {
  if (cols < 0 || (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8)) return -1;
  const int64_t q = 16 / elem_bytes;  // elements per 16 bytes
  return (cols + q - 1) / q * q;
}

int rocs_pad_cols(const void* src, int64_t rows, int64_t cols, int64_t ld_src, void* dst, int64_t ld_dst,
                  int64_t elem_bytes, rocs_stream_t stream) {
  if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8) return ROCS_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0 || ld_src < cols || ld_dst < cols) return ROCS_ERR_INVALID_ARG;
  if (rows == 0 || ld_dst == 0) return ROCS_OK;
  if (!dst || (cols > 0 && !src)) return ROCS_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) % (uintptr_t)elem_bytes)
    return ROCS_ERR_INVALID_ARG;
  const int64_t n = rows * ld_dst;
  int64_t grid = (n + 255) / 256;
  if (grid > 8 * sm_count()) grid = 8 * sm_count();
  if (launch_pad_cols(src, rows, cols, ld_src, dst, ld_dst, (int)elem_bytes, (int)grid,
                      reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ROCS_ERR_CUDA;
  g_last_launches = 1;
  return ROCS_OK;
}

static int fm_validate(const rocs_fm_args* a, int64_t* C, int64_t* ld_r, int64_t* ld_c) {
  if (!a) return ROCS_ERR_INVALID_ARG;
  if (a->R < 0 || a->n_r <= 0 || a->n_c <= 0 || a->d <= 0) return ROCS_ERR_INVALID_ARG;
  if ((a->d != 64 && a->d != 128) || (a->n_c != 32 && a->n_c != 64 && a->n_c != 128) || a->n_r > 256 || (a->n_r & 1))
    return ROCS_ERR_UNSUPPORTED;
  if (a->R > (1 << 28)) return ROCS_ERR_UNSUPPORTED;
  int rc = check_csr(a->cand_off_host, a->R, C);
  if (rc) return rc;
  if (a->R > 0 && (!a->cand_off_dev || !a->x_req || !a->y_req)) return ROCS_ERR_INVALID_ARG;
  if (*C > 0 && (!a->x_cand || !a->y_cand)) return ROCS_ERR_INVALID_ARG;
  const void* ptrs[] = {a->x_req, a->x_cand, a->y_req, a->y_cand};
  for (const void* p : ptrs)
    if (p && !al16(p)) return ROCS_ERR_INVALID_ARG;
  *ld_r = a->ld_req ? a->ld_req : rocs_align_cols(a->n_r, 2);
  *ld_c = a->ld_cand ? a->ld_cand : rocs_align_cols(a->n_r + a->n_c, 2);
  if (*ld_r < a->n_r || *ld_c < a->n_r + a->n_c) return ROCS_ERR_INVALID_ARG;
  if ((*ld_r * 2) % 16 || (*ld_c * 2) % 16 || *ld_r > 384 || *ld_c > 384) return ROCS_ERR_UNSUPPORTED;
  if (*C * a->n_c >= (int64_t(1) << 31) || a->R * a->n_r >= (int64_t(1) << 31)) return ROCS_ERR_UNSUPPORTED;
  return ROCS_OK;
}

static int64_t fm_units(const rocs_fm_args* a) {
  const int64_t rt = (a->n_r + 127) / 128;
  int64_t n = 0;
  for (int64_t r = 0; r < a->R; ++r) n += rt + ((int64_t)(a->cand_off_host[r + 1] - a->cand_off_host[r]) * a->n_c + 127) / 128;
  return n;
}

size_t rocs_fm_workspace_size(const rocs_fm_args* a) {
  int64_t C, lr, lc;
  if (fm_validate(a, &C, &lr, &lc) != ROCS_OK) return 0;
  return sizeof(WsHeader) + a256((size_t)(a->R + 1) * sizeof(int32_t));
}

int rocs_fm_forward(const rocs_fm_args* a, rocs_stream_t stream) {
  int64_t C = 0, ld_r = 0, ld_c = 0;
  int rc = fm_validate(a, &C, &ld_r, &ld_c);
  if (rc) return rc;
  const size_t need = sizeof(WsHeader) + a256((size_t)(a->R + 1) * sizeof(int32_t));
  if (!a->workspace || a->workspace_bytes < need || (reinterpret_cast<uintptr_t>(a->workspace) & 255))
    return ROCS_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  WsHeader* hdr = static_cast<WsHeader*>(a->workspace);
  int32_t* unit_off = reinterpret_cast<int32_t*>(hdr + 1);
  if (cudaMemsetAsync(hdr, 0, sizeof(WsHeader), st) != cudaSuccess) return ROCS_ERR_CUDA;
  if (a->R == 0) {
    g_last_launches = 0;
    return ROCS_OK;
  }
  const int64_t n_units = fm_units(a);
  if (n_units >= (int64_t(1) << 31)) return ROCS_ERR_UNSUPPORTED;
  const int rt = (int)((a->n_r + 127) / 128);
  if (launch_fm_schedule(a->cand_off_dev, unit_off, (int)a->R, (int)a->n_c, rt, st) != cudaSuccess) return ROCS_ERR_CUDA;
  FmParams p;
  std::memset(&p, 0, sizeof(p));
  const uint64_t d = a->d, n_r = a->n_r, R = a->R;
  const uint32_t n_b = (uint32_t)((n_r + 15) / 16 * 16);
  bool ok = tmap_bf16_3d(&p.tm_xr, a->x_req, d, n_r, R, d * 2, n_r * d * 2, 64, 128);
  ok &= tmap_bf16_3d(&p.tm_xrb, a->x_req, d, n_r, R, d * 2, n_r * d * 2, 64, n_b);
  ok &= tmap_bf16_3d(&p.tm_yr, a->y_req, (uint64_t)ld_r, n_r, R, (uint64_t)ld_r * 2, n_r * ld_r * 2, 64, 32);
  if (C > 0) {
    ok &= tmap_bf16(&p.tm_xc, a->x_cand, d, (uint64_t)C * a->n_c, d * 2, 64, 128);
    ok &= tmap_bf16(&p.tm_yc, a->y_cand, (uint64_t)ld_c, (uint64_t)C * a->n_c, (uint64_t)ld_c * 2, 64, 32);
  } else {  // no candidate tiles exist; any valid descriptor will do
    p.tm_xc = p.tm_xr;
    p.tm_yc = p.tm_yr;
  }
  if (!ok) return ROCS_ERR_CUDA;
  p.cand_off = a->cand_off_dev;
  p.unit_off = unit_off;
  p.ws = hdr;
  p.R = (int)R;
  p.n_r = (int)n_r;
  p.n_c = (int)a->n_c;
  p.n_b = (int)n_b;
  p.ld_req = (int)ld_r;
  p.ld_cand = (int)ld_c;
  p.n_units = (int)n_units;
  p.req_tiles = rt;
  p.wait_limit_ns = kDefaultWaitLimitNs;
  int64_t grid = n_units < sm_count() ? n_units : sm_count();
  if (launch_fm_sm100(p, (int)d, (int)grid, st) != cudaSuccess) return ROCS_ERR_CUDA;
  g_last_launches = 2;
  return ROCS_OK;
}

size_t rocs_proj_workspace_size(const rocs_proj_args* a) {
  (void)a;
  return sizeof(WsHeader);
}

// out[M, N] = in[M, K] (row stride lda) . w[N, K]^T (+ add[m_i, :]), bf16 or fp32 out; M > 0
static int proj_run(const void* in, int64_t lda, const void* w, void* out_bf16, float* out_f32, const float* add,
                    const int32_t* add_off, int64_t add_R, int64_t M, int64_t N, int64_t K, WsHeader* hdr,
                    cudaStream_t st) {
  ProjParams p;
  std::memset(&p, 0, sizeof(p));
  bool ok = tmap_bf16(&p.tm_a, in, (uint64_t)K, (uint64_t)M, (uint64_t)lda * 2, 64, 128);
  ok &= tmap_bf16(&p.tm_b, w, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, 64, 256);
  if (!ok) return ROCS_ERR_CUDA;
  p.out = static_cast<__nv_bfloat16*>(out_bf16);
  p.out_f32 = out_f32;
  p.add = add;
  p.add_off = add_off;
  p.add_R = (int)add_R;
  p.ws = hdr;
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.wait_limit_ns = kDefaultWaitLimitNs;
  const int64_t tiles = ((M + 127) / 128) * (N / 256);
  const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
  return launch_proj_sm100(p, grid, st) == cudaSuccess ? ROCS_OK : ROCS_ERR_CUDA;
}

int rocs_proj_forward(const rocs_proj_args* a, rocs_stream_t stream) {
  if (!a || a->M < 0 || a->N <= 0 || a->K <= 0) return ROCS_ERR_INVALID_ARG;
  if (a->N % 256 || a->K % 64) return ROCS_ERR_UNSUPPORTED;
  if (a->M >= (int64_t(1) << 31) || a->N >= (int64_t(1) << 31) || a->K >= (int64_t(1) << 31))
    return ROCS_ERR_UNSUPPORTED;
  if (a->M > 0 && (!a->in || !a->w || !a->out || !al16(a->in) || !al16(a->w) || !al16(a->out)))
    return ROCS_ERR_INVALID_ARG;
  if (!a->workspace || a->workspace_bytes < sizeof(WsHeader) || (reinterpret_cast<uintptr_t>(a->workspace) & 255))
    return ROCS_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(a->workspace, 0, sizeof(WsHeader), st) != cudaSuccess) return ROCS_ERR_CUDA;
  if (a->M == 0) {
    g_last_launches = 0;
    return ROCS_OK;
  }
  const int rc = proj_run(a->in, a->K, a->w, a->out, nullptr, nullptr, nullptr, 0, a->M, a->N, a->K,
                          static_cast<WsHeader*>(a->workspace), st);
  if (rc == ROCS_OK) g_last_launches = 1;
  return rc;
}

// ---------------------------------------------------------------- split chain
int rocs_chain_prepare_weights(const rocs_chain_weights_args* a, rocs_stream_t stream) {
  if (!a || a->n_out <= 0 || a->o_r <= 0 || a->o_c <= 0 || a->n_r <= 0 || a->n_c <= 0 || a->d <= 0)
    return ROCS_ERR_INVALID_ARG;
  if (a->n_out * a->n_c >= (int64_t(1) << 31) || a->d > 4096 || a->o_c > 4096) return ROCS_ERR_UNSUPPORTED;
  const void* ptrs[] = {a->w_q, a->w_rr, a->w_cr, a->w_cc, a->w_fold, a->w_rs};
  for (const void* p : ptrs)
    if (!p || !al16(p)) return ROCS_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t rr = (size_t)a->o_r * a->n_r * 2, cr = (size_t)a->o_c * a->n_r * 2;
  if (cudaMemcpyAsync(a->w_rs, a->w_rr, rr, cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(static_cast<uint8_t*>(a->w_rs) + rr, a->w_cr, cr, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return ROCS_ERR_CUDA;
  if (launch_chain_fold(static_cast<const __nv_bfloat16*>(a->w_q), static_cast<const __nv_bfloat16*>(a->w_cc),
                        static_cast<__nv_bfloat16*>(a->w_fold), (int)a->n_out, (int)a->o_c, (int)a->n_c, (int)a->d,
                        st) != cudaSuccess)
    return ROCS_ERR_CUDA;
  g_last_launches = 1;
  return ROCS_OK;
}

static int split_validate(const rocs_chain_split_args* a, int64_t* C) {
  if (!a) return ROCS_ERR_INVALID_ARG;
  if (a->R < 0 || a->n_out <= 0) return ROCS_ERR_INVALID_ARG;
  if (a->n_out % 256 || (a->o_c * a->d) % 64 || (a->n_c * a->d) % 64) return ROCS_ERR_UNSUPPORTED;
  // the request GEMM runs as an LCB with no candidates over the stacked [W_RR; W_CR]
  rocs_lcb_args l;
  std::memset(&l, 0, sizeof(l));
  l.R = a->R; l.n_r = a->n_r; l.n_c = a->n_c; l.d = a->d; l.o_r = a->o_r + a->o_c; l.o_c = a->o_c;
  l.dtype = ROCS_BF16; l.cand_off_dev = a->cand_off_dev; l.cand_off_host = a->cand_off_host;
  l.x_req = a->x_req; l.x_cand = a->x_cand; l.w_rr = a->w_rs; l.w_cr = a->w_rs; l.w_cc = a->w_rs;
  l.y_req = a->y_req; l.y_cand = a->q;
  int rc = lcb_validate(&l, C);
  if (rc) return rc;
  if (*C * a->n_c >= (int64_t(1) << 31) || *C * a->n_out >= (int64_t(1) << 31)) return ROCS_ERR_UNSUPPORTED;
  if (a->R > 0 && (!a->w_q || !al16(a->w_q))) return ROCS_ERR_INVALID_ARG;
  if (*C > 0 && (!a->w_fold || !a->q || !al16(a->w_fold) || !al16(a->q))) return ROCS_ERR_INVALID_ARG;
  return ROCS_OK;
}

static size_t split_bytes(const rocs_chain_split_args* a) {
  // [LCB workspace: header, flags, Z fp32 (request GEMM, discarded)] [q^R fp32 [R, n_out]]
  return a256(sizeof(WsHeader) + lcb_body(a->R, a->o_c, a->d).body) + (size_t)a->R * a->n_out * sizeof(float);
}

size_t rocs_chain_split_workspace_size(const rocs_chain_split_args* a) {
  int64_t C;
  if (split_validate(a, &C) != ROCS_OK) return 0;
  return split_bytes(a);
}

int rocs_chain_split_forward(const rocs_chain_split_args* a, rocs_stream_t stream) {
  int64_t C = 0;
  int rc = split_validate(a, &C);
  if (rc) return rc;
  if (!a->workspace || a->workspace_bytes < split_bytes(a) || (reinterpret_cast<uintptr_t>(a->workspace) & 255))
    return ROCS_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  WsHeader* hdr = static_cast<WsHeader*>(a->workspace);
  float* q_req = reinterpret_cast<float*>(static_cast<uint8_t*>(a->workspace) +
                                          a256(sizeof(WsHeader) + lcb_body(a->R, a->o_c, a->d).body));
  rocs_lcb_args l;
  std::memset(&l, 0, sizeof(l));
  l.R = a->R; l.n_r = a->n_r; l.n_c = a->n_c; l.d = a->d; l.o_r = a->o_r + a->o_c; l.o_c = a->o_c;
  l.dtype = ROCS_BF16; l.cand_off_dev = a->cand_off_dev; l.cand_off_host = a->cand_off_host;
  l.x_req = a->x_req; l.w_rr = a->w_rs; l.w_cr = static_cast<const uint8_t*>(a->w_rs) + (size_t)a->o_r * a->n_r * 2;
  l.w_cc = a->w_rs; l.y_req = a->y_req;
  int launches = 0;
  // 1. [Y^R_r; Z_r] = [W_RR; W_CR] X^R_r once per request (an LCB call without candidates)
  rc = lcb_run(&l, 0, hdr, reinterpret_cast<uint8_t*>(hdr + 1), st, &launches);
  if (rc) return rc;
  if (a->R == 0) {
    g_last_launches = launches;
    return ROCS_OK;
  }
  // 2. q^R_r = W_q vec(Z_r) in fp32 (Z_r = rows o_r.. of the request block, row stride (o_r + o_c) d)
  const int64_t zd = a->o_c * a->d, ld = (a->o_r + a->o_c) * a->d;
  rc = proj_run(static_cast<const uint8_t*>(a->y_req) + (size_t)a->o_r * a->d * 2, ld, a->w_q, nullptr, q_req, nullptr,
                nullptr, 0, a->R, a->n_out, zd, hdr, st);
  if (rc) return rc;
  ++launches;
  // 3. Q_i = W_fold vec(X^C_i) + q^R_{m_i}: the candidate GEMM with the broadcast-add fused
  if (C > 0) {
    rc = proj_run(a->x_cand, a->n_c * a->d, a->w_fold, a->q, nullptr, q_req, a->cand_off_dev, a->R, C, a->n_out,
                  a->n_c * a->d, hdr, st);
    if (rc) return rc;
    ++launches;
  }
  g_last_launches = launches;
  return ROCS_OK;
}

int rocs_read_status(const void* workspace, rocs_stream_t stream, int32_t* device_code, int32_t* detail) {
  if (!workspace || !device_code) return ROCS_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return ROCS_ERR_CUDA;
  int32_t h[2] = {0, 0};
  if (cudaMemcpy(h, workspace, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return ROCS_ERR_CUDA;
  *device_code = h[0];
  if (detail) *detail = h[1];
  return ROCS_OK;
}

const char* rocs_status_string(int code) {
  switch (code) {
    case ROCS_OK: return "ROCS_OK";
    case ROCS_ERR_INVALID_ARG: return "ROCS_ERR_INVALID_ARG";
    case ROCS_ERR_BAD_OFFSETS: return "ROCS_ERR_BAD_OFFSETS";
    case ROCS_ERR_UNSUPPORTED: return "ROCS_ERR_UNSUPPORTED";
    case ROCS_ERR_CUDA: return "ROCS_ERR_CUDA";
    case ROCS_ERR_TIMEOUT: return "ROCS_ERR_TIMEOUT";
    case ROCS_ERR_WORKSPACE: return "ROCS_ERR_WORKSPACE";
    case ROCS_ERR_DEVICE_INDEX: return "ROCS_ERR_DEVICE_INDEX";
    default: return "unknown rocs_status";
  }
}

int rocs_last_launch_count(void) { return g_last_launches; }

uint64_t rocs_configured_device_mask(void) { return configured_device_mask_ref().load(std::memory_order_acquire); }

}  // extern "C"
