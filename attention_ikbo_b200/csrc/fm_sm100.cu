// fm_sm100.cu -- IKBO for the GLM-masked factorization machine on B200.
//
// Computes the two-group masked FM of "ROCS: Request-Oriented Compute Sharing ..." (arXiv:2607.27744;
// paper-archivist notes, section 3.1.4, Eq. (10)):
//     Y^R_r = X^R_r X^R_r^T                                  (once per request)
//     Y^C_i = [ X^C_i X^R_{m_i}^T ,  X^C_i X^C_i^T ]          (candidate rows)
// with the request-to-candidate broadcast kept inside the kernel (section 4.1): the candidates of a
// request are stacked into 128-row tiles (candidates never straddle a tile because n_c divides 128)
// and every tile multiplies against the SAME shared-memory copy of X^R_r, loaded once per (CTA,
// request).  The self block is the 128x128 Gram matrix of the tile, of which each row keeps the
// n_c columns of its own candidate.
//
// Output rows are written in an aligned layout (section 4.2.4): Y^C rows hold n_r + n_c values
// followed by zeros up to ld_cand, Y^R rows n_r values and zeros up to ld_req, where the leading
// dimensions are 16-byte multiples, so every row moves by TMA even when n_r + n_c is not.
//
// Roles: warps 0-7 epilogue (TMEM -> bf16 rows in the store's swizzled staging -> TMA stores), two
// warps per TMEM lane quarter splitting the output columns, so one warp's TMEM loads and shared-memory
// writes overlap the other's and the accumulator drains in about half the time; warp 8 TMA producer,
// warp 9 tcgen05 issuer.  TMEM: cross block [0, 256), self block [256, 384).
#include <type_traits>

#include "lcb_sm100.h"

namespace rocs {

namespace {
constexpr int kThreads = 320;
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kStages = 2;
constexpr int kMaxLd = 384;  // max output row length (n_r + n_c <= 256 + 128)

template <int D>
struct FmSmem {
  static constexpr uint32_t kBox = 128 * 128;             // one [128 rows x 64 K] bf16 box
  static constexpr uint32_t kXr = (D / 64) * 256 * 128;   // X^R_r resident: D/64 boxes of [<=256 rows x 64]
  static constexpr uint32_t kA = (D / 64) * kBox;          // one 128-row A tile
  static constexpr uint32_t kStgWarp = (kMaxLd / 64) * 32 * 128;  // one warp's 32 output rows
  static constexpr uint32_t off_xr = 0;
  static constexpr uint32_t off_ring = kXr;
  static constexpr uint32_t off_stg = off_ring + kStages * kA;
  static constexpr uint32_t off_bar = off_stg + 4 * kStgWarp;
  static constexpr uint32_t n_bars = 2 * kStages + 2 + 2 + 1;
  static constexpr uint32_t off_misc = off_bar + n_bars * 8;
  static constexpr uint32_t alloc_bytes = off_misc + 64 + 1024;
  static_assert(alloc_bytes <= 232448, "shared memory budget");
};

// unit u -> (request, local tile index) for a CTA walking a contiguous unit range
struct UnitWalk {
  int r, next;  // current request and the first unit of the next one
};
__device__ __forceinline__ UnitWalk unit_walk_begin(const int32_t* unit_off, int R, int u) {
  int lo = 0, hi = R - 1;  // last r with unit_off[r] <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (unit_off[mid] <= u) lo = mid; else hi = mid - 1;
  }
  return UnitWalk{lo, unit_off[lo + 1]};
}
__device__ __forceinline__ void unit_walk_advance(UnitWalk& w, const int32_t* unit_off, int R, int u) {
  while (u >= w.next && w.r + 1 < R) {
    ++w.r;
    w.next = unit_off[w.r + 1];
  }
}
}  // namespace

// unit_off[r] = sum over requests s < r of (req_tiles + ceil(N_s * n_c / 128)); unit_off[R] = total
__global__ void rocs_fm_schedule_kernel(const int32_t* cand_off, int32_t* unit_off, int R, int n_c, int req_tiles) {
  // the FM kernel may start its set-up now; it waits for this grid before reading the unit offsets
  asm volatile("griddepcontrol.launch_dependents;");
  __shared__ int s_part[1024];
  const int T = blockDim.x, t = threadIdx.x;
  const int per = (R + T - 1) / T;
  const int b0 = min(R, t * per), b1 = min(R, b0 + per);
  int sum = 0;
  for (int r = b0; r < b1; ++r) sum += req_tiles + ((cand_off[r + 1] - cand_off[r]) * n_c + 127) / 128;
  s_part[t] = sum;
  __syncthreads();
  for (int off = 1; off < T; off <<= 1) {
    const int v = t >= off ? s_part[t - off] : 0;
    __syncthreads();
    s_part[t] += v;
    __syncthreads();
  }
  int run = s_part[t] - sum;
  for (int r = b0; r < b1; ++r) {
    unit_off[r] = run;
    run += req_tiles + ((cand_off[r + 1] - cand_off[r]) * n_c + 127) / 128;
  }
  if (t == T - 1) unit_off[R] = s_part[T - 1];
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) rocs_fm_sm100_kernel(const __grid_constant__ FmParams p) {
  using L = FmSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_xr = smem + L::off_xr;
  uint8_t* s_ring = smem + L::off_ring;
  uint8_t* s_stg = smem + L::off_stg;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::off_bar);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* xr_full = bars + 2 * kStages;
  uint64_t* xr_empty = xr_full + 1;
  uint64_t* acc_full = xr_empty + 1;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain_bar = acc_empty + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::off_misc);
  int* s_abort = reinterpret_cast<int*>(smem + L::off_misc + 16);

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  const Ctl ctl{s_abort, p.ws, (unsigned long long)p.wait_limit_ns};
  const int R = p.R, n_c = p.n_c, n_r = p.n_r, n_b = p.n_b, rt = p.req_tiles;
  const int ubeg = (int)(((int64_t)p.n_units * blockIdx.x) / gridDim.x);
  const int uend = (int)(((int64_t)p.n_units * (blockIdx.x + 1)) / gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(xr_full, 1);
    mbar_init(xr_empty, 1);
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8);
    mbar_init(drain_bar, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  // launched as a programmatic dependent of the scheduling kernel: the set-up above overlapped it; every
  // role reads the unit offsets it wrote, so every thread waits for it here
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (ubeg < uend && warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_xr);
      tma_prefetch_desc(&p.tm_xrb);
      tma_prefetch_desc(&p.tm_xc);
      UnitWalk w = unit_walk_begin(p.unit_off, R, ubeg);
      int r_loaded = -1, n_xr = 0, n_issued = 0;
      uint32_t s = 0, ph = 0;
      bool ok = true;
      for (int u = ubeg; ok && u < uend; ++u) {
        unit_walk_advance(w, p.unit_off, R, u);
        const int r = w.r, lt = u - p.unit_off[r];
        if (r != r_loaded) {  // X^R_r into the resident buffer once the previous request's MMAs are done
          if (!mbar_wait(xr_empty, (n_xr & 1) ^ 1, ctl, 801)) { ok = false; break; }
          mbar_arrive_expect_tx(xr_full, (uint32_t)((D / 64) * n_b * 128));
          for (int kb = 0; kb < D / 64; ++kb) tma_load_3d(s_xr + kb * (256 * 128), &p.tm_xrb, xr_full, kb * 64, 0, r);
          r_loaded = r;
          ++n_xr;
        }
        if (!mbar_wait(&empty[s], ph ^ 1, ctl, 802)) { ok = false; break; }
        uint8_t* a = s_ring + s * L::kA;
        mbar_arrive_expect_tx(&full[s], L::kA);
        if (lt < rt) {  // request tile: rows lt*128.. of X^R_r (rows past n_r read as zero)
          for (int kb = 0; kb < D / 64; ++kb) tma_load_3d(a + kb * L::kBox, &p.tm_xr, &full[s], kb * 64, lt * 128, r);
        } else {  // candidate tile: stacked X^C rows of request r
          const int row0 = p.cand_off[r] * n_c + (lt - rt) * 128;
          for (int kb = 0; kb < D / 64; ++kb) tma_load_2d(a + kb * L::kBox, &p.tm_xc, &full[s], kb * 64, row0);
        }
        ++n_issued;
        if (++s == kStages) { s = 0; ph ^= 1; }
      }
      if (!ok) {  // let loads in flight land before shared memory goes away
        for (int k = n_issued > kStages ? n_issued - kStages : 0; k < n_issued; ++k)
          mbar_drain(&full[k % kStages], (k / kStages) & 1, 20000000ull);
        if (n_xr > 0) mbar_drain(xr_full, (n_xr - 1) & 1, 20000000ull);
      }
    }
  } else if (ubeg < uend && warp == kMmaWarp) {
    // ------------------------------------------------------------------ tcgen05 issuer
    if (lane == 0) {
      const uint32_t id_cross = idesc_bf16(128, n_b, false, false);
      constexpr uint32_t id_self = idesc_bf16(128, 128, false, false);
      const uint64_t xr_desc = sdesc_sw128(smem_u32(s_xr), 16, 1024);
      UnitWalk w = unit_walk_begin(p.unit_off, R, ubeg);
      int r_cur = -1, n_xr = 0;
      uint32_t s = 0, ph = 0, aph = 0;
      bool ok = true;
      for (int u = ubeg; ok && u < uend; ++u) {
        unit_walk_advance(w, p.unit_off, R, u);
        const int r = w.r, lt = u - p.unit_off[r];
        if (r != r_cur) {
          if (!mbar_wait(xr_full, n_xr & 1, ctl, 811)) { ok = false; break; }
          r_cur = r;
          ++n_xr;
        }
        if (!mbar_wait(&full[s], ph, ctl, 812)) { ok = false; break; }
        if (!mbar_wait(acc_empty, aph ^ 1, ctl, 813)) { ok = false; break; }
        tc_fence_after();
        const uint64_t a_desc = sdesc_sw128(smem_u32(s_ring + s * L::kA), 16, 1024);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          umma_ss(tmem_base, sdesc_add(a_desc, (ks >> 2) * L::kBox + (ks & 3) * 32),
                  sdesc_add(xr_desc, (ks >> 2) * (256 * 128) + (ks & 3) * 32), id_cross, ks != 0);
        if (lt >= rt) {  // candidate tile: the tile's own Gram matrix
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            umma_ss(tmem_base + 256, sdesc_add(a_desc, (ks >> 2) * L::kBox + (ks & 3) * 32),
                    sdesc_add(a_desc, (ks >> 2) * L::kBox + (ks & 3) * 32), id_self, ks != 0);
        }
        umma_commit(&empty[s]);
        umma_commit(acc_full);
        // last unit of this request in this CTA: the resident X^R may be replaced once these MMAs finish
        if (u + 1 >= uend || u + 1 >= w.next) umma_commit(xr_empty);
        if (++s == kStages) { s = 0; ph ^= 1; }
        aph ^= 1;
      }
      umma_commit(drain_bar);
      mbar_drain(drain_bar, 0, 50000000ull);
    }
  } else if (ubeg < uend && warp < 8) {
    // ------------------------------------------------------------------ epilogue warps 0..7
    // Two warps per TMEM lane quarter q share its 32 staging rows: warp q writes and stores the 64-column
    // boxes below b_split = floor(n_r / 64) (whole cross-block boxes), warp q + 4 the boxes from b_split
    // on (the rest of the cross block, the self block, the padding), so neither waits on the other.
    const int q = warp & 3, half = warp >> 2;
    const int b_split = n_r >> 6;
    const uint32_t t_lane = (uint32_t)(32 * q) << 16;
    uint8_t* stg = s_stg + q * L::kStgWarp;
    const uint32_t stg_u = smem_u32(stg);
    UnitWalk w = unit_walk_begin(p.unit_off, R, ubeg);
    uint32_t aph = 0;
    // address of the 16-byte unit u (8 columns) of this lane's staging row (64-column TMA boxes,
    // 128-byte swizzle)
    const uint32_t lane_base = stg_u + lane * 128, lx = lane & 7;
    auto unit_addr = [&](int u) -> uint32_t {
      return lane_base + (uint32_t)(u >> 3) * (32 * 128) + ((((uint32_t)u & 7) ^ lx) << 4);
    };
    auto pack = [&](const uint32_t (&v)[32], uint32_t (&pk)[16]) {
#pragma unroll
      for (int k = 0; k < 16; ++k) pk[k] = pack_bf16x2(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]));
    };
    // output columns [col0, col0 + cnt) from 32 values, col0 a multiple of 8, cnt even
    auto put_aligned = [&](int col0, const uint32_t (&v)[32], int cnt) {
      uint32_t pk[16];
      pack(v, pk);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (8 * j + 8 <= cnt) st_shared_v4(unit_addr((col0 >> 3) + j), pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
#pragma unroll
      for (int k = 0; k < 16; ++k)
        if (2 * k >= (cnt & ~7) && 2 * k < cnt) st_shared_u32(unit_addr((col0 >> 3) + (k >> 2)) + (k & 3) * 4, pk[k]);
    };
    // 32 output columns starting at col0 with col0 % 8 == S (S even, fixed at compile time): a
    // partial unit of (8 - S) / 2 pairs, three whole units, a partial unit of S / 2 pairs
    auto put_shifted = [&](auto s_ct, int col0, const uint32_t (&v)[32]) {
      constexpr int S = decltype(s_ct)::value;
      uint32_t pk[16];
      pack(v, pk);
      const int u0 = col0 >> 3;
      if constexpr (S == 0) {
#pragma unroll
        for (int j = 0; j < 4; ++j) st_shared_v4(unit_addr(u0 + j), pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
      } else {
        constexpr int h = (8 - S) / 2;  // pairs in the first partial unit
#pragma unroll
        for (int k = 0; k < h; ++k) st_shared_u32(unit_addr(u0) + S * 2 + 4 * k, pk[k]);
#pragma unroll
        for (int j = 0; j < 3; ++j)
          st_shared_v4(unit_addr(u0 + 1 + j), pk[h + 4 * j], pk[h + 4 * j + 1], pk[h + 4 * j + 2], pk[h + 4 * j + 3]);
#pragma unroll
        for (int k = 0; k < S / 2; ++k) st_shared_u32(unit_addr(u0 + 4) + 4 * k, pk[h + 12 + k]);
      }
    };
    // 64 columns (two 32-column loads in flight) per TMEM round trip
    auto load64 = [&](uint32_t taddr, uint32_t (&v)[2][32], bool second) {
      tmem_ld32(taddr, v[0]);
      if (second) tmem_ld32(taddr + 32, v[1]);
      tmem_ld_wait();
    };
    for (int u = ubeg; u < uend; ++u) {
      unit_walk_advance(w, p.unit_off, R, u);
      const int r = w.r, lt = u - p.unit_off[r];
      const bool cand = lt >= rt;
      const int t = cand ? lt - rt : lt;
      const int ncols = cand ? n_r + n_c : n_r, ld = cand ? p.ld_cand : p.ld_req, nbox = (ld + 63) >> 6;
      const int lrow0 = t * 128 + 32 * q;  // first row of this warp within the request's stacked rows
      const bool valid = cand ? lrow0 < (p.cand_off[r + 1] - p.cand_off[r]) * n_c : lrow0 < n_r;
      if (!mbar_wait(acc_full, aph, ctl, 821)) break;
      tc_fence_after();
      if (valid) {
        if (lane == 0) bulk_wait_read<0>();  // this warp's previous stores have read its staging boxes
        __syncwarp();
        if (half == 1)
          for (int uu = ncols >> 3; uu < nbox * 8; ++uu) st_shared_v4(unit_addr(uu), 0u, 0u, 0u, 0u);  // pad
        const int h_lo = half == 0 ? 0 : b_split, h_hi = half == 0 ? b_split : (n_r + 63) >> 6;
#pragma unroll 1
        for (int h = h_lo; h < h_hi; ++h) {  // cross block (columns past n_r are the zero rows of B)
          uint32_t v[2][32];
          const int ch = n_r - 64 * h;
          load64(tmem_base + t_lane + 64 * h, v, ch > 32);
          put_aligned(64 * h, v[0], min(32, ch));
          if (ch > 32) put_aligned(64 * h + 32, v[1], min(32, ch - 32));
        }
        if (cand && half == 1) {  // self block: the n_c Gram columns of this row's own candidate
          const int cb = (32 * q / n_c) * n_c, sh = n_r & 7;
#pragma unroll 1
          for (int h = 0; 64 * h < n_c; ++h) {
            uint32_t v[2][32];
            const bool two = n_c - 64 * h > 32;
            load64(tmem_base + t_lane + 256 + cb + 64 * h, v, two);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              if (c == 1 && !two) break;
              const int col0 = n_r + 64 * h + 32 * c;
              if (sh == 0) put_shifted(std::integral_constant<int, 0>{}, col0, v[c]);
              else if (sh == 2) put_shifted(std::integral_constant<int, 2>{}, col0, v[c]);
              else if (sh == 4) put_shifted(std::integral_constant<int, 4>{}, col0, v[c]);
              else put_shifted(std::integral_constant<int, 6>{}, col0, v[c]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      aph ^= 1;
      if (valid) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          for (int b = half == 0 ? 0 : b_split; b < (half == 0 ? b_split : nbox); ++b) {
            if (cand) tma_store_2d(&p.tm_yc, stg + b * (32 * 128), b * 64, p.cand_off[r] * n_c + lrow0);
            else tma_store_3d(&p.tm_yr, stg + b * (32 * 128), b * 64, lrow0, r);
          }
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

cudaError_t launch_fm_schedule(const int32_t* cand_off, int32_t* unit_off, int R, int n_c, int req_tiles,
                               cudaStream_t st) {
  rocs_fm_schedule_kernel<<<1, 1024, 0, st>>>(cand_off, unit_off, R, n_c, req_tiles);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_t(const FmParams& p, int grid, cudaStream_t st) {
  using L = FmSmem<D>;
  auto k = rocs_fm_sm100_kernel<D>;
  static std::atomic<uint64_t> optin_done{0};  // per instantiation, one bit per device
  cudaError_t e = ensure_smem_optin(optin_done, k, (int)L::alloc_bytes);
  if (e != cudaSuccess) return e;
  return launch_dependent(k, grid, kThreads, L::alloc_bytes, st, p);
}

cudaError_t launch_fm_sm100(const FmParams& p, int d, int grid, cudaStream_t st) {
  if (d == 128) return launch_t<128>(p, grid, st);
  if (d == 64) return launch_t<64>(p, grid, st);
  return cudaErrorInvalidValue;
}

// out[r, 0:cols] = in[r, 0:cols]; out[r, cols:ld_out] = 0  (elements of `es` bytes, es in {1, 2, 4, 8})
template <typename T>
__global__ void rocs_pad_cols_kernel(const T* in, int64_t rows, int64_t cols, int64_t ld_in, T* out, int64_t ld_out) {
  const int64_t n = rows * ld_out;
  for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < n; k += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = k / ld_out, c = k - r * ld_out;
    out[k] = c < cols ? in[r * ld_in + c] : T(0);
  }
}

cudaError_t launch_pad_cols(const void* in, int64_t rows, int64_t cols, int64_t ld_in, void* out, int64_t ld_out,
                            int es, int grid, cudaStream_t st) {
  switch (es) {
    case 1: rocs_pad_cols_kernel<uint8_t><<<grid, 256, 0, st>>>((const uint8_t*)in, rows, cols, ld_in, (uint8_t*)out, ld_out); break;
    case 2: rocs_pad_cols_kernel<uint16_t><<<grid, 256, 0, st>>>((const uint16_t*)in, rows, cols, ld_in, (uint16_t*)out, ld_out); break;
    case 4: rocs_pad_cols_kernel<uint32_t><<<grid, 256, 0, st>>>((const uint32_t*)in, rows, cols, ld_in, (uint32_t*)out, ld_out); break;
    case 8: rocs_pad_cols_kernel<uint64_t><<<grid, 256, 0, st>>>((const uint64_t*)in, rows, cols, ld_in, (uint64_t*)out, ld_out); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace rocs
