// lcb_sm100.cu -- IKBO-LCB on B200: one persistent, warp-specialised tcgen05 kernel.
//
// Computes the two-group ROCSified linear compression block of "ROCS: Request-Oriented
// Compute Sharing ..." (arXiv:2607.27744; paper-archivist notes, section 3.1.2, Eq. (6))
// through the IKBO decomposition of section 4.1, Eq. (14):
//     request tiles    [Y^R_r ; Z_r] = [W_RR ; W_CR] . X^R_r        (once per request)
//     candidate tiles  Y^C_i = W_CC . X^C_i + Z_{m_i}                (Z added in the epilogue)
// with the section 4.2 refinements re-designed for sm_100a:
//   * 4.2.1 broadcast-and-add fused into the candidate GEMM epilogue: Z_{m_i} is added in
//     registers and only Y^C is written;  here Z_r is staged ONCE per (CTA, request) into
//     tensor memory next to the accumulators and re-read from TMEM for every candidate of r.
//   * 4.2.2 mainloop/epilogue overlap: instead of ping-ponging consumer warp groups, a TMA
//     producer warp, a single-thread tcgen05.mma issuer and four epilogue warps run
//     concurrently; the accumulator is double-buffered in TMEM so the MMA of tile t+1
//     runs while the epilogue drains tile t.
//   * 4.2.3 request and candidate tiles in one persistent kernel: request tiles are claimed
//     first from a global ticket (Z tiles before Y^R tiles); a CTA moves to its candidate
//     range only once every request tile has been claimed, so a candidate epilogue only
//     ever waits (release/acquire flag, bounded) on a request tile that a running CTA owns.
//     Candidates are split into equal contiguous ranges, one per CTA (all candidate tiles
//     cost the same), which also keeps one request's Z resident for many tiles.
//   * 4.2.4 alignment: rows are 16-byte multiples by contract, so every operand moves by TMA.
//
// Tile shapes: M = 128 output rows (o_c, or a 128-row slice of o_r), N = d, K = n_c for a
// candidate tile (K-blocks of 64 for request tiles, K = n_r).  A = weights (K-major),
// B = embeddings X [K rows x d] (MN-major, d contiguous), both 128-byte swizzled.
#include "lcb_sm100.h"

namespace rocs {

namespace {

constexpr int kEpiWarps = 4;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreads = 192;
constexpr int kStages = 4;
constexpr uint32_t kSlot = 32768;  // one ring slot: a request k-block (A 16 KB + B <=16 KB) or one X^C tile
constexpr int OC = 128;

template <int D, int NC>
struct LcbSmem {
  static constexpr uint32_t kWcc = NC * OC * 2;           // W_CC resident, NC/64 boxes of [128 x 64]
  static constexpr uint32_t kXc = NC * D * 2;             // one candidate's X^C tile
  static constexpr uint32_t kStgHalf = 32 * 128;          // 32 rows x 64 bf16 (one TMA store box)
  static constexpr uint32_t kStgBuf = (D / 64) * kStgHalf;  // one warp's 32-row output tile
  static constexpr uint32_t off_wcc = 0;
  static constexpr uint32_t off_ring = kWcc;
  static constexpr uint32_t off_stg = off_ring + kStages * kSlot;
  static constexpr uint32_t off_bar = off_stg + kEpiWarps * 2 * kStgBuf;
  static constexpr uint32_t n_bars = 2 * kStages + 2 + 2 + 2 + 2 + 1 + 1;
  static constexpr uint32_t off_misc = off_bar + n_bars * 8;
  static constexpr uint32_t bytes = off_misc + 64;
  static constexpr uint32_t alloc_bytes = bytes + 1024;  // slack for 1024-byte alignment
  static constexpr uint32_t tmem_cols = (3 * D <= 256) ? 256 : 512;
  static_assert(kXc <= kSlot, "X^C tile must fit one slot");
  static_assert(alloc_bytes <= 232448, "shared memory budget");
};

}  // namespace

template <int D, int NC>
__global__ void __launch_bounds__(kThreads, 1) rocs_lcb_sm100_kernel(const __grid_constant__ LcbParams p) {
  using L = LcbSmem<D, NC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_wcc = smem + L::off_wcc;
  uint8_t* s_ring = smem + L::off_ring;
  uint8_t* s_stg = smem + L::off_stg;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::off_bar);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* wq_full = acc_empty + 2;
  uint64_t* wq_empty = wq_full + 2;
  uint64_t* wcc_bar = wq_empty + 2;
  uint64_t* drain_bar = wcc_bar + 1;
  int* s_wq = reinterpret_cast<int*>(smem + L::off_misc);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::off_misc + 16);
  int* s_abort = reinterpret_cast<int*>(smem + L::off_misc + 32);

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  const Ctl ctl{s_abort, p.ws, (unsigned long long)p.wait_limit_ns};

  const int R = p.R, C = p.C;
  const int mt_r = p.o_r / OC;                // 128-row slices of Y^R per request
  const int n_req_tiles = R * (1 + mt_r);     // Z tiles [0, R), then Y^R tiles
  const int kblocks = p.n_r / 64;
  const int G = gridDim.x, b = blockIdx.x;
  const int cbeg = (int)(((int64_t)C * b) / G), cend = (int)(((int64_t)C * (b + 1)) / G);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&acc_full[k], 1);
      mbar_init(&acc_empty[k], kEpiWarps);
      mbar_init(&wq_full[k], 1);
      mbar_init(&wq_empty[k], 1 + kEpiWarps);
    }
    mbar_init(wcc_bar, 1);
    mbar_init(drain_bar, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(s_tmem, L::tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      if (cbeg < cend) tma_prefetch_desc(&p.tm_xc);
      tma_prefetch_desc(&p.tm_xr);
      int n_issued = 0;
      bool ok = true;
      if (cbeg < cend) {
        mbar_arrive_expect_tx(wcc_bar, L::kWcc);
        for (int kc = 0; kc < NC / 64; ++kc) tma_load_2d(s_wcc + kc * 16384, &p.tm_wcc, wcc_bar, kc * 64, 0);
      }
      uint32_t s = 0, ph = 0, qs = 0, qph = 0;
      while (ok) {  // request phase: claim tiles until the ticket runs past the last request tile
        const int t = atomicAdd(&p.ws->counter, 1);
        const int item = t < n_req_tiles ? t : -1;
        if (!mbar_wait(&wq_empty[qs], qph ^ 1, ctl, 101)) { ok = false; break; }
        s_wq[qs] = item;
        mbar_arrive(&wq_full[qs]);
        if (++qs == 2) { qs = 0; qph ^= 1; }
        if (item < 0) break;
        int r, arow;
        const CUtensorMap* tmA;
        if (item < R) { r = item; arow = 0; tmA = &p.tm_wcr; }
        else { const int u = item - R; r = u / mt_r; arow = (u % mt_r) * OC; tmA = &p.tm_wrr; }
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1, ctl, 102)) { ok = false; break; }
          uint8_t* slot = s_ring + s * kSlot;
          mbar_arrive_expect_tx(&full[s], 16384 + 64 * D * 2);
          tma_load_2d(slot, tmA, &full[s], kb * 64, arow);
          for (int cc = 0; cc < D / 64; ++cc)
            tma_load_2d(slot + 16384 + cc * 8192, &p.tm_xr, &full[s], cc * 64, r * p.n_r + kb * 64);
          ++n_issued;
          if (++s == kStages) { s = 0; ph ^= 1; }
        }
      }
      for (int i = cbeg; ok && i < cend; ++i) {  // candidate phase
        if (!mbar_wait(&empty[s], ph ^ 1, ctl, 103)) { ok = false; break; }
        uint8_t* slot = s_ring + s * kSlot;
        mbar_arrive_expect_tx(&full[s], L::kXc);
        for (int cc = 0; cc < D / 64; ++cc) tma_load_2d(slot + cc * (NC * 128), &p.tm_xc, &full[s], cc * 64, i * NC);
        ++n_issued;
        if (++s == kStages) { s = 0; ph ^= 1; }
      }
      if (!ok) {  // let loads already in flight land before the CTA's shared memory goes away
        for (int k = n_issued > kStages ? n_issued - kStages : 0; k < n_issued; ++k)
          mbar_drain(&full[k % kStages], (k / kStages) & 1, 20000000ull);
        if (cbeg < cend) mbar_drain(wcc_bar, 0, 20000000ull);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ tcgen05 issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, D, false, true);
      uint32_t s = 0, ph = 0, ab = 0, aph = 0, qs = 0, qph = 0;
      bool ok = true;
      for (;;) {  // request tiles
        if (!mbar_wait(&wq_full[qs], qph, ctl, 201)) { ok = false; break; }
        const int item = s_wq[qs];
        mbar_arrive(&wq_empty[qs]);
        if (++qs == 2) { qs = 0; qph ^= 1; }
        if (item < 0) break;
        if (!mbar_wait(&acc_empty[ab], aph ^ 1, ctl, 202)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * D;
        for (int kb = 0; kb < kblocks && ok; ++kb) {
          if (!mbar_wait(&full[s], ph, ctl, 203)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(s_ring + s * kSlot);
          const uint64_t ad = sdesc_sw128(a0, 16, 1024), bd = sdesc_sw128(a0 + 16384, 8192, 1024);
#pragma unroll
          for (int kin = 0; kin < 4; ++kin)
            umma_ss(d_tmem, sdesc_add(ad, kin * 32), sdesc_add(bd, kin * 2048), idesc, (kb | kin) != 0);
          umma_commit(&empty[s]);
          if (++s == kStages) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        umma_commit(&acc_full[ab]);
        if (++ab == 2) { ab = 0; aph ^= 1; }
      }
      if (ok && cbeg < cend && !mbar_wait(wcc_bar, 0, ctl, 204)) ok = false;
      const uint64_t wccd = sdesc_sw128(smem_u32(s_wcc), 16, 1024);
      for (int i = cbeg; ok && i < cend; ++i) {  // candidate tiles
        if (!mbar_wait(&acc_empty[ab], aph ^ 1, ctl, 205)) { ok = false; break; }
        if (!mbar_wait(&full[s], ph, ctl, 206)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * D;
        const uint64_t bd = sdesc_sw128(smem_u32(s_ring + s * kSlot), NC * 128, 1024);
#pragma unroll
        for (int ks = 0; ks < NC / 16; ++ks)
          umma_ss(d_tmem, sdesc_add(wccd, (ks >> 2) * 16384 + (ks & 3) * 32), sdesc_add(bd, ks * 2048), idesc, ks != 0);
        umma_commit(&empty[s]);
        umma_commit(&acc_full[ab]);
        if (++s == kStages) { s = 0; ph ^= 1; }
        if (++ab == 2) { ab = 0; aph ^= 1; }
      }
      umma_commit(drain_bar);  // wait for every MMA this thread issued before TMEM is freed
      mbar_drain(drain_bar, 0, 50000000ull);
    }
  } else {
    // ------------------------------------------------------------------ epilogue warps 0..3
    const int ew = warp;                       // owns TMEM lanes / tile rows 32*ew .. 32*ew+31
    const uint32_t row = 32 * ew + lane;
    const uint32_t t_lane = (uint32_t)(32 * ew) << 16;
    const uint32_t z_tmem = tmem_base + t_lane + 2 * D;
    uint32_t ab = 0, aph = 0, qs = 0, qph = 0, sb = 0;
    bool ok = true;

    // write 32 accumulator columns (+ optional Z columns) of this thread's row as bf16 into the
    // warp's swizzled staging tile
    auto stage_chunk = [&](uint32_t stg, int cc, const uint32_t (&v)[32]) {
      uint32_t pk[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) pk[k] = pack_bf16x2(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]));
      const uint32_t half = stg + (cc >> 1) * L::kStgHalf + lane * 128;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t c16 = (cc & 1) * 4 + q;
        st_shared_v4(half + ((c16 ^ (lane & 7)) << 4), pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      }
    };
    auto store_tile = [&](const CUtensorMap* tm, uint32_t stg_off, int y0) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        for (int h = 0; h < D / 64; ++h) tma_store_2d(tm, s_stg + stg_off + h * L::kStgHalf, h * 64, y0);
        bulk_commit();
      }
    };
    auto acquire_stage = [&]() {  // staging buffer sb is free once the store issued two tiles ago has read it
      if (lane == 0) bulk_wait_read<1>();
      __syncwarp();
      return (uint32_t)((ew * 2 + sb) * L::kStgBuf);
    };

    for (;;) {  // request tiles
      if (!mbar_wait(&wq_full[qs], qph, ctl, 301)) { ok = false; break; }
      const int item = s_wq[qs];
      __syncwarp();
      if (lane == 0) mbar_arrive(&wq_empty[qs]);
      if (++qs == 2) { qs = 0; qph ^= 1; }
      if (item < 0) break;
      if (!mbar_wait(&acc_full[ab], aph, ctl, 302)) { ok = false; break; }
      tc_fence_after();
      const uint32_t acc = tmem_base + t_lane + ab * D;
      if (item < R) {
        // Z tile: fp32 into the workspace in a [R][d/4][o_c][4] layout so that a warp's 32 rows
        // of one 4-column group are 512 contiguous bytes (coalesced store here and load later).
        const int r = item;
        float* zr = p.zws + (size_t)r * OC * D;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32(acc + cc * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_global_v4(zr + ((size_t)(cc * 8 + j) * OC + row) * 4, v[4 * j], v[4 * j + 1], v[4 * j + 2],
                         v[4 * j + 3]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&acc_empty[ab]);
          __threadfence();
          if (r != p.skip_release) red_release_gpu_add(&p.flags[r], 1);  // 4 warps x 1 = this request's Z is complete
        }
      } else {
        const int u = item - R, r = u / mt_r, mt = u % mt_r;
        const uint32_t stg_off = acquire_stage();
        const uint32_t stg = smem_u32(s_stg + stg_off);
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32(acc + cc * 32, v);
          tmem_ld_wait();
          stage_chunk(stg, cc, v);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
        store_tile(&p.tm_yr, stg_off, r * p.o_r + mt * OC + 32 * ew);
        sb ^= 1;
      }
      if (++ab == 2) { ab = 0; aph ^= 1; }
    }

    if (ok && cbeg < cend) {  // candidate tiles
      // request of the first candidate: last r with cand_off[r] <= cbeg
      int lo = 0, hi = R - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.cand_off[mid] <= cbeg) lo = mid; else hi = mid - 1;
      }
      int r = lo, next_off = p.cand_off[r + 1], r_staged = -1;
      for (int i = cbeg; i < cend; ++i) {
        while (i >= next_off) {
          if (++r >= R) break;
          next_off = p.cand_off[r + 1];
        }
        if (r >= R || r < 0) { ctl.fail(ROCS_ERR_DEVICE_INDEX, 310); ok = false; break; }
        if (r != r_staged) {  // stage Z_r (this warp's 32 rows) into TMEM once per request
          if (!wait_flag_geq(&p.flags[r], kEpiWarps, ctl, 311)) { ok = false; break; }
          const float* zr = p.zws + (size_t)r * OC * D;
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t v[32];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 f = ld_global_cg_f4(zr + ((size_t)(cc * 8 + j) * OC + row) * 4);
              v[4 * j] = __float_as_uint(f.x);
              v[4 * j + 1] = __float_as_uint(f.y);
              v[4 * j + 2] = __float_as_uint(f.z);
              v[4 * j + 3] = __float_as_uint(f.w);
            }
            tmem_st32(z_tmem + cc * 32, v);
          }
          tmem_st_wait();
          r_staged = r;
        }
        if (!mbar_wait(&acc_full[ab], aph, ctl, 312)) { ok = false; break; }
        tc_fence_after();
        const uint32_t acc = tmem_base + t_lane + ab * D;
        const uint32_t stg_off = acquire_stage();
        const uint32_t stg = smem_u32(s_stg + stg_off);
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t v[32], z[32];
          tmem_ld32(acc + cc * 32, v);
          tmem_ld32(z_tmem + cc * 32, z);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) + __uint_as_float(z[k]));
          stage_chunk(stg, cc, v);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
        store_tile(&p.tm_yc, stg_off, i * OC + 32 * ew);
        sb ^= 1;
        if (++ab == 2) { ab = 0; aph ^= 1; }
      }
    }
    if (lane == 0) bulk_wait<0>();  // every TMA store of this warp has completed
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::tmem_cols);
  }
}

// ------------------------------------------------------------------------------------ host
template <int D, int NC>
static cudaError_t launch_t(const LcbParams& p, int grid, cudaStream_t st) {
  using L = LcbSmem<D, NC>;
  auto k = rocs_lcb_sm100_kernel<D, NC>;
  static bool attr_set = false;  // per instantiation; harmless if two threads race
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::alloc_bytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  k<<<grid, kThreads, L::alloc_bytes, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_lcb_sm100(const LcbParams& p, int d, int n_c, int grid, cudaStream_t st) {
  if (d == 128 && n_c == 64) return launch_t<128, 64>(p, grid, st);
  if (d == 128 && n_c == 128) return launch_t<128, 128>(p, grid, st);
  if (d == 64 && n_c == 64) return launch_t<64, 64>(p, grid, st);
  if (d == 64 && n_c == 128) return launch_t<64, 128>(p, grid, st);
  return cudaErrorInvalidValue;
}

}  // namespace rocs
