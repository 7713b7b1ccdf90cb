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
//   * block epilogue (section 3.1.3, Eq. (7)-(8)): the candidate residual is accumulated by the tensor
//     core (an identity A operand against the residual tile, loaded with X^C), and each epilogue warp
//     reads its rows from TMEM once, hands the accumulator back and runs bias/norm/activation from
//     registers (setmaxnreg moves registers to the epilogue warpgroups).
//
// Tile shapes: M = 128 output rows (o_c, or a 128-row slice of o_r), N = d, K = n_c for a
// candidate tile (K-blocks of 64 for request tiles, K = n_r).  A = weights (K-major),
// B = embeddings X [K rows x d] (MN-major, d contiguous), both 128-byte swizzled.
#include <type_traits>

#include "lcb_sm100.h"

namespace rocs {

namespace {

constexpr int kWarpsPerGroup = 4;  // one epilogue group covers the 128 TMEM lanes (tile rows)

// NG epilogue groups of four warps, then the TMA producer warp and the tcgen05 issuer warp.
// NG = 1: the group drains both TMEM accumulator buffers in turn; NG = 2: group g drains buffer g
// only, so two tiles' epilogues run at once (used by the block epilogue, whose per-row work is long).
// NG = 2 launches a third full warpgroup (producer, issuer, two idle warps) so that setmaxnreg can
// move registers from it to the epilogue warps, which hold a whole output row in registers:
//   4 warps x 32 x kRegsCtl + 8 warps x 32 x kRegsEpi == 384 x kLaunchRegs,
// and per SM sub-partition (warps w, w+4, w+8) kRegsCtl + 2 kRegsEpi == 3 kLaunchRegs.
template <int NG>
struct LcbRoles {
  static constexpr int kEpiWarps = kWarpsPerGroup * NG;
  static constexpr int kProducerWarp = kEpiWarps;
  static constexpr int kMmaWarp = kEpiWarps + 1;
  static constexpr int kThreads = NG == 2 ? 384 : 32 * (kEpiWarps + 2);
  static constexpr uint32_t kLaunchRegs = 168, kRegsCtl = 56, kRegsEpi = 224;
};
static_assert(4 * 32 * LcbRoles<2>::kRegsCtl + 8 * 32 * LcbRoles<2>::kRegsEpi ==
                  LcbRoles<2>::kThreads * LcbRoles<2>::kLaunchRegs, "register split");
constexpr uint32_t kSlot = 32768;  // one ring slot: a request k-block (A 16 KB + B <=16 KB) or one X^C tile
constexpr int OC = 128;

template <int D, int NC, int NG>
struct LcbSmem {
  static constexpr int kEpiWarps = LcbRoles<NG>::kEpiWarps;
  static constexpr uint32_t kWcc = NC * OC * 2;           // W_CC resident, NC/64 boxes of [128 x 64]
  static constexpr uint32_t kXc = NC * D * 2;             // one candidate's X^C tile
  static constexpr uint32_t kRes = OC * D * 2;            // one candidate's residual tile [o_c x d]
  static constexpr uint32_t kEye = OC * OC * 2;           // identity [128 x 128], K-major A operand
  static constexpr uint32_t kStgHalf = 32 * 128;          // 32 rows x 64 bf16 (one TMA store box)
  static constexpr uint32_t kStgBuf = (D / 64) * kStgHalf;  // one warp's 32-row output tile
  // Block epilogue (NG = 2): where shared memory allows, the candidate residual is added by the tensor
  // core, Y^C += I . Res (an identity A operand against the residual tile as B, both bf16, accumulated
  // in fp32: every product is exact), so its rows travel with X^C through the ring and the epilogue
  // warps need one staging buffer each.  Otherwise two staging buffers per warp, so the next tile's
  // residual rows load while this tile is finished, and the ring gives up two stages for them.
  static constexpr bool kResMma =
      NG == 2 && kWcc + kEye + 2 * (kXc + kRes) + 8 * kStgBuf + 2 * D * 4 + 2048 <= 232448 - 1024;
  // Plain LCB (NG = 1): the output stream is twice the input stream, so shared memory goes to output
  // staging first (more TMA stores in flight per warp), then to the X^C ring: 3 stages and 3 staging
  // buffers per warp at n_c = 64 (a 16 KB X^C tile per 32 KB slot), 2 and 4 at n_c = 128.
  static constexpr int kStages = NG == 2 ? 2 : (NC == 64 ? 3 : 2);
  static constexpr int kStgPerWarp = kResMma ? 1 : (NG == 1 ? (NC == 64 ? 3 : 4) : 2);  // per epilogue warp
  // one ring slot: a request k-block (A 16 KB + B <= 16 KB) or one X^C tile (+ its residual tile)
  static constexpr uint32_t kSlotSz = kResMma && kXc + kRes > kSlot ? kXc + kRes : kSlot;
  static constexpr uint32_t off_wcc = 0;
  static constexpr uint32_t off_eye = kWcc;
  static constexpr uint32_t off_ring = off_eye + (kResMma ? kEye : 0);
  static constexpr uint32_t off_stg = off_ring + kStages * kSlotSz;
  static constexpr uint32_t off_par = off_stg + kEpiWarps * kStgPerWarp * kStgBuf;
  static constexpr uint32_t kPar = NG == 2 ? 2 * D * 4 : 0;  // block epilogue: candidate gamma, beta (fp32)
  static constexpr uint32_t off_bar = off_par + kPar;
  static constexpr uint32_t n_bars = 2 * kStages + 2 + 2 + 2 + 2 + 1 + 1 + kEpiWarps;
  static constexpr uint32_t off_misc = off_bar + n_bars * 8;
  static constexpr uint32_t bytes = off_misc + 64;
  static constexpr uint32_t alloc_bytes = bytes + 1024;  // slack for 1024-byte alignment
  static constexpr uint32_t tmem_cols = ((2 + NG) * D <= 256) ? 256 : 512;  // 2 accumulators + NG Z slots
  static_assert((2 + NG) * D <= 512, "tensor memory budget");
  static_assert(kXc <= kSlot, "X^C tile must fit one slot");
  static_assert(kSlotSz % 1024 == 0 && off_ring % 1024 == 0, "swizzled operands need 1024-byte alignment");
  static_assert(alloc_bytes <= 232448, "shared memory budget");
};

}  // namespace

// EPI_C < 0: the plain LCB.  EPI_C >= 0: the LCB block epilogue, with the candidate group's
// activation EPI_C fixed at compile time (the request group's is read at run time).
template <int D, int NC, int EPI_C, int NG = EPI_C >= 0 ? 2 : 1>
__global__ void __launch_bounds__(LcbRoles<NG>::kThreads, 1) rocs_lcb_sm100_kernel(const __grid_constant__ LcbParams p) {
  using L = LcbSmem<D, NC, NG>;
  constexpr bool EPI = EPI_C >= 0;
  constexpr int kEpiWarps = LcbRoles<NG>::kEpiWarps;
  constexpr int kProducerWarp = LcbRoles<NG>::kProducerWarp;
  constexpr int kMmaWarp = LcbRoles<NG>::kMmaWarp;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_wcc = smem + L::off_wcc;
  uint8_t* s_ring = smem + L::off_ring;
  uint8_t* s_stg = smem + L::off_stg;
  float* s_gb = reinterpret_cast<float*>(smem + L::off_par);  // block epilogue: gamma_C [D], beta_C [D]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::off_bar);
  uint64_t* full = bars;
  uint64_t* empty = bars + L::kStages;
  uint64_t* acc_full = bars + 2 * L::kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* wq_full = acc_empty + 2;
  uint64_t* wq_empty = wq_full + 2;
  uint64_t* wcc_bar = wq_empty + 2;
  uint64_t* drain_bar = wcc_bar + 1;
  uint64_t* res_bar = drain_bar + 1;  // [kEpiWarps]: residual tile of each epilogue warp landed (block epilogue)
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
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&acc_full[k], 1);
      mbar_init(&acc_empty[k], kWarpsPerGroup);  // the four warps of the group that drains buffer k
      mbar_init(&wq_full[k], 1);
      mbar_init(&wq_empty[k], 1 + kEpiWarps);
    }
    mbar_init(wcc_bar, 1);
    mbar_init(drain_bar, 1);
    for (int k = 0; k < kEpiWarps; ++k) mbar_init(&res_bar[k], 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(s_tmem, L::tmem_cols);
    tmem_relinquish();
  }
  if constexpr (EPI) {
    if (warp < kEpiWarps)
      for (int k = threadIdx.x; k < D; k += 32 * kEpiWarps) {
        s_gb[k] = p.epi_c.gamma ? p.epi_c.gamma[k] : 1.0f;
        s_gb[D + k] = p.epi_c.beta ? p.epi_c.beta[k] : 0.0f;
      }
    if constexpr (L::kResMma) {
      // identity A operand in the layout a 128-byte-swizzled TMA load of [128 rows x 64] boxes gives:
      // row m of box b at b*16 KB + m*128 bytes, its 16-byte chunk j stored at position j ^ (m & 7)
      if (threadIdx.x < OC) {
        const uint32_t m = threadIdx.x;
        uint8_t* s_eye = smem + L::off_eye;
#pragma unroll
        for (uint32_t bx = 0; bx < OC / 64; ++bx)
#pragma unroll
          for (uint32_t j = 0; j < 8; ++j) {
            uint32_t w[4] = {0u, 0u, 0u, 0u};
            if (bx == (m >> 6) && j == ((m & 63) >> 3)) w[(m & 7) >> 1] = (m & 1) ? 0x3F800000u : 0x00003F80u;
            st_shared_v4(smem_u32(s_eye + bx * 16384 + m * 128 + ((j ^ (m & 7)) << 4)), w[0], w[1], w[2], w[3]);
          }
        fence_proxy_async_smem();
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  if (warp >= kEpiWarps) {
   // NG = 2: warpgroup 2 hands registers to the epilogue warpgroups, then producer / issuer / idle
   if constexpr (NG == 2) reg_dealloc<LcbRoles<NG>::kRegsCtl>();
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
      // launched as a programmatic dependent of the kernel that zeroes the ticket and the ready flags: the
      // set-up above overlapped it; they are zero and visible to the whole grid after this wait
      asm volatile("griddepcontrol.wait;" ::: "memory");
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
          uint8_t* slot = s_ring + s * L::kSlotSz;
          mbar_arrive_expect_tx(&full[s], 16384 + 64 * D * 2);
          tma_load_2d(slot, tmA, &full[s], kb * 64, arow);
          for (int cc = 0; cc < D / 64; ++cc)
            tma_load_2d(slot + 16384 + cc * 8192, &p.tm_xr, &full[s], cc * 64, r * p.n_r + kb * 64);
          ++n_issued;
          if (++s == L::kStages) { s = 0; ph ^= 1; }
        }
      }
      for (int i = cbeg; ok && i < cend; ++i) {  // candidate phase
        if (!mbar_wait(&empty[s], ph ^ 1, ctl, 103)) { ok = false; break; }
        uint8_t* slot = s_ring + s * L::kSlotSz;
        const bool res_mma = L::kResMma && p.epi_c.has_residual;
        mbar_arrive_expect_tx(&full[s], L::kXc + (res_mma ? L::kRes : 0u));
        for (int cc = 0; cc < D / 64; ++cc) {
          // LCB block: X^C is read once; evict-first keeps the residual rows prefetched for the epilogue in L2
          if constexpr (EPI) tma_load_2d_hint(slot + cc * (NC * 128), &p.tm_xc, &full[s], cc * 64, i * NC, l2_evict_first());
          else tma_load_2d(slot + cc * (NC * 128), &p.tm_xc, &full[s], cc * 64, i * NC);
        }
        if (res_mma)  // the residual tile [o_c rows x d] as the B operand of Y^C += I . Res (read once)
          for (int cc = 0; cc < D / 64; ++cc)
            tma_load_2d_hint(slot + L::kXc + cc * (OC * 128), &p.tm_res_cb, &full[s], cc * 64, i * OC, l2_evict_first());
        ++n_issued;
        if (++s == L::kStages) { s = 0; ph ^= 1; }
      }
      if (!ok) {  // let loads already in flight land before the CTA's shared memory goes away
        for (int k = n_issued > L::kStages ? n_issued - L::kStages : 0; k < n_issued; ++k)
          mbar_drain(&full[k % L::kStages], (k / L::kStages) & 1, 20000000ull);
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
          const uint32_t a0 = smem_u32(s_ring + s * L::kSlotSz);
          const uint64_t ad = sdesc_sw128(a0, 16, 1024), bd = sdesc_sw128(a0 + 16384, 8192, 1024);
#pragma unroll
          for (int kin = 0; kin < 4; ++kin)
            umma_ss(d_tmem, sdesc_add(ad, kin * 32), sdesc_add(bd, kin * 2048), idesc, (kb | kin) != 0);
          umma_commit(&empty[s]);
          if (++s == L::kStages) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        umma_commit(&acc_full[ab]);
        if (++ab == 2) { ab = 0; aph ^= 1; }
      }
      if (ok && cbeg < cend && !mbar_wait(wcc_bar, 0, ctl, 204)) ok = false;
      const uint64_t wccd = sdesc_sw128(smem_u32(s_wcc), 16, 1024);
      const uint64_t eyed = sdesc_sw128(smem_u32(smem + L::off_eye), 16, 1024);
      const bool res_mma = L::kResMma && p.epi_c.has_residual;
      for (int i = cbeg; ok && i < cend; ++i) {  // candidate tiles
        if (!mbar_wait(&acc_empty[ab], aph ^ 1, ctl, 205)) { ok = false; break; }
        if (!mbar_wait(&full[s], ph, ctl, 206)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * D;
        const uint64_t bd = sdesc_sw128(smem_u32(s_ring + s * L::kSlotSz), NC * 128, 1024);
#pragma unroll
        for (int ks = 0; ks < NC / 16; ++ks)
          umma_ss(d_tmem, sdesc_add(wccd, (ks >> 2) * 16384 + (ks & 3) * 32), sdesc_add(bd, ks * 2048), idesc, ks != 0);
        if (res_mma) {  // Y^C += I . Res: K runs over the residual tile's o_c rows
          const uint64_t rd = sdesc_sw128(smem_u32(s_ring + s * L::kSlotSz + L::kXc), OC * 128, 1024);
#pragma unroll
          for (int ks = 0; ks < OC / 16; ++ks)
            umma_ss(d_tmem, sdesc_add(eyed, (ks >> 2) * 16384 + (ks & 3) * 32), sdesc_add(rd, ks * 2048), idesc, 1u);
        }
        umma_commit(&empty[s]);
        umma_commit(&acc_full[ab]);
        if (++s == L::kStages) { s = 0; ph ^= 1; }
        if (++ab == 2) { ab = 0; aph ^= 1; }
      }
      umma_commit(drain_bar);  // wait for every MMA this thread issued before TMEM is freed
      mbar_drain(drain_bar, 0, 50000000ull);
    }
   }
  } else {
    // ------------------------------------------------------------------ epilogue warps
    if constexpr (NG == 2) reg_alloc<LcbRoles<NG>::kRegsEpi>();
    const int ew = warp;                 // epilogue warp index: staging buffers, residual barrier
    const int quarter = warp & 3;        // owns TMEM lanes / tile rows 32*quarter .. 32*quarter+31
    const int grp = warp >> 2;           // NG = 2: drains accumulator buffer grp only
    const uint32_t row = 32 * quarter + lane;
    const uint32_t t_lane = (uint32_t)(32 * quarter) << 16;
    const uint32_t z_tmem = tmem_base + t_lane + (2 + grp) * D;  // this group's copy of Z_r
    uint32_t ab = 0, aphs = 0, qs = 0, qph = 0, sb = 0;  // aphs bit b: phase of accumulator buffer b
    bool ok = true;
    auto mine = [&]() { return NG == 1 || (int)ab == grp; };

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
    auto store_tile = [&](const CUtensorMap* tm, uint32_t stg_off, int y0, bool stream = false) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (stream) {  // written once and not read again here: leaves L2 first
          const uint64_t pol = l2_evict_first();
          for (int h = 0; h < D / 64; ++h) tma_store_2d_hint(tm, s_stg + stg_off + h * L::kStgHalf, h * 64, y0, pol);
        } else {
          for (int h = 0; h < D / 64; ++h) tma_store_2d(tm, s_stg + stg_off + h * L::kStgHalf, h * 64, y0);
        }
        bulk_commit();
      }
    };
    // block epilogue: fetch the residual rows of this warp's 32-row output tile into its staging
    // buffer (same swizzled box as the store), add them, write the finished rows back in place
    uint32_t rph = 0;
    auto load_residual = [&](const CUtensorMap* tm, uint32_t stg_off, int y0) {  // its last use: evict-first
      if (lane == 0) {
        mbar_arrive_expect_tx(&res_bar[ew], (uint32_t)(D * 32 * 2));
        const uint64_t pol = l2_evict_first();
        for (int h = 0; h < D / 64; ++h)
          tma_load_2d_hint(s_stg + stg_off + h * L::kStgHalf, tm, &res_bar[ew], h * 64, y0, pol);
      }
    };
    auto drain_residual = [&]() {  // a wait failed with a residual load possibly in flight
      if (lane == 0) mbar_drain(&res_bar[ew], rph, 20000000ull);
      __syncwarp();
    };
    // One 64-column chunk of this thread's row (= one staging half) as 32 pairs: accumulator (+ Z)
    // or + a per-row constant, + the residual from the staging buffer (loaded there in the store's
    // swizzled layout).  Both 32-column TMEM loads (and both Z loads) are in flight before the wait.
    auto load_chunk = [&](float2 (&xs)[32], uint32_t acc, bool use_z, float add, bool res, uint32_t stg, int c) {
      if (use_z) {
        uint32_t v0[32], v1[32], z0[32], z1[32];
        tmem_ld32(acc + c * 64, v0);
        tmem_ld32(z_tmem + c * 64, z0);
        tmem_ld32(acc + c * 64 + 32, v1);
        tmem_ld32(z_tmem + c * 64 + 32, z1);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          xs[k] = __fadd2_rn(make_float2(__uint_as_float(v0[2 * k]), __uint_as_float(v0[2 * k + 1])),
                             make_float2(__uint_as_float(z0[2 * k]), __uint_as_float(z0[2 * k + 1])));
          xs[16 + k] = __fadd2_rn(make_float2(__uint_as_float(v1[2 * k]), __uint_as_float(v1[2 * k + 1])),
                                  make_float2(__uint_as_float(z1[2 * k]), __uint_as_float(z1[2 * k + 1])));
        }
      } else {
        uint32_t v0[32], v1[32];
        tmem_ld32(acc + c * 64, v0);
        tmem_ld32(acc + c * 64 + 32, v1);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          xs[k] = __fadd2_rn(make_float2(__uint_as_float(v0[2 * k]), __uint_as_float(v0[2 * k + 1])), f2(add));
          xs[16 + k] = __fadd2_rn(make_float2(__uint_as_float(v1[2 * k]), __uint_as_float(v1[2 * k + 1])), f2(add));
        }
      }
      if (res) {
#pragma unroll
        for (int c16 = 0; c16 < 8; ++c16) {
          const uint4 u = ld_shared_v4(stg + c * L::kStgHalf + lane * 128 + ((c16 ^ (lane & 7)) << 4));
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            xs[c16 * 4 + j] = __fadd2_rn(xs[c16 * 4 + j],
                                         make_float2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xffff0000u)));
        }
      }
    };
    auto stage_chunk_f = [&](uint32_t stg, int c, const float2 (&xs)[32]) {
#pragma unroll
      for (int c16 = 0; c16 < 8; ++c16)
        st_shared_v4(stg + c * L::kStgHalf + lane * 128 + ((c16 ^ (lane & 7)) << 4),
                     pack_bf16x2(xs[c16 * 4].x, xs[c16 * 4].y), pack_bf16x2(xs[c16 * 4 + 1].x, xs[c16 * 4 + 1].y),
                     pack_bf16x2(xs[c16 * 4 + 2].x, xs[c16 * 4 + 2].y),
                     pack_bf16x2(xs[c16 * 4 + 3].x, xs[c16 * 4 + 3].y));
    };
    // The group's epilogue over the row.  With a norm: a statistics pass over the chunks that also
    // writes acc (+ Z) (+ bias) (+ residual) back into the accumulator's TMEM columns, then an output
    // pass that reads only those columns.  Without a norm: one pass.  No whole row is ever held in
    // registers.  `act_ct` >= 0: activation fixed at compile time and gamma/beta from shared memory
    // (the candidate group); < 0: e.act read at run time, gamma/beta from global memory.
    auto epilogue_row = [&](auto act_ct, uint32_t acc, bool use_z, float add, bool res, uint32_t stg,
                            const EpiGroup& e) {
      constexpr int ACT = decltype(act_ct)::value;
      if (e.norm != EPI_NORM_NONE) {
        RowStats st{0.0f, 0.0f, 0.0f};
#pragma unroll 1
        for (int c = 0; c < D / 64; ++c) {
          float2 xs[32];
          load_chunk(xs, acc, use_z, add, res, stg, c);
          stats_add_chunk(st, xs, e.norm);
          uint32_t u0[32], u1[32];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            u0[2 * k] = __float_as_uint(xs[k].x);
            u0[2 * k + 1] = __float_as_uint(xs[k].y);
            u1[2 * k] = __float_as_uint(xs[16 + k].x);
            u1[2 * k + 1] = __float_as_uint(xs[16 + k].y);
          }
          tmem_st32(acc + c * 64, u0);
          tmem_st32(acc + c * 64 + 32, u1);
        }
        tmem_st_wait();
        float mean, inv;
        stats_finish(st, D, e, mean, inv);
#pragma unroll 1
        for (int c = 0; c < D / 64; ++c) {
          uint32_t v0[32], v1[32];
          tmem_ld32(acc + c * 64, v0);
          tmem_ld32(acc + c * 64 + 32, v1);
          tmem_ld_wait();
          float2 xs[32];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            xs[k] = make_float2(__uint_as_float(v0[2 * k]), __uint_as_float(v0[2 * k + 1]));
            xs[16 + k] = make_float2(__uint_as_float(v1[2 * k]), __uint_as_float(v1[2 * k + 1]));
          }
          if constexpr (ACT >= 0) {
            norm_chunk_smem(xs, s_gb + c * 64, s_gb + D + c * 64, mean, inv);
            act_chunk<ACT>(xs);
          } else {
            norm_chunk(xs, c * 64, mean, inv, e);
            act_chunk_rt(e.act, xs);
          }
          stage_chunk_f(stg, c, xs);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < D / 64; ++c) {
          float2 xs[32];
          load_chunk(xs, acc, use_z, add, res, stg, c);
          if constexpr (ACT >= 0) act_chunk<ACT>(xs);
          else act_chunk_rt(e.act, xs);
          stage_chunk_f(stg, c, xs);
        }
      }
    };

    auto acquire_stage = [&]() {  // staging buffer sb is free once the store that last used it has read it
      if (lane == 0) bulk_wait_read<L::kStgPerWarp - 1>();
      __syncwarp();
      return (uint32_t)((ew * L::kStgPerWarp + sb) * L::kStgBuf);
    };
    auto next_stage = [&]() { sb = (sb + 1) % L::kStgPerWarp; };

    for (;;) {  // request tiles: every epilogue warp reads every item (each item occupies one buffer)
      if (!mbar_wait(&wq_full[qs], qph, ctl, 301)) { ok = false; break; }
      const int item = s_wq[qs];
      __syncwarp();
      if (lane == 0) mbar_arrive(&wq_empty[qs]);
      if (++qs == 2) { qs = 0; qph ^= 1; }
      if (item < 0) break;
      if (!mine()) { ab ^= 1; continue; }
      if (!mbar_wait(&acc_full[ab], (aphs >> ab) & 1, ctl, 302)) { ok = false; break; }
      tc_fence_after();
      const uint32_t acc = tmem_base + t_lane + ab * D;
      if (item < R) {
        // Z tile: fp32 into the workspace in a [R][d/4][o_c][4] layout so that a warp's 32 rows
        // of one 4-column group are 512 contiguous bytes (coalesced store here and load later).
        const int r = item;
        float* zr = p.zws + (size_t)r * OC * D;
        // block epilogue: the candidate group's bias is folded into Z once per request
        const float bz = (EPI && p.epi_c.bias) ? __ldg(p.epi_c.bias + row) : 0.0f;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32(acc + cc * 32, v);
          tmem_ld_wait();
          if constexpr (EPI) {
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) + bz);
          }
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
          // the four warps of this group x 1 = this request's Z is complete
          if (r != p.skip_release) red_release_gpu_add(&p.flags[r], 1);
        }
      } else if constexpr (!EPI) {
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
        store_tile(&p.tm_yr, stg_off, r * p.o_r + mt * OC + 32 * quarter);
        next_stage();
      } else {  // Y^R tile with the request group's epilogue
        const int u = item - R, r = u / mt_r, mt = u % mt_r;
        const int y0 = r * p.o_r + mt * OC + 32 * quarter;
        const uint32_t stg_off = acquire_stage();
        const uint32_t stg = smem_u32(s_stg + stg_off);
        const bool res = p.epi_r.has_residual != 0;
        if (res) {
          load_residual(&p.tm_res_r, stg_off, y0);
          if (!mbar_wait(&res_bar[ew], rph, ctl, 303)) { drain_residual(); ok = false; break; }
          rph ^= 1;
        }
        const float br = p.epi_r.bias ? __ldg(p.epi_r.bias + mt * OC + row) : 0.0f;
        epilogue_row(std::integral_constant<int, -1>{}, acc, false, br, res, stg, p.epi_r);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
        store_tile(&p.tm_yr, stg_off, y0);
        next_stage();
      }
      aphs ^= 1u << ab;
      ab ^= 1;
    }

    if (ok && cbeg < cend) {  // candidate tiles
      // request of the first candidate: last r with cand_off[r] <= cbeg
      int lo = 0, hi = R - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.cand_off[mid] <= cbeg) lo = mid; else hi = mid - 1;
      }
      int r = lo, next_off = p.cand_off[r + 1], r_staged = -1, res_next = -1;
      for (int i = cbeg; i < cend; ++i) {
        while (i >= next_off) {
          if (++r >= R) break;
          next_off = p.cand_off[r + 1];
        }
        if (r >= R || r < 0) { ctl.fail(ROCS_ERR_DEVICE_INDEX, 310); ok = false; break; }
        if (!mine()) { ab ^= 1; continue; }
        if (r != r_staged) {  // stage Z_r (this warp's 32 rows) into this group's TMEM slot once per request
          if (!wait_flag_geq(&p.flags[r], kWarpsPerGroup, ctl, 311)) { ok = false; break; }
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
        if constexpr (!EPI) {
          if (!mbar_wait(&acc_full[ab], (aphs >> ab) & 1, ctl, 312)) { ok = false; break; }
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
          store_tile(&p.tm_yc, stg_off, i * OC + 32 * quarter);
        } else {  // candidate group's epilogue (a residual either in the accumulator already, see kResMma,
                  // or loaded one tile ahead into the warp's other staging buffer)
          const uint32_t stg_off = acquire_stage();
          const uint32_t stg = smem_u32(s_stg + stg_off);
          const bool res = !L::kResMma && p.epi_c.has_residual != 0;
          if (res) {
            if (res_next != i) load_residual(&p.tm_res_c, stg_off, i * OC + 32 * quarter);
            // this group's tile after next: start its residual rows towards L2 now
            if (lane == 0 && i + 2 * NG < cend) {  // evict-last: it must survive until its load two tiles on
              const uint64_t pol = l2_evict_last();
              for (int h = 0; h < D / 64; ++h)
                tma_prefetch_l2_2d_hint(&p.tm_res_c, h * 64, (i + 2 * NG) * OC + 32 * quarter, pol);
            }
          }
          if (!mbar_wait(&acc_full[ab], (aphs >> ab) & 1, ctl, 312)) {
            if (res) drain_residual();
            ok = false;
            break;
          }
          if (res) {
            if (!mbar_wait(&res_bar[ew], rph, ctl, 313)) { drain_residual(); ok = false; break; }
            rph ^= 1;
          }
          tc_fence_after();
          if (p.epi_c.norm != EPI_NORM_NONE) {
            // the whole row in registers: acc and Z read from TMEM once, the accumulator handed back to the
            // MMA before any arithmetic, then exact row statistics, norm, activation and the bf16 store
            float2 xr[D / 2];
            const uint32_t acc = tmem_base + t_lane + ab * D;
#pragma unroll
            for (int q = 0; q < D / 16; ++q) {
              uint32_t v[16], z[16];
              tmem_ld16(acc + q * 16, v);
              tmem_ld16(z_tmem + q * 16, z);
              tmem_ld_wait();
#pragma unroll
              for (int k = 0; k < 8; ++k)
                xr[q * 8 + k] = __fadd2_rn(make_float2(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1])),
                                           make_float2(__uint_as_float(z[2 * k]), __uint_as_float(z[2 * k + 1])));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
            if (res) {
#pragma unroll
              for (int c = 0; c < D / 64; ++c)
#pragma unroll
                for (int c16 = 0; c16 < 8; ++c16) {
                  const uint4 u = ld_shared_v4(stg + c * L::kStgHalf + lane * 128 + ((c16 ^ (lane & 7)) << 4));
                  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                  for (int j = 0; j < 4; ++j)
                    xr[c * 32 + c16 * 4 + j] = __fadd2_rn(
                        xr[c * 32 + c16 * 4 + j],
                        make_float2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xffff0000u)));
                }
            }
            RowStats st{0.0f, 0.0f, 0.0f};
            stats_add_chunk(st, xr, p.epi_c.norm);
            float mean, inv;
            stats_finish(st, D, p.epi_c, mean, inv);
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
              float2(&xs)[32] = *reinterpret_cast<float2(*)[32]>(&xr[c * 32]);
              norm_chunk_smem(xs, s_gb + c * 64, s_gb + D + c * 64, mean, inv);
              act_chunk<EPI_C>(xs);
              stage_chunk_f(stg, c, xs);
            }
          } else {
            epilogue_row(std::integral_constant<int, EPI_C>{}, tmem_base + t_lane + ab * D, true, 0.0f, res, stg,
                         p.epi_c);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
          }
          store_tile(&p.tm_yc, stg_off, i * OC + 32 * quarter, true);
          // this group's next tile: its residual rows into the other staging buffer (whose last store,
          // two groups back, must have finished reading it)
          if (res && i + NG < cend) {
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
            load_residual(&p.tm_res_c, (uint32_t)((ew * L::kStgPerWarp + (sb ^ 1)) * L::kStgBuf), (i + NG) * OC + 32 * quarter);
            res_next = i + NG;
          }
        }
        next_stage();
        aphs ^= 1u << ab;
        ab ^= 1;
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
template <int D, int NC, int EPI_C>
static cudaError_t launch_t(const LcbParams& p, int grid, cudaStream_t st) {
  constexpr int NG = EPI_C >= 0 ? 2 : 1;
  using L = LcbSmem<D, NC, NG>;
  auto k = rocs_lcb_sm100_kernel<D, NC, EPI_C, NG>;
  static std::atomic<uint64_t> optin_done{0};  // per instantiation, one bit per device
  if constexpr (NG == 2) {
    static std::atomic<int> regs_checked{0};  // a property of the binary: checked once per process
    if (!regs_checked.load(std::memory_order_acquire)) {
      // the setmaxnreg split is only valid for the register count it was computed for
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, k) != cudaSuccess || fa.numRegs != (int)LcbRoles<NG>::kLaunchRegs)
        return cudaErrorInvalidConfiguration;
      regs_checked.store(1, std::memory_order_release);
    }
  }
  cudaError_t e = ensure_smem_optin(optin_done, k, (int)L::alloc_bytes);
  if (e != cudaSuccess) return e;
  return launch_dependent(k, grid, LcbRoles<NG>::kThreads, L::alloc_bytes, st, p);
}

__global__ void rocs_zero_ints_kernel(int* a, int na, int* b, int nb) {
  asm volatile("griddepcontrol.launch_dependents;");
  const int t = blockIdx.x * blockDim.x + threadIdx.x, n = gridDim.x * blockDim.x;
  for (int i = t; i < na; i += n) a[i] = 0;
  for (int i = t; i < nb; i += n) b[i] = 0;
}

cudaError_t launch_zero_ints(int* a, int na, int* b, int nb, cudaStream_t st) {
  const int n = na > nb ? na : nb;
  int grid = (n + 255) / 256;
  if (grid > 64) grid = 64;
  if (grid < 1) grid = 1;
  rocs_zero_ints_kernel<<<grid, 256, 0, st>>>(a, na, b, nb);
  return cudaGetLastError();
}

template <int EPI_C>
static cudaError_t launch_e(const LcbParams& p, int d, int n_c, int grid, cudaStream_t st) {
  if (d == 128 && n_c == 64) return launch_t<128, 64, EPI_C>(p, grid, st);
  if (d == 128 && n_c == 128) return launch_t<128, 128, EPI_C>(p, grid, st);
  if (d == 64 && n_c == 64) return launch_t<64, 64, EPI_C>(p, grid, st);
  if (d == 64 && n_c == 128) return launch_t<64, 128, EPI_C>(p, grid, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_lcb_sm100(const LcbParams& p, int d, int n_c, bool epilogue, int grid, cudaStream_t st) {
  if (!epilogue) return launch_e<-1>(p, d, n_c, grid, st);
  switch (p.epi_c.act) {
    case EPI_ACT_NONE: return launch_e<EPI_ACT_NONE>(p, d, n_c, grid, st);
    case EPI_ACT_RELU: return launch_e<EPI_ACT_RELU>(p, d, n_c, grid, st);
    case EPI_ACT_SILU: return launch_e<EPI_ACT_SILU>(p, d, n_c, grid, st);
    case EPI_ACT_GELU: return launch_e<EPI_ACT_GELU>(p, d, n_c, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace rocs
