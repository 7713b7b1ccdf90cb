// proj_sm100.cu -- dense bf16 projection GEMM for the chained block:
//     out[M, N] = in[M, K] . W[N, K]^T        (fp32 accumulate in TMEM, bf16 out)
// used for the query generation of the chained block ("ROCS ...", arXiv:2607.27744,
// section 3.2, Eq. (12): queries are produced from the LCB output; read here as a plain
// linear map Q_i = W_q . vec(Y^C_i)).
//
// Persistent CTAs take output tiles of 128 x 256 in (m, n) order with n innermost so the
// CTAs that run together share one 128-row block of `in` through L2.  Warp 0 issues TMA
// loads (K-blocks of 64, 4-stage ring), warp 1 issues tcgen05.mma (M=128, N=256, K=16),
// warps 2-5 drain the double-buffered TMEM accumulator and store bf16 (or fp32) rows, optionally
// adding a per-request row of an fp32 matrix first (the IKBO broadcast-add of the split chain:
// row i gets add[m_i, :], m_i from CSR offsets).
#include "lcb_sm100.h"

namespace rocs {

namespace {
constexpr int kThreads = 192;
constexpr int kProducer = 0, kMma = 1;
constexpr int BM = 128, BN = 256, BK = 64, kStages = 4;
constexpr uint32_t kA = BM * BK * 2, kB = BN * BK * 2, kStage = kA + kB;
constexpr uint32_t off_bar = kStages * kStage;
constexpr uint32_t n_bars = 2 * kStages + 4 + 1;
constexpr uint32_t off_misc = off_bar + n_bars * 8;
constexpr uint32_t alloc_bytes = off_misc + 64 + 1024;
static_assert(alloc_bytes <= 232448, "shared memory budget");
}  // namespace

__global__ void __launch_bounds__(kThreads, 1) rocs_proj_sm100_kernel(const __grid_constant__ ProjParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + off_bar);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain_bar = acc_empty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + off_misc);
  int* s_abort = reinterpret_cast<int*>(smem + off_misc + 16);

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  const Ctl ctl{s_abort, p.ws, (unsigned long long)p.wait_limit_ns};
  const int mt = (p.M + BM - 1) / BM, nt = p.N / BN, tiles = mt * nt, kb_n = p.K / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&acc_full[k], 1);
      mbar_init(&acc_empty[k], 4);
    }
    mbar_init(drain_bar, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == kMma) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  if (warp == kProducer) {
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_a);
      tma_prefetch_desc(&p.tm_b);
      uint32_t s = 0, ph = 0;
      int n_issued = 0;
      bool ok = true;
      // `in` streams past once (its 128-row block is shared only by the CTAs running the same m at the same
      // time); the weight is read again by every wave of tiles, so it is kept in L2 ahead of `in`
      const uint64_t pol_a = l2_evict_first(), pol_b = l2_evict_last();
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        const int m0 = (t / nt) * BM, n0 = (t % nt) * BN;
        for (int kb = 0; kb < kb_n; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1, ctl, 901)) { ok = false; break; }
          uint8_t* st = smem + s * kStage;
          mbar_arrive_expect_tx(&full[s], kStage);
          tma_load_2d_hint(st, &p.tm_a, &full[s], kb * BK, m0, pol_a);
          tma_load_2d_hint(st + kA, &p.tm_b, &full[s], kb * BK, n0, pol_b);
          ++n_issued;
          if (++s == kStages) { s = 0; ph ^= 1; }
        }
      }
      if (!ok)
        for (int k = n_issued > kStages ? n_issued - kStages : 0; k < n_issued; ++k)
          mbar_drain(&full[k % kStages], (k / kStages) & 1, 20000000ull);
    }
  } else if (warp == kMma) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(BM, BN, false, false);
      uint32_t s = 0, ph = 0, ab = 0, aph = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        if (!mbar_wait(&acc_empty[ab], aph ^ 1, ctl, 902)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + ab * BN;
        for (int kb = 0; kb < kb_n; ++kb) {
          if (!mbar_wait(&full[s], ph, ctl, 903)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * kStage);
          const uint64_t ad = sdesc_sw128(a0, 16, 1024), bd = sdesc_sw128(a0 + kA, 16, 1024);
#pragma unroll
          for (int kin = 0; kin < BK / 16; ++kin)
            umma_ss(d, sdesc_add(ad, kin * 32), sdesc_add(bd, kin * 32), idesc, (kb | kin) != 0);
          umma_commit(&empty[s]);
          if (++s == kStages) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        umma_commit(&acc_full[ab]);
        if (++ab == 2) { ab = 0; aph ^= 1; }
      }
      umma_commit(drain_bar);
      mbar_drain(drain_bar, 0, 50000000ull);
    }
  } else {
    const int quarter = warp & 3;
    const uint32_t t_lane = (uint32_t)(32 * quarter) << 16;
    uint32_t ab = 0, aph = 0;
    int m_row = -1, m_row_for = -1;  // request of this thread's row (IKBO broadcast-add)
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      const int m0 = (t / nt) * BM, n0 = (t % nt) * BN;
      if (!mbar_wait(&acc_full[ab], aph, ctl, 904)) break;
      tc_fence_after();
      const int row = m0 + 32 * quarter + (int)lane;
      if (p.add && row < p.M && row != m_row_for) {  // last r with add_off[r] <= row
        int lo = 0, hi = p.add_R - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (__ldg(p.add_off + mid) <= row) lo = mid; else hi = mid - 1;
        }
        m_row = lo;
        m_row_for = row;
      }
      const float* arow = p.add ? p.add + (size_t)m_row * p.N + n0 : nullptr;
#pragma unroll 1
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(tmem_base + t_lane + ab * BN + cc * 32, v);
        tmem_ld_wait();
        if (row < p.M) {
          if (arow) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float4 a4 = __ldg(reinterpret_cast<const float4*>(arow + cc * 32) + k);
              v[4 * k + 0] = __float_as_uint(__uint_as_float(v[4 * k + 0]) + a4.x);
              v[4 * k + 1] = __float_as_uint(__uint_as_float(v[4 * k + 1]) + a4.y);
              v[4 * k + 2] = __float_as_uint(__uint_as_float(v[4 * k + 2]) + a4.z);
              v[4 * k + 3] = __float_as_uint(__uint_as_float(v[4 * k + 3]) + a4.w);
            }
          }
          if (p.out_f32) {
            float* frow = p.out_f32 + (size_t)row * p.N + n0 + cc * 32;
#pragma unroll
            for (int k = 0; k < 8; ++k) st_global_v4(frow + 4 * k, v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
          } else {
            __nv_bfloat16* orow = p.out + (size_t)row * p.N + n0;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              st_global_v4(orow + cc * 32 + 8 * k,
                           pack_bf16x2(__uint_as_float(v[8 * k + 0]), __uint_as_float(v[8 * k + 1])),
                           pack_bf16x2(__uint_as_float(v[8 * k + 2]), __uint_as_float(v[8 * k + 3])),
                           pack_bf16x2(__uint_as_float(v[8 * k + 4]), __uint_as_float(v[8 * k + 5])),
                           pack_bf16x2(__uint_as_float(v[8 * k + 6]), __uint_as_float(v[8 * k + 7])));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
      if (++ab == 2) { ab = 0; aph ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMma) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// one CTA per (k, n), one thread per c: sum over o of W_q[k, o*d + c] W_CC[o, n]
__global__ void rocs_chain_fold_kernel(const __nv_bfloat16* __restrict__ w_q, const __nv_bfloat16* __restrict__ w_cc,
                                       __nv_bfloat16* __restrict__ w_fold, int o_c, int n_c, int d) {
  const int kn = blockIdx.x, k = kn / n_c, n = kn - k * n_c;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float acc = 0.0f;
    for (int o = 0; o < o_c; ++o)
      acc = fmaf(__bfloat162float(w_q[((size_t)k * o_c + o) * d + c]), __bfloat162float(w_cc[(size_t)o * n_c + n]), acc);
    w_fold[((size_t)k * n_c + n) * d + c] = __float2bfloat16_rn(acc);
  }
}

cudaError_t launch_chain_fold(const __nv_bfloat16* w_q, const __nv_bfloat16* w_cc, __nv_bfloat16* w_fold, int n_out,
                              int o_c, int n_c, int d, cudaStream_t st) {
  const int threads = d < 1024 ? ((d + 31) / 32) * 32 : 1024;
  rocs_chain_fold_kernel<<<n_out * n_c, threads, 0, st>>>(w_q, w_cc, w_fold, o_c, n_c, d);
  return cudaGetLastError();
}

cudaError_t launch_proj_sm100(const ProjParams& p, int grid, cudaStream_t st) {
  static std::atomic<uint64_t> optin_done{0};  // one bit per device
  cudaError_t e = ensure_smem_optin(optin_done, rocs_proj_sm100_kernel, (int)alloc_bytes);
  if (e != cudaSuccess) return e;
  rocs_proj_sm100_kernel<<<grid, kThreads, alloc_bytes, st>>>(p);
  return cudaGetLastError();
}

}  // namespace rocs
