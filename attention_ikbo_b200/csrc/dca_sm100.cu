// dca_sm100.cu -- IKBO-DCA on B200: persistent flash-style cross attention over K/V that is
// stored once per request.
//
// Computes the candidate-group cross attention of "ROCS: Request-Oriented Compute Sharing ..."
// (arXiv:2607.27744; paper-archivist notes, section 3.2, Eq. (13)),
//     O_i = softmax(scale . Q_i K_{m_i}^T) V_{m_i}        (non-causal),
// resolving m_i inside the kernel (section 4.3.1): K/V stay at batch size B_r and every
// candidate of a request reads the same physical K/V tiles.
//
// sm_100a design (the pages' design targeted Hopper warp-group MMA; what carries over is
// "stack many short candidate queries of one request into a full query tile" and
// "persistent, warp-specialised, pipelined across tiles"):
//   * work unit = (request r, head h, 256 consecutive query rows of r).  The query rows of
//     ALL candidates of r are one M dimension (q tokens per candidate, candidates
//     contiguous), so two 128-row tcgen05 tiles (A and B) are filled with many candidates
//     and share every K/V tile loaded into shared memory (section 4.3.2's "several
//     candidates per CTA", generalised).  Tiles never cross requests.
//   * warp roles: warp 0 TMA producer (Q tiles, then K/V tiles in consumption order through
//     one ring), warp 1 single-thread tcgen05.mma issuer, warps 4-7 softmax/epilogue of
//     tile A, warps 8-11 of tile B.  S = Q K^T lands in TMEM (fp32), the softmax warps write
//     P (bf16) back over S in TMEM, and P V is issued with P as the TMEM A operand, O
//     accumulating in TMEM.  The issuer alternates [PV_A, S_A] and [PV_B, S_B] so the
//     tensor core works on one tile while the softmax warps of the other tile run.  With
//     dh = 64 the O accumulators leave 128 TMEM columns free, so P gets columns of its own:
//     the next S of a tile is issued as soon as the softmax has read the current one, and P
//     is rewritten only after the previous P V has completed.
//   * online softmax in the exp2 domain with lazy rescaling: O and the running sum are
//     rescaled only when a row's maximum grows by more than 2^8; row maxima with 3-input max
//     chains, exponent arguments and row sums with packed fp32x2 FMA/ADD, exp2 on the MUFU.
//   * three warpgroups (producer/issuer, tile A softmax, tile B softmax); setmaxnreg moves
//     registers from the first to the other two so all 128 scores of a row stay in registers.
//   * work units are claimed from a global ticket in a table ordered longest request first
//     (load balance), units of one (request, head) adjacent (K/V L2 locality; section 4.3.1's
//     grid reordering, expressed as the claim order of a persistent kernel).
#include "lcb_sm100.h"

namespace rocs {

namespace {

constexpr int kThreads = 384;
constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kSoftmaxWarp0 = 4;  // warpgroup 1 (warps 4..7) tile A, warpgroup 2 (8..11) tile B
// Register split (setmaxnreg): launched at kLaunchRegs per thread (checked on the host before
// the first launch), warpgroup 0 gives registers back, the two softmax warpgroups take them:
//   4 warps x 32 x kRegsCtl + 8 warps x 32 x kRegsSoftmax == 384 x kLaunchRegs,
// and per SM sub-partition (warps w, w+4, w+8) kRegsCtl + 2 kRegsSoftmax == 3 kLaunchRegs.
constexpr uint32_t kLaunchRegs = 168, kRegsCtl = 120, kRegsSoftmax = 192;
static_assert(4 * 32 * kRegsCtl + 8 * 32 * kRegsSoftmax == kThreads * kLaunchRegs, "register split");
constexpr int BM = 128, BN = 128;
constexpr int kRowsPerUnit = 2 * BM;

template <int DH>
struct DcaSmem {
  static constexpr uint32_t kTile = BM * DH * 2;  // one Q tile or one K/V tile of one head (bf16)
  // K/V ring slot: one head's tile (dh = 128), or room for two heads' tiles (dh = 64: a head pair's)
  static constexpr int kHeadsPerSlot = DH == 128 ? 1 : 2;  // head pairs are formed at dh = 64 only
  static constexpr uint32_t kSlot = kHeadsPerSlot * kTile;
  static constexpr int kRing = DH == 128 ? 4 : 5;
  static constexpr uint32_t kStage = 32 * 128;     // per softmax warp: 32 rows x 64 columns of O (bf16)
  static constexpr uint32_t off_q = 0;
  static constexpr uint32_t off_ring = 2 * kTile;
  static constexpr uint32_t off_stage = off_ring + kRing * kSlot;  // 8 warps x kStage, 1024-byte aligned
  static constexpr uint32_t off_bar = off_stage + 8 * kStage;
  static constexpr uint32_t n_bars = 2 * kRing + 2 * 8 + 1 + 4;
  static constexpr uint32_t off_misc = off_bar + n_bars * 8;
  static constexpr uint32_t bytes = off_misc + 64;
  static constexpr uint32_t alloc_bytes = bytes + 1024;
  static_assert(alloc_bytes <= 232448, "shared memory budget");
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// tcgen05.wait::ld that also names 64 registers of the second half of S as in/out operands, so the compiler
// keeps every use of them after the wait
__device__ __forceinline__ void tmem_ld_wait_regs(uint32_t (&a)[32], uint32_t (&b)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]), "+r"(a[6]), "+r"(a[7]),
                 "+r"(a[8]), "+r"(a[9]), "+r"(a[10]), "+r"(a[11]), "+r"(a[12]), "+r"(a[13]), "+r"(a[14]), "+r"(a[15]),
                 "+r"(a[16]), "+r"(a[17]), "+r"(a[18]), "+r"(a[19]), "+r"(a[20]), "+r"(a[21]), "+r"(a[22]), "+r"(a[23]),
                 "+r"(a[24]), "+r"(a[25]), "+r"(a[26]), "+r"(a[27]), "+r"(a[28]), "+r"(a[29]), "+r"(a[30]), "+r"(a[31]),
                 "+r"(b[0]), "+r"(b[1]), "+r"(b[2]), "+r"(b[3]), "+r"(b[4]), "+r"(b[5]), "+r"(b[6]), "+r"(b[7]),
                 "+r"(b[8]), "+r"(b[9]), "+r"(b[10]), "+r"(b[11]), "+r"(b[12]), "+r"(b[13]), "+r"(b[14]), "+r"(b[15]),
                 "+r"(b[16]), "+r"(b[17]), "+r"(b[18]), "+r"(b[19]), "+r"(b[20]), "+r"(b[21]), "+r"(b[22]), "+r"(b[23]),
                 "+r"(b[24]), "+r"(b[25]), "+r"(b[26]), "+r"(b[27]), "+r"(b[28]), "+r"(b[29]), "+r"(b[30]), "+r"(b[31])
               :
               : "memory");
}

struct Unit {
  int r, h, row0;  // request, head, first query row (within the request's rows)
  int rows;        // query rows of the request (q * N_r)
  int qbase;       // global query row of the request's first row (q * cand_off[r])
  int s0, L;       // first key row, number of keys
  int nkv;         // K/V tiles
  bool hasB;       // second 128-row tile has at least one valid row
  int half;        // 0: whole unit; 1, 2: first / second half of a unit split along the keys
  int slot;        // split units: index of the pair's merge area
  int nh;          // heads whose K/V the unit reads: 2 for a head pair (tile B = the next head, same rows)
  int hB, rowB0;   // head and first row (within the request's rows) of tile B
};

__device__ __forceinline__ Unit load_unit(const DcaParams& p, int u) {
  const int4 e = p.units[u];
  Unit w;
  w.r = e.x;
  w.h = e.y;
  w.row0 = e.z;
  const int c0 = p.cand_off[w.r], c1 = p.cand_off[w.r + 1];
  w.rows = p.q * (c1 - c0);
  w.qbase = p.q * c0;
  w.s0 = p.seq_off[w.r];
  w.L = p.seq_off[w.r + 1] - w.s0;
  w.nkv = (w.L + BN - 1) / BN;
  const bool paired = (e.w >> 2) & 1;
  w.nh = paired ? 2 : 1;
  w.hB = paired ? w.h + 1 : w.h;
  w.rowB0 = paired ? w.row0 : w.row0 + BM;
  w.hasB = paired || w.row0 + BM < w.rows;
  w.half = e.w & 3;
  w.slot = e.w >> 3;
  if (w.half) {  // a half of the keys: the first nkv/2 tiles, or the rest (the key range is rebased)
    const int n0 = w.nkv / 2;
    if (w.half == 1) {
      w.L = n0 * BN;
      w.nkv = n0;
    } else {
      w.s0 += n0 * BN;
      w.L -= n0 * BN;
      w.nkv -= n0;
    }
  }
  return w;
}

}  // namespace

template <int DH>
__global__ void __launch_bounds__(kThreads, 1) rocs_dca_sm100_kernel(const __grid_constant__ DcaParams p) {
  using L = DcaSmem<DH>;
  constexpr int kRing = L::kRing;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_q = smem + L::off_q;
  uint8_t* s_ring = smem + L::off_ring;
  uint8_t* s_stage = smem + L::off_stage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::off_bar);
  uint64_t* ring_full = bars;
  uint64_t* ring_empty = bars + kRing;
  uint64_t* q_full = bars + 2 * kRing;  // [2]
  uint64_t* q_empty = q_full + 2;
  uint64_t* s_full = q_empty + 2;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* o_empty = o_full + 2;
  uint64_t* wq_full = o_empty + 2;  // two-slot work queue: the producer runs one unit ahead
  uint64_t* wq_empty = wq_full + 2;
  uint64_t* drain_bar = wq_empty + 2;
  uint64_t* s_free = drain_bar + 1;  // [2] separate-P layout: S of tile x read into registers
  uint64_t* pv_done = s_free + 2;    // [2] separate-P layout: P V of tile x complete (P may be rewritten)
  int* s_wq = reinterpret_cast<int*>(smem + L::off_misc);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::off_misc + 16);
  int* s_abort = reinterpret_cast<int*>(smem + L::off_misc + 32);

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  const Ctl ctl{s_abort, p.ws, (unsigned long long)p.wait_limit_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&ring_full[s], 1);
      mbar_init(&ring_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&q_full[x], 1);
      mbar_init(&q_empty[x], 1);
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], 4);
      mbar_init(&o_full[x], 1);
      mbar_init(&o_empty[x], 4);
      mbar_init(&s_free[x], 4);
      mbar_init(&pv_done[x], 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&wq_full[k], 1);
      mbar_init(&wq_empty[k], 1 + 8);
    }
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
  // TMEM columns: S_A [0,128) S_B [128,256) O_A [256,256+DH) O_B [256+DH,256+2DH).  dh = 128: P_X over
  // S_X [0,64), so S of the next K/V tile waits for P V.  dh = 64 leaves 128 columns free: P_A [384,448),
  // P_B [448,512) of their own, so S of the next tile is computed while the softmax works on this one.
  constexpr bool kSepP = 256 + 2 * DH + 128 <= 512;
  constexpr uint32_t kPCol = 256 + 2 * DH;

  if (warp < kSoftmaxWarp0) {
   // warpgroup 0: hand registers to the softmax warpgroups, then producer / issuer / idle
   reg_dealloc<kRegsCtl>();
   if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      uint32_t rs = 0, rph = 0, ws_ = 0, wph = 0, qeph[2] = {0, 0};
      int n_issued = 0;
      bool ok = true;
      // one K/V tile (128 keys) of heads h0 .. h0+nh-1 into the next ring slot, head hh at offset hh * kTile
      auto load_kv = [&](const CUtensorMap* tm, int y, int h0, int nh) -> bool {
        if (!mbar_wait(&ring_empty[rs], rph ^ 1, ctl, 501)) return false;
        uint8_t* slot = s_ring + rs * L::kSlot;
        mbar_arrive_expect_tx(&ring_full[rs], nh * L::kTile);
        for (int hh = 0; hh < nh; ++hh)
#pragma unroll
          for (int cc = 0; cc < DH / 64; ++cc)
            tma_load_2d(slot + hh * L::kTile + cc * (BM * 128), tm, &ring_full[rs], (h0 + hh) * DH + cc * 64, y);
        ++n_issued;
        if (++rs == kRing) { rs = 0; rph ^= 1; }
        return true;
      };
      // launched as a programmatic dependent of the scheduling kernel: the prologue above overlapped it;
      // the unit table and the zeroed ticket are visible after this wait
      asm volatile("griddepcontrol.wait;" ::: "memory");
      while (ok) {
        const int t = atomicAdd(p.ticket, 1);
        const int item = t < p.n_units ? t : -1;
        if (!mbar_wait(&wq_empty[ws_], wph ^ 1, ctl, 502)) { ok = false; break; }
        s_wq[ws_] = item;
        mbar_arrive(&wq_full[ws_]);
        if (++ws_ == 2) { ws_ = 0; wph ^= 1; }
        if (item < 0) break;
        const Unit w = load_unit(p, item);
        if (w.nkv == 0) continue;
        for (int x = 0; x < (w.hasB ? 2 : 1); ++x) {
          if (!mbar_wait(&q_empty[x], qeph[x] ^ 1, ctl, 503)) { ok = false; break; }
          qeph[x] ^= 1;
          mbar_arrive_expect_tx(&q_full[x], L::kTile);
#pragma unroll
          for (int cc = 0; cc < DH / 64; ++cc)
            tma_load_2d(s_q + x * L::kTile + cc * (BM * 128), &p.tm_q, &q_full[x],
                        ((L::kHeadsPerSlot == 2 && x) ? w.hB : w.h) * DH + cc * 64,
                        w.qbase + ((L::kHeadsPerSlot == 2) ? (x ? w.rowB0 : w.row0) : w.row0 + x * BM));
        }
        if (!ok) break;
        // K/V in the order the MMA issuer consumes them: K0, (K1, V0), (K2, V1), ..., V_last; a head pair
        // loads each tile for both heads into one slot
        auto kv_step = [&](const CUtensorMap* tm, int y) -> bool {
          return load_kv(tm, y, w.h, L::kHeadsPerSlot == 2 ? w.nh : 1);
        };
        ok = kv_step(&p.tm_k, w.s0);
        for (int j = 1; ok && j < w.nkv; ++j) {
          ok = kv_step(&p.tm_k, w.s0 + j * BN);
          if (ok) ok = kv_step(&p.tm_v, w.s0 + (j - 1) * BN);
        }
        if (ok) ok = kv_step(&p.tm_v, w.s0 + (w.nkv - 1) * BN);
      }
      if (!ok) {
        for (int k = n_issued > kRing ? n_issued - kRing : 0; k < n_issued; ++k)
          mbar_drain(&ring_full[k % kRing], (k / kRing) & 1, 20000000ull);
      }
    }
   } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ tcgen05 issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(BM, BN, false, false);  // S = Q K^T : both K-major
      constexpr uint32_t idesc_o = idesc_bf16(BM, DH, false, true);   // O += P V  : V is MN-major
      uint32_t rs = 0, rph = 0, ws_ = 0, wph = 0;
      uint32_t qfph[2] = {0, 0}, pph[2] = {0, 0}, oeph[2] = {0, 0};
      bool ok = true;
      const uint32_t q0 = smem_u32(s_q);
      auto next_slot = [&](uint32_t& slot_addr, int where) -> bool {
        if (!mbar_wait(&ring_full[rs], rph, ctl, where)) return false;
        slot_addr = smem_u32(s_ring + rs * L::kSlot);
        return true;
      };
      auto release_slot = [&](uint32_t slot_addr) {  // slots are consumed in ring order
        const uint32_t idx = (slot_addr - smem_u32(s_ring)) / L::kSlot;
        umma_commit(&ring_empty[idx]);
      };
      auto advance = [&]() {
        if (++rs == kRing) { rs = 0; rph ^= 1; }
      };
      auto issue_s = [&](int x, uint32_t kslot) {
        const uint64_t ad = sdesc_sw128(q0 + x * L::kTile, 16, 1024), bd = sdesc_sw128(kslot, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk)
          umma_ss(tmem_base + x * 128, sdesc_add(ad, (kk >> 2) * (BM * 128) + (kk & 3) * 32),
                  sdesc_add(bd, (kk >> 2) * (BN * 128) + (kk & 3) * 32), idesc_s, kk != 0);
        umma_commit(&s_full[x]);
      };
      auto issue_pv = [&](int x, uint32_t vslot, bool acc) {
        const uint64_t vd = sdesc_sw128(vslot, BN * 128, 1024);
        const uint32_t pa = tmem_base + (kSepP ? kPCol + x * 64 : x * 128);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_ts(tmem_base + 256 + x * DH, pa + kk * 8, sdesc_add(vd, kk * 2048), idesc_o, (acc || kk != 0) ? 1u : 0u);
      };
      uint32_t sfph[2] = {0, 0};
      bool s_pend[2] = {false, false};
      // separate-P layout: S_x may be overwritten once the softmax has read the previous S_x
      auto issue_s_free = [&](int x, uint32_t kslot) -> bool {
        if (s_pend[x]) {
          if (!mbar_wait(&s_free[x], sfph[x], ctl, 610)) return false;
          sfph[x] ^= 1;
          tc_fence_after();
        }
        issue_s(x, kslot);
        s_pend[x] = true;
        return true;
      };
      auto wait_p = [&](int x, bool first_pv) -> bool {
        if (!mbar_wait(&p_full[x], pph[x], ctl, 601)) return false;
        pph[x] ^= 1;
        if (first_pv) {  // O_x of the previous unit must have been read out
          if (!mbar_wait(&o_empty[x], oeph[x] ^ 1, ctl, 602)) return false;
          oeph[x] ^= 1;
        }
        tc_fence_after();
        return true;
      };
      for (;;) {
        if (!mbar_wait(&wq_full[ws_], wph, ctl, 603)) { ok = false; break; }
        const int item = s_wq[ws_];
        mbar_arrive(&wq_empty[ws_]);
        if (++ws_ == 2) { ws_ = 0; wph ^= 1; }
        if (item < 0) break;
        const Unit w = load_unit(p, item);
        if (w.nkv == 0) continue;
        const int nx = w.hasB ? 2 : 1;
        for (int x = 0; x < nx && ok; ++x) {
          if (!mbar_wait(&q_full[x], qfph[x], ctl, 604)) ok = false;
          qfph[x] ^= 1;
        }
        if (!ok) break;
        tc_fence_after();
        // a head pair's two tiles read the two halves of each K/V slot (tile B at byte offset pb)
        const uint32_t pb = (L::kHeadsPerSlot == 2 && w.nh == 2) ? L::kTile : 0u;
        uint32_t kslot, vslot;
        if (!next_slot(kslot, 605)) { ok = false; break; }
        advance();
        tc_fence_after();
        if constexpr (kSepP) {
          for (int x = 0; x < nx && ok; ++x) ok = issue_s_free(x, kslot + pb * x);
          if (!ok) break;
          release_slot(kslot);
          // per K/V step: S of the next tile as soon as the softmax has read the current one, then P V
          for (int j = 1; j < w.nkv; ++j) {
            if (!next_slot(kslot, 606)) { ok = false; break; }
            advance();
            for (int x = 0; x < nx && ok; ++x) ok = issue_s_free(x, kslot + pb * x);
            if (!ok) break;
            release_slot(kslot);
            if (!next_slot(vslot, 607)) { ok = false; break; }
            advance();
            for (int x = 0; x < nx; ++x) {
              if (!wait_p(x, j == 1)) { ok = false; break; }
              issue_pv(x, vslot + pb * x, j > 1);
              umma_commit(&pv_done[x]);
            }
            if (!ok) break;
            release_slot(vslot);
          }
          if (!ok) break;
          for (int x = 0; x < nx; ++x) umma_commit(&q_empty[x]);
          if (!next_slot(vslot, 608)) { ok = false; break; }
          advance();
          for (int x = 0; x < nx; ++x) {
            if (!wait_p(x, w.nkv == 1)) { ok = false; break; }
            issue_pv(x, vslot + pb * x, w.nkv > 1);
            umma_commit(&pv_done[x]);
            umma_commit(&o_full[x]);
          }
          if (!ok) break;
          release_slot(vslot);
          continue;
        }
        issue_s(0, kslot);
        if (nx == 2) issue_s(1, kslot + pb);
        release_slot(kslot);
        for (int j = 1; j < w.nkv; ++j) {
          if (!next_slot(kslot, 606)) { ok = false; break; }
          advance();
          if (!next_slot(vslot, 607)) { ok = false; break; }
          advance();
          for (int x = 0; x < nx; ++x) {
            if (!wait_p(x, j == 1)) { ok = false; break; }
            issue_pv(x, vslot + pb * x, j > 1);
            issue_s(x, kslot + pb * x);
          }
          if (!ok) break;
          release_slot(vslot);
          release_slot(kslot);
        }
        if (!ok) break;
        for (int x = 0; x < nx; ++x) umma_commit(&q_empty[x]);
        if (!next_slot(vslot, 608)) { ok = false; break; }
        advance();
        for (int x = 0; x < nx; ++x) {
          if (!wait_p(x, w.nkv == 1)) { ok = false; break; }
          issue_pv(x, vslot + pb * x, w.nkv > 1);
          umma_commit(&o_full[x]);
        }
        if (!ok) break;
        release_slot(vslot);
      }
      umma_commit(drain_bar);
      mbar_drain(drain_bar, 0, 50000000ull);
    }
   }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    reg_alloc<kRegsSoftmax>();
    const int x = (warp - kSoftmaxWarp0) >> 2;  // 0: tile A, 1: tile B
    const int quarter = warp & 3;               // TMEM lanes 32*quarter .. +31
    const uint32_t t_lane = (uint32_t)(32 * quarter) << 16;
    const uint32_t s_addr = tmem_base + t_lane + x * 128;
    const uint32_t p_addr = kSepP ? tmem_base + t_lane + kPCol + x * 64 : s_addr;
    const uint32_t o_addr = tmem_base + t_lane + 256 + x * DH;
    uint8_t* stage = s_stage + (warp - kSoftmaxWarp0) * L::kStage;  // this warp's O staging slab
    const uint32_t stage_a = smem_u32(stage);
    const float c = p.scale_log2;
    uint32_t ws_ = 0, wph = 0, sph = 0, ofph = 0, n_sig = 0;
    bool ok = true;
    for (;;) {
      if (!mbar_wait(&wq_full[ws_], wph, ctl, 701)) { ok = false; break; }
      const int item = s_wq[ws_];
      __syncwarp();
      if (lane == 0) mbar_arrive(&wq_empty[ws_]);
      if (++ws_ == 2) { ws_ = 0; wph ^= 1; }
      if (item < 0) break;
      const Unit w = load_unit(p, item);
      if (x == 1 && !w.hasB) continue;
      const int hx = (L::kHeadsPerSlot == 2 && x) ? w.hB : w.h;          // this tile's head
      const int tile0 = (L::kHeadsPerSlot == 2) ? (x ? w.rowB0 : w.row0) : w.row0 + x * BM;  // its first row
      const int row = tile0 + 32 * quarter + (int)lane;  // row within the request
      const bool row_ok = row < w.rows;
      __nv_bfloat16* orow = p.o + ((size_t)(w.qbase + row) * p.H + hx) * DH;
      if (w.nkv == 0) {  // request without keys: O = 0, LSE = -inf
        if (row_ok) {
#pragma unroll
          for (int k = 0; k < DH / 8; ++k) st_global_v4(orow + 8 * k, 0u, 0u, 0u, 0u);
          if (p.lse) p.lse[(size_t)(w.qbase + row) * p.H + hx] = -INFINITY;
        }
        continue;
      }
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < w.nkv; ++j) {
        if (!mbar_wait(&s_full[x], sph, ctl, 702)) { ok = false; break; }
        sph ^= 1;
        tc_fence_after();
        uint32_t sv[4][32];
        // first half of S, then the second half in flight while the first half's exponentials run (steady
        // state of a full tile); the first tile of a unit and partial tiles wait for all of it
        const bool split_ld = !kSepP && j > 0 && w.L - j * BN >= BN;
        tmem_ld32(s_addr, sv[0]);
        tmem_ld32(s_addr + 32, sv[1]);
        tmem_ld_wait();
        tmem_ld32(s_addr + 64, sv[2]);
        tmem_ld32(s_addr + 96, sv[3]);
        if (!split_ld) tmem_ld_wait_regs(sv[2], sv[3]);
        if constexpr (kSepP) {
          // S is in registers: the next S may be computed; P is rewritten only once P V of the last
          // handed-over P is complete (which also makes O current for a rescale)
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_free[x]);
          if (n_sig > 0) {
            if (!mbar_wait(&pv_done[x], (n_sig - 1) & 1, ctl, 706)) { ok = false; break; }
            tc_fence_after();
          }
        }
        const int kvalid = w.L - j * BN;
        if (kvalid < BN) {
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (c4 * 32 + k >= kvalid) sv[c4][k] = __float_as_uint(-INFINITY);
        }
        // P = exp2(c S - m) written over S.  From the second tile on, the exponentials use the running
        // max m_used at once and the tile's own row max is computed alongside them (off the critical
        // path); if some row's max exceeds m_used by more than 2^8 the tile is redone with the new max
        // after rescaling O (rare: the max settles after the first tiles).  Until then P <= 2^8, which
        // bf16 and the fp32 sums hold.
        uint64_t ls0, ls1;
        float mq[8];
        auto exps_pass = [&](bool with_max) {
          uint64_t c2, nm2;
          asm("mov.b64 %0, {%1, %1};" : "=l"(c2) : "f"(c));
          asm("mov.b64 %0, {%1, %1};" : "=l"(nm2) : "f"(-m_used));
          ls0 = 0;
          ls1 = 0;
#pragma unroll
          for (int k = 0; k < 8; ++k) mq[k] = -INFINITY;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            if (c4 == 2 && split_ld && with_max) tmem_ld_wait_regs(sv[2], sv[3]);
            uint32_t pk[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              if (with_max) {
                float y;
                asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(mq[k & 7]), "f"(__uint_as_float(sv[c4][2 * k])),
                    "f"(__uint_as_float(sv[c4][2 * k + 1])));
                mq[k & 7] = y;
              }
              uint64_t sp, xp, ep;
              asm("mov.b64 %0, {%1, %2};" : "=l"(sp) : "r"(sv[c4][2 * k]), "r"(sv[c4][2 * k + 1]));
              asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(xp) : "l"(sp), "l"(c2), "l"(nm2));
              float x0, x1;
              asm("mov.b64 {%0, %1}, %2;" : "=f"(x0), "=f"(x1) : "l"(xp));
              const float p0 = ex2(x0), p1 = ex2(x1);
              asm("mov.b64 %0, {%1, %2};" : "=l"(ep) : "f"(p0), "f"(p1));
              if (k & 1) asm("add.f32x2 %0, %1, %2;" : "=l"(ls1) : "l"(ls1), "l"(ep));
              else asm("add.f32x2 %0, %1, %2;" : "=l"(ls0) : "l"(ls0), "l"(ep));
              pk[k] = pack_bf16x2(p0, p1);
            }
            tmem_st16(p_addr + c4 * 16, pk);
          }
        };
        auto row_max = [&]() {
          return fmaxf(fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])), fmaxf(fmaxf(mq[4], mq[5]), fmaxf(mq[6], mq[7])));
        };
        if (j == 0) {  // first tile: the max first
#pragma unroll
          for (int k = 0; k < 8; ++k) mq[k] = -INFINITY;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              float y;
              asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(mq[k & 7]), "f"(__uint_as_float(sv[c4][2 * k])),
                  "f"(__uint_as_float(sv[c4][2 * k + 1])));
              mq[k & 7] = y;
            }
          m_used = row_max() * c;
          exps_pass(false);
        } else {
          exps_pass(true);
          const float mxs = row_max() * c;
          if (__any_sync(0xffffffffu, mxs > m_used + 8.0f)) {  // rare: rescale O, redo the tile
            const float m_new = fmaxf(m_used, mxs);
            const float f = ex2(m_used - m_new);
            l *= f;
            tmem_st_wait();
#pragma unroll 1
            for (int cc = 0; cc < DH / 32; ++cc) {
              uint32_t ov[32];
              tmem_ld32(o_addr + cc * 32, ov);
              tmem_ld_wait();
#pragma unroll
              for (int k = 0; k < 32; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * f);
              tmem_st32(o_addr + cc * 32, ov);
            }
            m_used = m_new;
            exps_pass(false);
          }
        }
        float la, lb, lc, ld;
        asm("mov.b64 {%0, %1}, %2;" : "=f"(la), "=f"(lb) : "l"(ls0));
        asm("mov.b64 {%0, %1}, %2;" : "=f"(lc), "=f"(ld) : "l"(ls1));
        const float lsum = (la + lb) + (lc + ld);
        l += lsum;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[x]);
        ++n_sig;
      }
      if (!ok) break;
      if (!mbar_wait(&o_full[x], ofph, ctl, 703)) { ok = false; break; }
      ofph ^= 1;
      tc_fence_after();
      // A unit split along the keys: each half leaves its unnormalised O, running max and row sum in its merge
      // area, then counts itself in; the half that counts second (it may run on either CTA, or on both the
      // same) merges the two, O = (a O_own + b O_other) / (a l_own + b l_other), and writes the output.  No
      // half waits for the other.
      const float* oth = nullptr;  // the other half's O (second finisher only)
      float a_own = 1.0f, b_oth = 0.0f;
      if (w.half) {
        const size_t area = (size_t)32 * (DH + 2);
        float* mine = p.split_buf + ((((size_t)w.slot * 2 + (w.half - 1)) * 2 + x) * 4 + quarter) * area;
#pragma unroll 1
        for (int cc = 0; cc < DH / 32; ++cc) {  // [column/4][row][4]: each store a contiguous 512 bytes
          uint32_t ov[32];
          tmem_ld32(o_addr + cc * 32, ov);
          tmem_ld_wait();
#pragma unroll
          for (int k4 = 0; k4 < 8; ++k4)
            *reinterpret_cast<uint4*>(mine + ((cc * 8 + k4) * 32 + lane) * 4) =
                make_uint4(ov[4 * k4], ov[4 * k4 + 1], ov[4 * k4 + 2], ov[4 * k4 + 3]);
        }
        mine[DH * 32 + lane] = m_used;
        mine[DH * 32 + 32 + lane] = l;
        __threadfence();
        __syncwarp();
        int order = 0;
        if (lane == 0) order = atomicAdd(&p.split_cnt[w.slot * 8 + x * 4 + quarter], 1);
        order = __shfl_sync(0xffffffffu, order, 0);
        if (order == 0) {  // the other half is still running: it writes this slab
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&o_empty[x]);
          continue;
        }
        __threadfence();
        oth = p.split_buf + ((((size_t)w.slot * 2 + (2 - w.half)) * 2 + x) * 4 + quarter) * area;
        const float m_o = __ldcg(oth + DH * 32 + lane), l_o = __ldcg(oth + DH * 32 + 32 + lane);
        const float mm = fmaxf(m_used, m_o);
        a_own = ex2(m_used - mm);
        b_oth = ex2(m_o - mm);
        l = l * a_own + l_o * b_oth;
        m_used = mm;
      }
      const float inv = 1.0f / l;
      // This warp's 32 rows of the tile.  A full slab leaves through its shared-memory slab and a TMA store,
      // one 64-column box at a time: a handful of instructions per warp, where row-by-row 16-byte stores
      // (32 rows apart per instruction) would queue thousands of small writes in the SM's memory pipeline, in
      // front of the producer's and the issuer's own memory instructions.  A slab cut by the end of the
      // request's rows is stored row by row, so that no row of the next request is written.
      const int slab0 = tile0 + 32 * quarter;  // first row of the slab within the request
      const bool tma_slab = slab0 + 32 <= w.rows;
#pragma unroll 1
      for (int cc = 0; cc < DH / 64; ++cc) {
        uint32_t ov[2][32];
        tmem_ld32(o_addr + cc * 64, ov[0]);
        tmem_ld32(o_addr + cc * 64 + 32, ov[1]);
        tmem_ld_wait_regs(ov[0], ov[1]);
        if (oth) {  // second half of a split unit: a O_own + b O_other (the other's columns cc*64 .. +63)
#pragma unroll
          for (int k4 = 0; k4 < 16; ++k4) {
            const float4 o4 = __ldcg(reinterpret_cast<const float4*>(oth + ((cc * 16 + k4) * 32 + lane) * 4));
            uint32_t* v = &ov[k4 >> 3][(k4 & 7) * 4];
            v[0] = __float_as_uint(__uint_as_float(v[0]) * a_own + o4.x * b_oth);
            v[1] = __float_as_uint(__uint_as_float(v[1]) * a_own + o4.y * b_oth);
            v[2] = __float_as_uint(__uint_as_float(v[2]) * a_own + o4.z * b_oth);
            v[3] = __float_as_uint(__uint_as_float(v[3]) * a_own + o4.w * b_oth);
          }
        }
        if (tma_slab) {
          if (lane == 0) bulk_wait_read<0>();  // the slab's previous store has finished reading it
          __syncwarp();
#pragma unroll
          for (int c16 = 0; c16 < 8; ++c16) {  // row `lane`: 8 chunks of 16 bytes, 128-byte swizzle
            const uint32_t* v = &ov[c16 >> 2][(c16 & 3) * 8];
            st_shared_v4(stage_a + lane * 128 + ((c16 ^ (lane & 7)) << 4),
                         pack_bf16x2(__uint_as_float(v[0]) * inv, __uint_as_float(v[1]) * inv),
                         pack_bf16x2(__uint_as_float(v[2]) * inv, __uint_as_float(v[3]) * inv),
                         pack_bf16x2(__uint_as_float(v[4]) * inv, __uint_as_float(v[5]) * inv),
                         pack_bf16x2(__uint_as_float(v[6]) * inv, __uint_as_float(v[7]) * inv));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&p.tm_o, stage, hx * DH + cc * 64, w.qbase + slab0);
            bulk_commit();
          }
        } else if (row_ok) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t* v = &ov[k >> 2][(k & 3) * 8];
            st_global_v4(orow + cc * 64 + 8 * k, pack_bf16x2(__uint_as_float(v[0]) * inv, __uint_as_float(v[1]) * inv),
                         pack_bf16x2(__uint_as_float(v[2]) * inv, __uint_as_float(v[3]) * inv),
                         pack_bf16x2(__uint_as_float(v[4]) * inv, __uint_as_float(v[5]) * inv),
                         pack_bf16x2(__uint_as_float(v[6]) * inv, __uint_as_float(v[7]) * inv));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_empty[x]);
      if (row_ok && p.lse) p.lse[(size_t)(w.qbase + row) * p.H + hx] = (m_used + lg2(l)) * 0.69314718055994531f;
    }
    (void)ok;
    if (lane == 0) bulk_wait<0>();  // every TMA store of this warp has completed
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ------------------------------------------------------------------------------------
// Work-unit table: one block.  units_r = H * ceil(q*N_r / 256); requests ordered by key
// length descending (ties by index) so the longest units are claimed first.  The last n_split units
// in that order (the shortest) become two entries each, the halves of their K/V tiles, so that the
// final partial wave of the persistent grid is made of half-length work.
// Per-request arrays len[R], sorted[R], start[R+1] (first unit of each sorted position, then the total): in
// shared memory for R <= 2048, else in the workspace scratch.
// ------------------------------------------------------------------------------------
__global__ void rocs_dca_schedule_kernel(const DcaSchedParams p) {
  // the attention kernel may start its prologue now; it waits for this grid before claiming units
  asm volatile("griddepcontrol.launch_dependents;");
  // per-request arrays in shared memory when they fit (every phase below reads them back, the last one by
  // binary search), else in the workspace scratch
  constexpr int kSmemR = 2048;
  __shared__ int s_part[1024];
  __shared__ int s_len[kSmemR], s_sorted[kSmemR], s_start[kSmemR + 1];
  const bool in_smem = p.R <= kSmemR;
  int* len = in_smem ? s_len : p.scratch;
  int* sorted = in_smem ? s_sorted : p.scratch + p.R;
  int* start = in_smem ? s_start : p.scratch + 2 * p.R;
  const int R = p.R, T = blockDim.x, t = threadIdx.x;
  for (int r = t; r < R; r += T) len[r] = p.seq_off[r + 1] - p.seq_off[r];
  __syncthreads();
  // rank by (len desc, index asc); identity order for very many requests
  for (int r = t; r < R; r += T) {
    int rank = r;
    if (R <= 8192) {
      rank = 0;
      const int lr = len[r];
      for (int k = 0; k < R; ++k) {
        const int lk = len[k];
        rank += (lk > lr) || (lk == lr && k < r);
      }
    }
    sorted[rank] = r;
  }
  __syncthreads();
  // units of each sorted position, exclusive scan over positions.  With pair_heads, a request's last chunk of
  // at most 128 rows (one query tile) is taken for two heads at once: one unit per head pair, tile B holding
  // the next head's rows (an odd last head stays alone).
  const int per = (R + T - 1) / T;
  const int b0 = min(R, t * per), b1 = min(R, b0 + per);
  auto units_of = [&](int rows, int& nb, bool& pair_last) {
    nb = (rows + p.rows_per_unit - 1) / p.rows_per_unit;
    pair_last = p.pair_heads && p.H >= 2 && nb > 0 && rows - (nb - 1) * p.rows_per_unit <= BM;
    return pair_last ? p.H * (nb - 1) + (p.H + 1) / 2 : p.H * nb;
  };
  int sum = 0;
  for (int k = b0; k < b1; ++k) {
    const int r = sorted[k];
    int nb;
    bool pl;
    sum += units_of(p.q * (p.cand_off[r + 1] - p.cand_off[r]), nb, pl);
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
  const int whole = p.max_units - p.n_split, first_split = whole - p.n_split;
  auto put = [&](int u, int4 e) {
    if (u >= whole || u < 0) {
      record_error(p.ws, ROCS_ERR_DEVICE_INDEX, 801);
    } else if (u < first_split) {
      p.units[u] = e;
    } else {  // the two halves of split unit i, claimed one after the other
      const int i = u - first_split;
      e.w |= (i << 3) | 1;
      p.units[first_split + 2 * i] = e;
      e.w ^= 3;  // half 1 -> 2
      p.units[first_split + 2 * i + 1] = e;
    }
  };
  for (int k = b0; k < b1; ++k) {  // first unit of each sorted position
    const int r = sorted[k];
    int nb;
    bool pl;
    start[k] = run;
    run += units_of(p.q * (p.cand_off[r + 1] - p.cand_off[r]), nb, pl);
  }
  if (t == T - 1) {
    start[R] = s_part[T - 1];
    if (s_part[T - 1] != whole) record_error(p.ws, ROCS_ERR_DEVICE_INDEX, 802);
  }
  __syncthreads();
  // every thread writes every T-th unit: its sorted position by binary search over start[], then the unit's
  // head and chunk (a few requests can own most of the units, so positions are not split over threads)
  const int n_all = start[R] < whole ? start[R] : whole;
  for (int u = t; u < n_all; u += T) {
    int lo = 0, hi = R - 1;  // last k with start[k] <= u
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (start[mid] <= u) lo = mid;
      else hi = mid - 1;
    }
    const int r = sorted[lo], local = u - start[lo];
    int nb;
    bool pl;
    units_of(p.q * (p.cand_off[r + 1] - p.cand_off[r]), nb, pl);
    const int nbw = pl ? nb - 1 : nb;  // chunks taken one head at a time
    if (local < p.H * nbw)
      put(u, make_int4(r, local / nbw, (local % nbw) * p.rows_per_unit, 0));
    else {
      const int hp = local - p.H * nbw;
      put(u, make_int4(r, 2 * hp, nbw * p.rows_per_unit, 2 * hp + 1 < p.H ? 4 : 0));
    }
  }
  for (int i = t; i < 8 * p.n_split; i += T) p.split_cnt[i] = 0;
  if (t == 0) *p.ticket = 0;
}

cudaError_t launch_dca_schedule(const DcaSchedParams& p, cudaStream_t st) {
  rocs_dca_schedule_kernel<<<1, 1024, 0, st>>>(p);
  return cudaGetLastError();
}

template <int DH>
static cudaError_t launch_t(const DcaParams& p, int grid, cudaStream_t st) {
  using L = DcaSmem<DH>;
  auto k = rocs_dca_sm100_kernel<DH>;
  static std::atomic<uint64_t> optin_done{0};  // one bit per device
  static std::atomic<int> regs_checked{0};       // a property of the binary: checked once per process
  if (!regs_checked.load(std::memory_order_acquire)) {
    // the setmaxnreg split is only valid for the register count it was computed for
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, k) != cudaSuccess || fa.numRegs != (int)kLaunchRegs) return cudaErrorInvalidConfiguration;
    regs_checked.store(1, std::memory_order_release);
  }
  cudaError_t e = ensure_smem_optin(optin_done, k, (int)L::alloc_bytes);
  if (e != cudaSuccess) return e;
  // programmatic dependent launch: set-up (barriers, TMEM, descriptor prefetch) overlaps the scheduling
  // kernel that precedes it on the stream
  return launch_dependent(k, grid, kThreads, L::alloc_bytes, st, p);
}

cudaError_t launch_dca_sm100(const DcaParams& p, int dh, int grid, cudaStream_t st) {
  if (dh == 128) return launch_t<128>(p, grid, st);
  if (dh == 64) return launch_t<64>(p, grid, st);
  return cudaErrorInvalidValue;
}

int dca_rows_per_unit() { return kRowsPerUnit; }

}  // namespace rocs
