// Fused exact-attention forward for sm_100a (B200).
//
// What it computes ("FlashAttention (KO)": the attention formula, tiling,
// online softmax, fusion into one kernel):
//   O = softmax(scale * Q K^T + causal mask) V, LSE = ln sum exp(scale * Q K^T)
// without writing S to device memory.  Each CTA owns NT query tiles of 128
// rows of one (batch, query head) and streams the KV head's K/V in blocks of
// BN keys through shared memory:
//
//   producer warp   TMA: Q tiles once, then a ring of K and V blocks
//   MMA warp        one thread issues tcgen05.mma:  S = Q K^T  into TMEM,
//                   then O += P V with P read from TMEM (it overwrites S)
//   softmax WGs     one warpgroup per Q tile, one TMEM lane (= query row) per
//                   thread: load S, mask, running max, p = 2^(s*scale*log2e - m),
//                   running sum, P -> bf16 -> TMEM; rescale O only when the
//                   row max grew by more than 2^8 (exact: O and the sum share
//                   the same reference max); epilogue O/l -> bf16 -> TMA store,
//                   LSE -> fp32.
//
// Two Q tiles per CTA (head dims 64 and 128) let the tensor core work on one
// tile while the other tile's softmax runs.  Head dim 256 keeps one tile with
// two S buffers instead (TMEM holds 128 lanes x 512 fp32 columns: O alone
// takes 256 of them).
//
// FP8 option (attn_fwd_fp8, head dim 128; "FlashAttention (KO)", section
// "FlashAttention-3 (2024)"): Q, K, V tiles hold E4M3 bytes, both products
// run as kind::f8f6f4 MMAs (32 bytes = 32 elements of reduction per MMA), P is
// rounded to e4m3 and packed four to a TMEM column, and the Q/K descales are
// folded into the score scale and the V descale into the epilogue.
#include <math.h>

#include "host_common.h"
#include "sm100.cuh"
#include "softmax_row.cuh"

namespace ea {

template <int D_, bool CAUSAL_, int BN_, bool FP8_ = false>
struct FwdCfg {
  static constexpr int D = D_;
  static constexpr bool CAUSAL = CAUSAL_;
  // FP8: Q, K, V are e4m3 bytes and P is rounded to e4m3 for P V (O, LSE as
  // in the bf16 path).
  static constexpr bool FP8 = FP8_;
  static constexpr int ES = FP8 ? 1 : 2;             // bytes per Q/K/V element
  static constexpr int BM = 128;                     // query rows per tile = TMEM lanes
  static constexpr int NT = (D <= 128) ? 2 : 1;      // Q tiles per CTA
  static constexpr int BN = BN_;                     // keys per block
  // S buffers per tile: two whenever they fit next to O in the tile's 256
  // TMEM columns, so S of block j+1 overlaps the softmax of block j.
  static constexpr int NSL = (NT == 1 || 2 * BN + D <= 256) ? 2 : 1;
  static constexpr int KV_TILE = BN * D * ES;
  // FP8 stages the bf16 O tiles in a region of their own (the e4m3 Q tile is
  // half their size); bf16 reuses the dead Q tile.
  static constexpr int O_STAGE_BYTES = FP8 ? NT * 128 * D * 2 : 0;
  static constexpr int KV_BUDGET = 224 * 1024 - NT * BM * D * ES - O_STAGE_BYTES;   // shared memory left for K/V
  static constexpr int KSTAGES = (KV_BUDGET / KV_TILE + 1) / 2;      // K ring (released after S)
  static constexpr int VSTAGES = KV_BUDGET / KV_TILE - KSTAGES;      // V ring (held until P V)
  static constexpr int DCH = D * ES / 128;           // 128-byte column chunks
  static constexpr int CH_ELEMS = 128 / ES;          // elements in a 128-byte chunk row
  static constexpr int K_MMA = 32 / ES;              // reduction depth of one MMA (32 bytes)
  static constexpr int P_WORDS = BN * ES / 4;        // TMEM columns of one packed P row
  static constexpr int Q_CHUNK = BM * 128;           // bytes of one chunk of a Q tile
  static constexpr int KV_CHUNK = BN * 128;
  static constexpr int Q_BYTES = BM * D * ES;
  static constexpr int KV_BYTES = BN * D * ES;
  // Lazy rescale: O is rescaled only when a row max grows by more than 2^THR.
  // FP8 also measures p from 2^SHIFT below the running max, so that p lies in
  // (0, 2^(THR + SHIFT)] = (0, 256]: inside e4m3's range (max 448) and mostly
  // above its smallest normal (2^-6).
  static constexpr float RESCALE_THR = FP8 ? 4.0f : 8.0f;
  static constexpr float P_SHIFT = FP8 ? 4.0f : 0.0f;
  static constexpr int SOFTMAX_WARPS = 4 * NT;
  static constexpr int PRODUCER_WARP = SOFTMAX_WARPS;       // Q and K loads
  static constexpr int MMA_WARP = SOFTMAX_WARPS + 1;
  static constexpr int V_PRODUCER_WARP = SOFTMAX_WARPS + 2;  // V loads, never queued behind K
  // The three issuing warps plus one idle warp form a full warpgroup, so the
  // register budget can move from it to the softmax warpgroups.
  static constexpr int THREADS = 32 * (SOFTMAX_WARPS + 4);
  static constexpr int LAUNCH_REGS = (65536 / THREADS) / 8 * 8;
  static constexpr int ISSUE_REGS = 56;
  static constexpr int SOFTMAX_REGS =
      ((65536 - 128 * ISSUE_REGS) / (SOFTMAX_WARPS * 32)) / 8 * 8 > 248
          ? 248
          : ((65536 - 128 * ISSUE_REGS) / (SOFTMAX_WARPS * 32)) / 8 * 8;
  // TMEM columns: tile t owns [t*TILE_COLS, ...): NSL S buffers of BN
  // columns, then O (D columns).
  static constexpr int TILE_COLS = 256;
  static constexpr int O_COL = NSL * BN;
  static constexpr int TMEM_COLS = 512;
  // barriers
  static constexpr int B_QF = 0;
  static constexpr int B_KF = B_QF + NT;
  static constexpr int B_KE = B_KF + KSTAGES;
  static constexpr int B_VF = B_KE + KSTAGES;
  static constexpr int B_VE = B_VF + VSTAGES;
  static constexpr int B_SF = B_VE + VSTAGES;
  // P ready, one per (tile, S buffer): the softmax of block j+NSL cannot
  // arrive before the MMA warp has taken block j's phase (S_{j+NSL} is only
  // issued after P_j V_j), so no barrier ever runs two phases ahead.
  static constexpr int B_PF = B_SF + NT * NSL;
  static constexpr int B_OD = B_PF + NT * NSL;      // one phase per P V product of the tile
  static constexpr int B_OF = B_OD + NT;      // single phase: the tile's last P V is done
  static constexpr int B_DR = B_OF + NT;
  static constexpr int NBAR = B_DR + 1;
  // shared memory (offsets from a 1024-byte aligned base)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NT * Q_BYTES;
  static constexpr int OFF_V = OFF_K + KSTAGES * KV_BYTES;
  static constexpr int OFF_OST = OFF_V + VSTAGES * KV_BYTES;   // FP8 only: bf16 O staging
  static constexpr int OFF_BAR = OFF_OST + O_STAGE_BYTES;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(O_COL + D <= TILE_COLS || NT == 1, "TMEM budget per tile");
  static_assert(NT * TILE_COLS <= TMEM_COLS || NT == 1, "TMEM budget");
  static_assert(O_COL + D <= TMEM_COLS, "TMEM budget");
};

struct FwdArgs {
  float* lse;
  int* status;
  int Hq, Nq, Nk, group, n_qblk, causal_off;
  float scale_log2;   // scale * log2(e) (FP8: times the Q and K descales)
  float o_mul;        // 1 (FP8: the V descale)
};

constexpr float kLn2 = 0.6931471805599453f;

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    const FwdArgs a) {
  constexpr int NT = C::NT, BN = C::BN, NSL = C::NSL, KST = C::KSTAGES, VST = C::VSTAGES, D = C::D;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::OFF_MISC + 4);
  auto bar = [&](int i) -> uint32_t { return base + C::OFF_BAR + 8u * i; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qblk = C::CAUSAL ? (a.n_qblk - 1 - (int)blockIdx.x) : (int)blockIdx.x;   // heaviest first
  const int hq = blockIdx.y, b = blockIdx.z;
  const int hk = hq / a.group;

  // Number of key blocks each tile visits.
  int nblk[NT];
  int nmax = 0;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int r0 = (qblk * NT + t) * C::BM;
    int n = 0;
    if (r0 < a.Nq) {
      int kv_end = a.Nk;
      if (C::CAUSAL) {
        const int last_row = min(r0 + C::BM, a.Nq) - 1;
        kv_end = min(a.Nk, last_row + a.causal_off + 1);
      }
      n = kv_end > 0 ? (kv_end + BN - 1) / BN : 0;
    }
    nblk[t] = n;
    nmax = max(nmax, n);
  }

  if (threadIdx.x == 0) {
#pragma unroll
    for (int t = 0; t < NT; ++t) mbar_init(bar(C::B_QF + t), 1);
#pragma unroll
    for (int s = 0; s < KST; ++s) {
      mbar_init(bar(C::B_KF + s), 1);
      mbar_init(bar(C::B_KE + s), 1);
    }
#pragma unroll
    for (int s = 0; s < VST; ++s) {
      mbar_init(bar(C::B_VF + s), 1);
      mbar_init(bar(C::B_VE + s), 1);
    }
#pragma unroll
    for (int i = 0; i < NT * NSL; ++i) {
      mbar_init(bar(C::B_SF + i), 1);
      mbar_init(bar(C::B_PF + i), 4);   // one arrival per softmax warp
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      mbar_init(bar(C::B_OD + t), 1);
      mbar_init(bar(C::B_OF + t), 1);
    }
    mbar_init(bar(C::B_DR), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == C::PRODUCER_WARP && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_o);
  }
  if (warp == 0) {
    tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= C::SOFTMAX_WARPS) {
    // ============================================================ issue warpgroup
    if constexpr (C::NT == 2) regs_decrease<C::ISSUE_REGS>();
  if (warp == C::PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        if (nblk[t] > 0) {
          const int r0 = (qblk * NT + t) * C::BM;
          mbar_arrive_expect_tx(bar(C::B_QF + t), C::Q_BYTES);
#pragma unroll
          for (int ch = 0; ch < C::DCH; ++ch)
            tma_load_4d(base + C::OFF_Q + t * C::Q_BYTES + ch * C::Q_CHUNK, &tm_q, bar(C::B_QF + t),
                        ch * C::CH_ELEMS, hq, r0, b);
        }
      }
      int k_issued = 0;
      for (int j = 0; j < nmax; ++j) {
        const int st = j % KST;
        if (!mbar_wait(bar(C::B_KE + st), ((j / KST) & 1) ^ 1, abort_flag, a.status)) break;
        mbar_arrive_expect_tx(bar(C::B_KF + st), C::KV_BYTES);
#pragma unroll
        for (int ch = 0; ch < C::DCH; ++ch)
          tma_load_4d(base + C::OFF_K + st * C::KV_BYTES + ch * C::KV_CHUNK, &tm_k, bar(C::B_KF + st),
                      ch * C::CH_ELEMS, hk, j * BN, b);
        ++k_issued;
      }
      // Drain: every issued copy must land before shared memory is released.
      for (int j = max(0, k_issued - KST); j < k_issued; ++j) mbar_wait_drain(bar(C::B_KF + j % KST), (j / KST) & 1);
#pragma unroll
      for (int t = 0; t < NT; ++t)
        if (nblk[t] > 0) mbar_wait_drain(bar(C::B_QF + t), 0);
    }
    __syncwarp();
  } else if (warp == C::V_PRODUCER_WARP) {
    // ------------------------------------------------------------ V producer
    if (lane == 0) {
      int v_issued = 0;
      for (int j = 0; j < nmax; ++j) {
        const int st = j % VST;
        if (!mbar_wait(bar(C::B_VE + st), ((j / VST) & 1) ^ 1, abort_flag, a.status)) break;
        mbar_arrive_expect_tx(bar(C::B_VF + st), C::KV_BYTES);
#pragma unroll
        for (int ch = 0; ch < C::DCH; ++ch)
          tma_load_4d(base + C::OFF_V + st * C::KV_BYTES + ch * C::KV_CHUNK, &tm_v, bar(C::B_VF + st),
                      ch * C::CH_ELEMS, hk, j * BN, b);
        ++v_issued;
      }
      for (int j = max(0, v_issued - VST); j < v_issued; ++j) mbar_wait_drain(bar(C::B_VF + j % VST), (j / VST) & 1);
    }
    __syncwarp();
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the schedule (descriptors stay warp-uniform); one
    // elected lane issues each tcgen05 instruction, predicated (no branch).
    const bool leader = elect_one();
    constexpr uint32_t idesc_s = C::FP8 ? idesc_e4m3_f32(128, BN, false) : idesc_bf16_f32(128, BN, false);
    constexpr uint32_t idesc_o = C::FP8 ? idesc_e4m3_f32(128, D, true) : idesc_bf16_f32(128, D, true);
    bool ok = true;
#pragma unroll
    for (int t = 0; t < NT; ++t)
      if (ok && nblk[t] > 0) ok = warp_wait(bar(C::B_QF + t), 0, abort_flag, a.status);

    auto last_tile = [&](int j) {
      int lt = -1;
#pragma unroll
      for (int t = 0; t < NT; ++t)
        if (j < nblk[t]) lt = t;
      return lt;
    };
    // S(t, j) = Q_t K_j^T into S buffer j % NSL of tile t.
    auto issue_s = [&](int t, int j) -> bool {
      const int st = j % KST;
      if (!warp_wait(bar(C::B_KF + st), (j / KST) & 1, abort_flag, a.status)) return false;
      tc_fence_after();
      const uint32_t d_tmem = tmem + t * C::TILE_COLS + (j % NSL) * BN;
      const uint64_t qdesc = sdesc_sw128(base + C::OFF_Q + t * C::Q_BYTES, 16, 1024);
      const uint64_t kdesc = sdesc_sw128(base + C::OFF_K + st * C::KV_BYTES, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < D / C::K_MMA; ++ks) {
        // advance the start-address field (16-byte units) to k-step ks (32 bytes of a row)
        const uint32_t dq = ((ks >> 2) * C::Q_CHUNK + (ks & 3) * 32) >> 4;
        const uint32_t dk = ((ks >> 2) * C::KV_CHUNK + (ks & 3) * 32) >> 4;
        if constexpr (C::FP8) mma_ss_f8(d_tmem, qdesc + dq, kdesc + dk, idesc_s, ks > 0, leader);
        else mma_ss(d_tmem, qdesc + dq, kdesc + dk, idesc_s, ks > 0, leader);
      }
      mma_commit(bar(C::B_SF + t * NSL + (j % NSL)), leader);
      if (t == last_tile(j)) mma_commit(bar(C::B_KE + st), leader);
      __syncwarp();
      return true;
    };

    for (int i = 0; ok && i < NSL; ++i)
#pragma unroll
      for (int t = 0; t < NT; ++t)
        if (ok && i < nblk[t]) ok = issue_s(t, i);

    for (int j = 0; ok && j < nmax; ++j) {
      const int st = j % VST;
      bool v_ready = false;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        if (!ok || j >= nblk[t]) continue;
        if (!warp_wait(bar(C::B_PF + t * NSL + j % NSL), (j / NSL) & 1, abort_flag, a.status)) { ok = false; break; }
        if (!v_ready) {
          if (!warp_wait(bar(C::B_VF + st), (j / VST) & 1, abort_flag, a.status)) { ok = false; break; }
          v_ready = true;
        }
        tc_fence_after();
        const uint32_t p_tmem = tmem + t * C::TILE_COLS + (j % NSL) * BN;
        const uint32_t o_tmem = tmem + t * C::TILE_COLS + C::O_COL;
        const uint64_t vdesc = sdesc_sw128(base + C::OFF_V + st * C::KV_BYTES, C::KV_CHUNK, 1024);
#pragma unroll
        for (int ks = 0; ks < BN / C::K_MMA; ++ks) {
          // K_MMA keys per step: 8 TMEM columns of packed P, K_MMA rows of V
          const uint64_t vd = vdesc + ((ks * C::K_MMA * 128) >> 4);
          if constexpr (C::FP8) mma_ts_f8(o_tmem, p_tmem + ks * 8, vd, idesc_o, (j > 0 || ks > 0) ? 1u : 0u, leader);
          else mma_ts(o_tmem, p_tmem + ks * 8, vd, idesc_o, (j > 0 || ks > 0) ? 1u : 0u, leader);
        }
        mma_commit(bar(C::B_OD + t), leader);
        if (j == nblk[t] - 1) mma_commit(bar(C::B_OF + t), leader);
        if (t == last_tile(j)) mma_commit(bar(C::B_VE + st), leader);
        __syncwarp();
        if (j + NSL < nblk[t]) ok = issue_s(t, j + NSL);
      }
    }
    // Drain: no MMA may still run when TMEM is released.
    mma_commit(bar(C::B_DR), leader);
    __syncwarp();
    mbar_wait_drain(bar(C::B_DR), 0);
    __syncwarp();
  }
  } else {
    // ------------------------------------------------------------ softmax
    if constexpr (C::NT == 2) regs_increase<C::SOFTMAX_REGS>();
    const int t = warp >> 2;
    const int wq = warp & 3;
    const int row_in_tile = wq * 32 + lane;
    const int r0 = (qblk * NT + t) * C::BM;
    const int row = r0 + row_in_tile;
    const int n = nblk[t];
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const uint32_t t_tmem = tmem + t * C::TILE_COLS + lane_off;
    int lim = a.Nk;   // keys kk < lim are visible to this row
    if (C::CAUSAL) lim = min(a.Nk, row + a.causal_off + 1);
    const float sl2 = a.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;

    for (int j = 0; j < n; ++j) {
      const int slot = j % NSL;
      if (!warp_wait(bar(C::B_SF + t * NSL + slot), (j / NSL) & 1, abort_flag, a.status)) { ok = false; break; }
      tc_fence_after();
      uint32_t s[BN];
if constexpr (BN == 128) tmem_ld128_sync(t_tmem + slot * BN, s);
      else tmem_ld64_sync(t_tmem + slot * BN, s);

      const bool need_mask = ((j + 1) * BN > a.Nk) || (C::CAUSAL && (j + 1) * BN - 1 > r0 + a.causal_off);
      if (need_mask) {
        const int cl = lim - j * BN;
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c >= cl) s[c] = __float_as_uint(-INFINITY);
      }
      const float mx = row_max<BN>(s);
      const float m_new = fmaxf(m_run, mx * sl2);
      const bool grow = m_new > m_run + C::RESCALE_THR;
      const float m_use = grow ? m_new : m_run;
      const float alpha = grow ? ex2(m_run - m_use) : 1.f;
      // p is measured from 2^P_SHIFT below the reference max (l and O carry
      // the same factor, so O/l is unchanged; the LSE subtracts it again)
      const float m_eff = ((m_use == -INFINITY) ? 0.f : m_use) - C::P_SHIFT;
      uint32_t p[C::P_WORDS];
      // Blocks with masked keys use the MUFU exp2 only (masked scores are -inf
      // and must give exactly 0); full blocks send part of the work to the FMA pipe.
      float sum;
      if constexpr (C::FP8)
        sum = need_mask ? exp_row_e4m3<BN, false>(s, p, sl2, m_eff) : exp_row_e4m3<BN, true>(s, p, sl2, m_eff);
      else
        sum = need_mask ? exp_row<BN, false>(s, p, sl2, m_eff) : exp_row<BN, true>(s, p, sl2, m_eff);
      l_run = l_run * alpha + sum;
      m_run = m_use;
#pragma unroll
      for (int c = 0; c < C::P_WORDS / 32; ++c) tmem_st32(t_tmem + slot * BN + c * 32, p + c * 32);
      tmem_st_wait();
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        // O must hold P_{j-1} V_{j-1} before it is rescaled.  The wait is
        // unambiguous although most phases of this barrier are never waited
        // on: S_j is done, so every P V issued before it (up to P_{j-2} V_{j-2})
        // is done, and P_j V_j cannot start before this warp's arrival below;
        // the barrier therefore sits at phase j-1 or j.
        if (!warp_wait(bar(C::B_OD + t), (j - 1) & 1, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32_sync(t_tmem + C::O_COL + c * 32, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(t_tmem + C::O_COL + c * 32, o);
        }
        tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_PF + t * NSL + slot));
    }

    // ------------------------------------------------------------ epilogue
    if (ok && n > 0) {
      ok = warp_wait(bar(C::B_OF + t), 0, abort_flag, a.status);
      tc_fence_after();
    }
    const bool write = ok && !*abort_flag;
    // bf16 O staging: the dead Q tile, or (FP8, whose Q tile is smaller) a region of its own
    const uint32_t stage = C::FP8 ? base + C::OFF_OST + t * (128 * D * 2) : base + C::OFF_Q + t * C::Q_BYTES;
    if (write) {
      const float inv_l = (l_run > 0.f) ? a.o_mul / l_run : 0.f;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (n > 0) {
          tmem_ld32_sync(t_tmem + C::O_COL + c * 32, o);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
        const uint32_t chunk = stage + (c >> 1) * C::Q_CHUNK + row_in_tile * 128;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t unit = ((c & 1) * 4 + i) ^ (row_in_tile & 7);
          st_shared_v4(chunk + unit * 16, pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      fence_proxy_async_smem();
    }
    named_bar_sync(1 + t, 128);
    if (write && wq == 0 && lane == 0 && r0 < a.Nq) {
#pragma unroll
      for (int ch = 0; ch < D / 64; ++ch) tma_store_4d(&tm_o, stage + ch * C::Q_CHUNK, ch * 64, hq, r0, b);   // bf16 O
      tma_store_commit();
      tma_store_wait_read();
    }
    if (write && row < a.Nq)
      a.lse[((size_t)b * a.Hq + hq) * a.Nq + row] =
          (l_run > 0.f) ? (m_run - C::P_SHIFT + log2f(l_run)) * kLn2 : -INFINITY;
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D, bool CAUSAL, bool FP8 = false>
int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
               int Nk, float scale, cudaStream_t stream, float qk_descale = 1.f, float v_descale = 1.f) {
  using C = FwdCfg<D, CAUSAL, (D <= 128) ? 128 : 64, FP8>;
  static int attr_done = 0;
  const void* kfn = reinterpret_cast<const void*>(&attn_fwd_kernel<C>);
  if (int rc = ensure_smem_attr(kfn, C::SMEM_BYTES, &attr_done)) return rc;
  int* status = device_status_ptr();
  if (!status) return ATTN_ERR_CUDA;

  CUtensorMap tq, tk, tv, to;
  const uint64_t es = C::ES;
  const uint32_t box_q[4] = {(uint32_t)C::CH_ELEMS, 1, (uint32_t)C::BM, 1};
  const uint32_t box_kv[4] = {(uint32_t)C::CH_ELEMS, 1, (uint32_t)C::BN, 1};
  auto encode_in = [&](CUtensorMap* m, const void* ptr, const uint64_t* dims, const uint64_t* strides,
                       const uint32_t* box) {
    return FP8 ? encode_u8_4d(m, ptr, dims, strides, box) : encode_bf16_4d(m, ptr, dims, strides, box);
  };
  {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)Hq, (uint64_t)Nq, (uint64_t)B};
    const uint64_t strides[3] = {D * es, (uint64_t)Hq * D * es, (uint64_t)Nq * Hq * D * es};
    if (!encode_in(&tq, q, dims, strides, box_q)) return ATTN_ERR_CUDA;
    // O is bf16 in both forms
    const uint64_t ostrides[3] = {D * 2ull, (uint64_t)Hq * D * 2, (uint64_t)Nq * Hq * D * 2};
    const uint32_t box_o[4] = {64, 1, (uint32_t)C::BM, 1};
    if (!encode_bf16_4d(&to, o, dims, ostrides, box_o)) return ATTN_ERR_CUDA;
  }
  {
    // With Nk == 0 no key block is ever loaded: describe a 1-row tensor at q.
    const uint64_t nk = Nk > 0 ? (uint64_t)Nk : 1;
    const void* kb = Nk > 0 ? k : q;
    const void* vb = Nk > 0 ? v : q;
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)Hkv, nk, (uint64_t)B};
    const uint64_t strides[3] = {D * es, (uint64_t)Hkv * D * es, nk * Hkv * D * es};
    if (!encode_in(&tk, kb, dims, strides, box_kv)) return ATTN_ERR_CUDA;
    if (!encode_in(&tv, vb, dims, strides, box_kv)) return ATTN_ERR_CUDA;
  }
  FwdArgs a;
  a.lse = lse;
  a.status = status;
  a.Hq = Hq;
  a.Nq = Nq;
  a.Nk = Nk;
  a.group = Hq / Hkv;
  a.n_qblk = (Nq + C::BM * C::NT - 1) / (C::BM * C::NT);
  a.causal_off = Nk - Nq;
  a.scale_log2 = scale * qk_descale * 1.4426950408889634f;
  a.o_mul = v_descale;
  dim3 grid(a.n_qblk, Hq, B);
  attn_fwd_kernel<C><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, to, a);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace ea

extern "C" int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                        int Nq, int Nk, int D, int Dv, int causal, float scale, void* stream) {
  using namespace ea;
  // k and v may be null when Nk == 0 (no key is ever read)
  if (!q || !o || !lse || (Nk > 0 && (!k || !v))) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 0 || Nk < 0 || B > 65535 || Hq > 65535) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (D != Dv) return ATTN_ERR_UNSUPPORTED;
  if (D != 64 && D != 128 && D != 256) return ATTN_ERR_UNSUPPORTED;
  if (Nq == 0) return ATTN_OK;
  if ((uint64_t)B * Nq * Hq * D * 2 >= (1ull << 40) || (uint64_t)B * Nk * Hkv * D * 2 >= (1ull << 40))
    return ATTN_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool c = causal != 0;
  switch (D) {
    case 64: return c ? launch_fwd<64, true>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, s)
                      : launch_fwd<64, false>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, s);
    case 128: return c ? launch_fwd<128, true>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, s)
                       : launch_fwd<128, false>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, s);
    default: return c ? launch_fwd<256, true>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, s)
                      : launch_fwd<256, false>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, s);
  }
}

extern "C" int attn_fwd_fp8(const void* q, const void* k, const void* v, float q_descale, float k_descale,
                            float v_descale, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nk, int D,
                            int causal, float scale, void* stream) {
  using namespace ea;
  if (!q || !o || !lse || (Nk > 0 && (!k || !v))) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 0 || Nk < 0 || B > 65535 || Hq > 65535) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  for (float d : {q_descale, k_descale, v_descale})
    if (!(d > 0.f) || !isfinite(d)) return ATTN_ERR_INVALID_ARG;
  if (D != 128) return ATTN_ERR_UNSUPPORTED;
  if (Nq == 0) return ATTN_OK;
  if ((uint64_t)B * Nq * Hq * D * 2 >= (1ull << 40) || (uint64_t)B * Nk * Hkv * D >= (1ull << 40))
    return ATTN_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const float qk = q_descale * k_descale;
  return causal ? launch_fwd<128, true, true>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, s, qk, v_descale)
                : launch_fwd<128, false, true>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, s, qk, v_descale);
}
