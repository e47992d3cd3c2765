// Fused exact-attention forward for sm_100a (B200).
//
// What it computes ("FlashAttention (KO)": the attention formula, tiling,
// online softmax, fusion into one kernel):
//   O = softmax(scale * Q K^T + causal mask) V, LSE = ln sum exp(scale * Q K^T)
// without writing S to device memory.  The kernel is persistent: one CTA per
// SM walks work units (NT query tiles of 128 rows of one (batch, query head))
// in a static snake order over a list ordered heaviest first, keeping its
// tensor memory, barriers and rings across units, so one unit's loads and
// first score tile overlap the previous unit's epilogue.  Per unit it streams the
// KV head's K/V in blocks of BN keys through shared memory:
//
//   producer warps  TMA: a ring of K blocks, a ring of V blocks, and each
//                   unit's Q tiles once their buffers are free again
//   MMA warp        one thread issues tcgen05.mma:  S = Q K^T  into TMEM,
//                   then O += P V with P read from TMEM (it overwrites S);
//                   with O staged apart, a tile's first score tiles of the
//                   next unit follow its last P V of the current unit
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

#include <algorithm>

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
  // half their size), and so does head dim 64, whose rings have room to
  // spare: the next unit's Q tiles can then be loaded while this unit's O is
  // stored.  Head dims 128 and 256 stage O in the dead Q tile.
  static constexpr bool SEP_OSTAGE = FP8 || D == 64;
  static constexpr int O_STAGE_BYTES = SEP_OSTAGE ? NT * 128 * D * 2 : 0;
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
  // Column pairs c with (c mod 16) >= POLY_T take exp2 on the FMA pipe in
  // full blocks: 6 of 16 for bf16 at head dim 128, 5 of 16 otherwise (a sweep
  // of 3..7 of 16: head dim 128 bf16 +2 % at 6, head dim 64 and FP8 best at 5).
  static constexpr int POLY_T = (D == 128 && !FP8) ? 10 : 11;
  static constexpr float P_SHIFT = FP8 ? 4.0f : 0.0f;
  static constexpr int SOFTMAX_WARPS = 4 * NT;
  static constexpr int PRODUCER_WARP = SOFTMAX_WARPS;       // K loads
  static constexpr int MMA_WARP = SOFTMAX_WARPS + 1;
  static constexpr int V_PRODUCER_WARP = SOFTMAX_WARPS + 2;  // V loads, never queued behind K
  static constexpr int Q_PRODUCER_WARP = SOFTMAX_WARPS + 3;  // Q tiles, which wait for the previous epilogue
  // The four issuing warps form a full warpgroup, so the register budget can
  // move from it to the softmax warpgroups.
  static constexpr int THREADS = 32 * (SOFTMAX_WARPS + 4);
  static constexpr int LAUNCH_REGS = (65536 / THREADS) / 8 * 8;
  static constexpr int ISSUE_REGS = 56;
  // setmaxnreg.inc draws on the registers the block was launched with
  // (THREADS x LAUNCH_REGS), not on the SM's 65,536: the split must fit
  // that total, or the increase waits forever.
  static constexpr int SOFTMAX_REGS =
      ((THREADS * LAUNCH_REGS - 128 * ISSUE_REGS) / (SOFTMAX_WARPS * 32)) / 8 * 8 > 248
          ? 248
          : ((THREADS * LAUNCH_REGS - 128 * ISSUE_REGS) / (SOFTMAX_WARPS * 32)) / 8 * 8;
  static_assert(NT == 1 || 128 * ISSUE_REGS + SOFTMAX_WARPS * 32 * SOFTMAX_REGS <= THREADS * LAUNCH_REGS,
                "register split within the launch allocation");
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
  static constexpr int B_OF = B_OD + NT;      // one phase per unit: the tile's last P V is done
  // Q tile t may be reloaded: its staging of O has been read by the TMA store
  // (O staged in the Q tile), or its unit's last score tile is done (O staged
  // apart).  One phase per unit that arrives on it.
  static constexpr int B_QE = B_OF + NT;
  static constexpr int B_OR = B_QE + NT;      // the epilogue has read O of tile t from TMEM (4 warps)
  static constexpr int B_DR = B_OR + NT;
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
  int B, Hq, Nq, Nk, group, n_qblk, causal_off;
  int n_units;        // n_qblk * Hq * B work units
  float scale_log2;   // scale * log2(e) (FP8: times the Q and K descales)
  float o_mul;        // 1 (FP8: the V descale)
};

// Work unit u: query-block index slowest (heaviest first under the causal
// mask), then query head (heads of one KV group adjacent, so their K/V are
// read from L2), then batch.
struct Unit {
  int qblk, hq, b;
};

// The k-th unit of CTA `cta` in a grid of `grid` CTAs: a static snake order
// over the heaviest-first list (rounds of `grid` units, every other round
// taken backwards), so that under the causal mask each CTA's total work is
// even.  Returns -1 past the last unit.
__device__ __forceinline__ int unit_index(int cta, int grid, int k, int n_units) {
  const long long u = (long long)k * grid + ((k & 1) ? (grid - 1 - cta) : cta);
  return u < n_units ? (int)u : -1;
}
__device__ __forceinline__ Unit unit_of(const FwdArgs& a, int u, bool causal) {
  const int per = a.Hq * a.B;
  const int qi = u / per, r = u - qi * per;
  Unit x;
  x.qblk = causal ? (a.n_qblk - 1 - qi) : qi;
  x.hq = r % a.Hq;
  x.b = r / a.Hq;
  return x;
}

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

  // Key blocks each tile of unit x visits (0 for a tile past Nq, or one whose
  // rows see no key); returns the most over the tiles.
  auto unit_blocks = [&](const Unit& x, int* nblk) -> int {
    int nmax = 0;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int r0 = (x.qblk * NT + t) * C::BM;
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
    return nmax;
  };
  // A tile is active in unit x when it holds rows below Nq: its epilogue
  // writes O and LSE (zeros and -inf if it saw no key).
  auto tile_active = [&](const Unit& x, int t) { return (x.qblk * NT + t) * C::BM < a.Nq; };
  // Arrivals unit x brings on the Q-free barrier of tile t.
  auto qe_arrivals = [&](const Unit& x, const int* nblk, int t) -> int {
    return C::SEP_OSTAGE ? (nblk[t] > 0 ? 1 : 0) : (tile_active(x, t) ? 1 : 0);
  };

  if (threadIdx.x == 0) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      mbar_init(bar(C::B_QF + t), 1);
      mbar_init(bar(C::B_QE + t), 1);
      mbar_init(bar(C::B_OR + t), 4);   // one arrival per softmax warp of the tile
    }
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
    // ------------------------------------------------------------ K producer
    // K blocks of every unit through the K ring; never waits on an epilogue,
    // so the next unit's first blocks are loaded while this unit finishes.
    if (lane == 0) {
      int kc = 0;   // K blocks issued so far (ring slot and phase)
      bool ok = true;
      for (int k = 0, u; ok && (u = unit_index(blockIdx.x, gridDim.x, k, a.n_units)) >= 0; ++k) {
        const Unit x = unit_of(a, u, C::CAUSAL);
        int nblk[NT];
        const int nmax = unit_blocks(x, nblk);
        const int hk = x.hq / a.group;
        for (int j = 0; j < nmax; ++j, ++kc) {
          const int st = kc % KST;
          if (!mbar_wait(bar(C::B_KE + st), ((kc / KST) & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(C::B_KF + st), C::KV_BYTES);
#pragma unroll
          for (int ch = 0; ch < C::DCH; ++ch)
            tma_load_4d(base + C::OFF_K + st * C::KV_BYTES + ch * C::KV_CHUNK, &tm_k, bar(C::B_KF + st),
                        ch * C::CH_ELEMS, hk, j * BN, x.b);
        }
      }
      // Drain: every issued copy must land before shared memory is released.
      for (int j = max(0, kc - KST); j < kc; ++j) mbar_wait_drain(bar(C::B_KF + j % KST), (j / KST) & 1);
    }
    __syncwarp();
  } else if (warp == C::V_PRODUCER_WARP) {
    // ------------------------------------------------------------ V producer
    if (lane == 0) {
      int vc = 0;
      bool ok = true;
      for (int k = 0, u; ok && (u = unit_index(blockIdx.x, gridDim.x, k, a.n_units)) >= 0; ++k) {
        const Unit x = unit_of(a, u, C::CAUSAL);
        int nblk[NT];
        const int nmax = unit_blocks(x, nblk);
        const int hk = x.hq / a.group;
        for (int j = 0; j < nmax; ++j, ++vc) {
          const int st = vc % VST;
          if (!mbar_wait(bar(C::B_VE + st), ((vc / VST) & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(C::B_VF + st), C::KV_BYTES);
#pragma unroll
          for (int ch = 0; ch < C::DCH; ++ch)
            tma_load_4d(base + C::OFF_V + st * C::KV_BYTES + ch * C::KV_CHUNK, &tm_v, bar(C::B_VF + st),
                        ch * C::CH_ELEMS, hk, j * BN, x.b);
        }
      }
      for (int j = max(0, vc - VST); j < vc; ++j) mbar_wait_drain(bar(C::B_VF + j % VST), (j / VST) & 1);
    }
    __syncwarp();
  } else if (warp == C::Q_PRODUCER_WARP) {
    // ------------------------------------------------------------ Q producer
    // Q tile t of a unit is loaded once the tile's buffer is free again: its
    // O staging has been read by the previous epilogue's TMA store (O staged
    // in the Q tile) or the previous unit's last score tile is done.
    if (lane == 0) {
      int qld[NT] = {};   // Q loads issued per tile
      int qe[NT] = {};    // arrivals earlier units bring on the tile's Q-free barrier
      bool ok = true;
      for (int k = 0, u; ok && (u = unit_index(blockIdx.x, gridDim.x, k, a.n_units)) >= 0; ++k) {
        const Unit x = unit_of(a, u, C::CAUSAL);
        int nblk[NT];
        unit_blocks(x, nblk);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          if (!ok) break;
          if (nblk[t] > 0) {
            // the latest earlier arrival is the last one: a later unit's cannot
            // come before this load (it needs this Q, or has no Q tile to wait for)
            if (qe[t] > 0 && !mbar_wait(bar(C::B_QE + t), (qe[t] - 1) & 1, abort_flag, a.status)) {
              ok = false;
              break;
            }
            const int r0 = (x.qblk * NT + t) * C::BM;
            mbar_arrive_expect_tx(bar(C::B_QF + t), C::Q_BYTES);
#pragma unroll
            for (int ch = 0; ch < C::DCH; ++ch)
              tma_load_4d(base + C::OFF_Q + t * C::Q_BYTES + ch * C::Q_CHUNK, &tm_q, bar(C::B_QF + t),
                          ch * C::CH_ELEMS, x.hq, r0, x.b);
            ++qld[t];
          }
          qe[t] += qe_arrivals(x, nblk, t);
        }
      }
#pragma unroll
      for (int t = 0; t < NT; ++t)
        if (qld[t] > 0) mbar_wait_drain(bar(C::B_QF + t), (qld[t] - 1) & 1);
    }
    __syncwarp();
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the schedule (descriptors stay warp-uniform); one
    // elected lane issues each tcgen05 instruction, predicated (no branch).
    // Ring slots, S buffers and barrier phases are indexed by running counts
    // over the units, so they carry across units unchanged.
    const bool leader = elect_one();
    constexpr uint32_t idesc_s = C::FP8 ? idesc_e4m3_f32(128, BN, false) : idesc_bf16_f32(128, BN, false);
    constexpr uint32_t idesc_o = C::FP8 ? idesc_e4m3_f32(128, D, true) : idesc_bf16_f32(128, D, true);
    int kc = 0, vc = 0;   // K and V blocks consumed before this unit
    int sc[NT] = {};      // score tiles of tile t before this unit
    int qld[NT] = {};     // Q loads of tile t consumed
    int orc[NT] = {};     // epilogues of tile t before this unit (arrivals on its O-read barrier)
    int pre[NT] = {};     // score tiles of this unit issued while the previous one ran
    bool qpre[NT] = {};   // Q of tile t for this unit already waited for then
    bool ok = true;
    auto last_tile_of = [&](const int* nb, int j) {
      int lt = -1;
#pragma unroll
      for (int t = 0; t < NT; ++t)
        if (j < nb[t]) lt = t;
      return lt;
    };
    // S(t, j) of a unit whose K blocks start at ring count kb and whose tile-t
    // score tiles start at running count sb: Q_t K_j^T into S buffer (sb + j) % NSL.
    auto issue_s = [&](int t, int j, int kb, int sb, const int* nb) -> bool {
      const int kj = kb + j, st = kj % KST;
      if (!warp_wait(bar(C::B_KF + st), (kj / KST) & 1, abort_flag, a.status)) return false;
      tc_fence_after();
      const int c = sb + j;
      const uint32_t d_tmem = tmem + t * C::TILE_COLS + (c % NSL) * BN;
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
      mma_commit(bar(C::B_SF + t * NSL + (c % NSL)), leader);
      if (t == last_tile_of(nb, j)) mma_commit(bar(C::B_KE + st), leader);
      // O staged apart: the Q tile is free once the unit's last score tile is done
      if (C::SEP_OSTAGE && j == nb[t] - 1) mma_commit(bar(C::B_QE + t), leader);
      __syncwarp();
      return true;
    };
    for (int k = 0, u = unit_index(blockIdx.x, gridDim.x, 0, a.n_units); ok && u >= 0; ++k) {
      const Unit x = unit_of(a, u, C::CAUSAL);
      int nblk[NT];
      const int nmax = unit_blocks(x, nblk);
      const int un = unit_index(blockIdx.x, gridDim.x, k + 1, a.n_units);
      int nblk_n[NT] = {};
      if (un >= 0) unit_blocks(unit_of(a, un, C::CAUSAL), nblk_n);
      int pre_n[NT] = {};
      bool qpre_n[NT] = {};
#pragma unroll
      for (int t = 0; t < NT; ++t)
        if (ok && nblk[t] > 0 && !qpre[t]) {
          ok = warp_wait(bar(C::B_QF + t), qld[t] & 1, abort_flag, a.status);
          ++qld[t];
        }
      for (int i = 0; ok && i < NSL; ++i)
#pragma unroll
        for (int t = 0; t < NT; ++t)
          if (ok && i < nblk[t] && i >= pre[t]) ok = issue_s(t, i, kc, sc[t], nblk);

      for (int j = 0; ok && j < nmax; ++j) {
        const int vj = vc + j, st = vj % VST;
        bool v_ready = false;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          if (!ok || j >= nblk[t]) continue;
          const int c = sc[t] + j;
          if (!warp_wait(bar(C::B_PF + t * NSL + c % NSL), (c / NSL) & 1, abort_flag, a.status)) { ok = false; break; }
          if (!v_ready) {
            if (!warp_wait(bar(C::B_VF + st), (vj / VST) & 1, abort_flag, a.status)) { ok = false; break; }
            v_ready = true;
          }
          // The unit's first product overwrites O: the previous epilogue of
          // this tile must have read it (its latest arrival is the last one,
          // since the next epilogue needs this unit's products).
          if (j == 0 && orc[t] > 0 &&
              !warp_wait(bar(C::B_OR + t), (orc[t] - 1) & 1, abort_flag, a.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t p_tmem = tmem + t * C::TILE_COLS + (c % NSL) * BN;
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
          if (t == last_tile_of(nblk, j)) mma_commit(bar(C::B_VE + st), leader);
          __syncwarp();
          if (j + NSL < nblk[t]) {
            ok = issue_s(t, j + NSL, kc, sc[t], nblk);
          } else if (C::SEP_OSTAGE && j == nblk[t] - 1 && un >= 0 && nblk_n[t] > 0) {
            // Tile t is done with this unit.  Its score tiles of the next unit
            // are issued now if that unit's Q and K blocks have landed (tested,
            // not waited for), so they are computed during this tile's
            // epilogue instead of after the other tile's last products.  The
            // S buffers they overwrite held this unit's last blocks, whose
            // P V products were issued above.  (With O staged in the Q tile,
            // the next Q cannot have landed before this tile's epilogue.)
            if (__all_sync(0xffffffffu, mbar_try_wait(bar(C::B_QF + t), qld[t] & 1))) {
              ++qld[t];
              qpre_n[t] = true;
              tc_fence_after();
              for (int i = 0; ok && i < NSL && i < nblk_n[t]; ++i) {
                const int kj = kc + nmax + i;
                if (!__all_sync(0xffffffffu, mbar_try_wait(bar(C::B_KF + kj % KST), (kj / KST) & 1))) break;
                ok = issue_s(t, i, kc + nmax, sc[t] + nblk[t], nblk_n);
                ++pre_n[t];
              }
            }
          }
        }
      }
      kc += nmax;
      vc += nmax;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        sc[t] += nblk[t];
        orc[t] += tile_active(x, t) ? 1 : 0;
        pre[t] = pre_n[t];
        qpre[t] = qpre_n[t];
      }
      u = un;
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
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const uint32_t t_tmem = tmem + t * C::TILE_COLS + lane_off;
    const float sl2 = a.scale_log2;
    int sc = 0;    // score tiles of this tile before the current unit
    int ofc = 0;   // phases of this tile's last-product barrier consumed
    bool ok = true;
    for (int k = 0, u; ok && (u = unit_index(blockIdx.x, gridDim.x, k, a.n_units)) >= 0; ++k) {
      const Unit x = unit_of(a, u, C::CAUSAL);
      int nblk[NT];
      unit_blocks(x, nblk);
      const int n = nblk[t];
      const int r0 = (x.qblk * NT + t) * C::BM;
      const int row = r0 + row_in_tile;
      int lim = a.Nk;   // keys kk < lim are visible to this row
      if (C::CAUSAL) lim = min(a.Nk, row + a.causal_off + 1);
      float m_run = -INFINITY, l_run = 0.f;

      for (int j = 0; j < n; ++j) {
        const int c = sc + j;
        const int slot = c % NSL;
        if (!warp_wait(bar(C::B_SF + t * NSL + slot), (c / NSL) & 1, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        uint32_t s[BN];
        if constexpr (BN == 128) tmem_ld128_sync(t_tmem + slot * BN, s);
        else tmem_ld64_sync(t_tmem + slot * BN, s);

        const bool need_mask = ((j + 1) * BN > a.Nk) || (C::CAUSAL && (j + 1) * BN - 1 > r0 + a.causal_off);
        if (need_mask) {
          const int cl = lim - j * BN;
#pragma unroll
          for (int cc = 0; cc < BN; ++cc)
            if (cc >= cl) s[cc] = __float_as_uint(-INFINITY);
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
          sum = need_mask ? exp_row_e4m3<BN, false>(s, p, sl2, m_eff)
                          : exp_row_e4m3<BN, true, C::POLY_T>(s, p, sl2, m_eff);
        else
          sum = need_mask ? exp_row<BN, false>(s, p, sl2, m_eff) : exp_row<BN, true, C::POLY_T>(s, p, sl2, m_eff);
        l_run = l_run * alpha + sum;
        m_run = m_use;
        static_assert(C::P_WORDS % 32 == 0, "P rows are stored 32 columns at a time");
#pragma unroll
        for (int cc = 0; cc < C::P_WORDS / 32; ++cc) tmem_st32(t_tmem + slot * BN + cc * 32, p + cc * 32);
        tmem_st_wait();
        if (j > 0 && __any_sync(0xffffffffu, grow)) {
          // O must hold P_{j-1} V_{j-1} before it is rescaled.  The wait is
          // unambiguous although most phases of this barrier are never waited
          // on: S_j is done, so every P V issued before it (up to P_{j-2} V_{j-2})
          // is done, and P_j V_j cannot start before this warp's arrival below;
          // the barrier therefore sits at phase c-1 or c (c = running index of S_j).
          if (!warp_wait(bar(C::B_OD + t), (c - 1) & 1, abort_flag, a.status)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32_sync(t_tmem + C::O_COL + cc * 32, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(t_tmem + C::O_COL + cc * 32, o);
          }
          tmem_st_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::B_PF + t * NSL + slot));
      }
      sc += n;

      // ------------------------------------------------------------ epilogue
      if (!tile_active(x, t)) continue;
      if (ok && n > 0) {
        ok = warp_wait(bar(C::B_OF + t), ofc & 1, abort_flag, a.status);
        tc_fence_after();
      }
      if (n > 0) ++ofc;
      // O staged apart: the previous unit's TMA store of this staging area
      // is waited for here, just before it is rewritten, not right after it
      // was issued.
      if (C::SEP_OSTAGE && wq == 0 && lane == 0) tma_store_wait_read();
      // The four warps of the tile take the same path from here on (a warp
      // whose wait failed must not leave the others at a named barrier); the
      // barrier also orders this staging after the previous unit's TMA store
      // of the same area, which its issuing thread waited for before arriving.
      ok = named_bar_and(1 + t, 128, ok && !*abort_flag);
      const bool write = ok;
      // bf16 O staging: the dead Q tile, or a region of its own
      const uint32_t stage = C::SEP_OSTAGE ? base + C::OFF_OST + t * (128 * D * 2) : base + C::OFF_Q + t * C::Q_BYTES;
      const float inv_l = (l_run > 0.f) ? a.o_mul / l_run : 0.f;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        if (write && n > 0) {
          tmem_ld32_sync(t_tmem + C::O_COL + cc * 32, o);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        if (write) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
          const uint32_t chunk = stage + (cc >> 1) * C::Q_CHUNK + row_in_tile * 128;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t unit = ((cc & 1) * 4 + i) ^ (row_in_tile & 7);
            st_shared_v4(chunk + unit * 16, pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      }
      // O of this tile has been read: the next unit's first product may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_OR + t));
      if (write) fence_proxy_async_smem();
      named_bar_sync(1 + t, 128);
      if (wq == 0 && lane == 0) {
        if (write) {
#pragma unroll
          for (int ch = 0; ch < D / 64; ++ch) tma_store_4d(&tm_o, stage + ch * C::Q_CHUNK, ch * 64, x.hq, r0, x.b);   // bf16 O
          tma_store_commit();
          if (!C::SEP_OSTAGE) tma_store_wait_read();
        }
        if (!C::SEP_OSTAGE) mbar_arrive(bar(C::B_QE + t));   // the Q tile may be reloaded
      }
      if (write && row < a.Nq)
        a.lse[((size_t)x.b * a.Hq + x.hq) * a.Nq + row] =
            (l_run > 0.f) ? (m_run - C::P_SHIFT + log2f(l_run)) * kLn2 : -INFINITY;
      __syncwarp();
    }
    // the last TMA store of O has read its staging before the CTA ends
    if (C::SEP_OSTAGE && wq == 0 && lane == 0) tma_store_wait_all();
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
  // 128-key blocks for head dims 64 and 128 (64-key blocks with two score
  // buffers per tile measured slower there: 1169 against 1299 TFLOP/s for
  // FP8, no change for head dim 64), 64-key blocks for head dim 256, whose
  // single tile then fits two score buffers next to its 256-column O.
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
  a.B = B;
  const long long units = (long long)a.n_qblk * Hq * B;
  if (units >= (1ll << 31)) return ATTN_ERR_UNSUPPORTED;
  a.n_units = (int)units;
  a.causal_off = Nk - Nq;
  a.scale_log2 = scale * qk_descale * 1.4426950408889634f;
  a.o_mul = v_descale;
  // Persistent: one CTA per SM (the shared memory allows no more), each
  // walking its units in the snake order.
  const int sms = current_sm_count();
  if (sms < 1) return ATTN_ERR_CUDA;
  const int grid = (int)std::min<long long>(units, sms);
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
