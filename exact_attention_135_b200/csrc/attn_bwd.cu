// Exact-attention backward pass for sm_100a (B200), with recomputation.
//
// What it computes ("Flash Attention" wiki page, section "구조화된 지식
// (Synthesized Content)", item "Recomputation (재계산)": the backward pass
// recomputes the intermediate matrices instead of reading stored N x N ones):
// the gradients of O = softmax(scale * Q K^T + causal mask) V for an upstream
// gradient dO, with S and P rebuilt block by block from Q, K and the forward's
// LSE.  For one query head and its KV head:
//
//   P  = exp(scale * Q K^T - LSE)            (0 where masked)
//   dV = P^T dO        dP = dO V^T           Drow = rowsum(dO * O)
//   dS = P * (dP - Drow)
//   dQ = scale * dS K  dK = scale * dS^T Q   (dK, dV summed over the group's heads)
//
// Drow equals rowsum(P * dP) because O = P V, which is what makes the softmax
// Jacobian cheap.  Three launches:
//
//   bwd_prep_kernel   Drow (fp32) from O and dO, and a zeroed fp32 dQ accumulator
//   attn_bwd_dqt_kernel (D = 128; described where it is defined) or
//   attn_bwd_kernel (D = 64, below)
//   bwd_dqt_kernel / bwd_dq_kernel   dQ accumulator -> bf16
//
// Both attention kernels run one CTA per (key block of 128, KV head, batch),
// in the order that unit_pos and choose_head_group describe.
// dK and dV stay in TMEM while the CTA walks every query block of every query
// head of the group that sees its keys; each step's dQ contribution is added
// to the accumulator by a TMA reduce-add (at L2, coalesced whole tiles).
//
// Roles inside attn_bwd_kernel (320 threads):
//   warps 0-3  (WG0)  one key row per thread: S^T, dP^T from TMEM, P -> bf16 into
//                     TMEM (for dV) and dS -> bf16 into shared memory (for dK
//                     and dQ: the same tile is K-major for dS^T and MN-major for dS)
//   warps 4-7  (WG1)  one query row per thread: dQ from TMEM -> shared memory
//                     (the dS tile, free once dQ is computed) -> TMA reduce-add;
//                     at the end dK, dV -> bf16 -> global
//   warp 8            TMA: K, V once; a two-stage ring of (Q, dO) tiles plus the
//                     step's LSE and Drow values
//   warp 9            tcgen05.mma issue
//
// TMEM (128 lanes x 512 fp32 columns): dV [0, D), dK [D, 2D), region A
// [2D, 2D+128) = S^T then P^T (bf16, first 64 columns), region B
// [2D+128, 2D+256) = dP^T then dQ.  Issue order per step i (tcgen05.mma
// executes in issue order, so an MMA may overwrite columns an earlier one
// reads):
//   dV_i (reads P^T_i) -> S^T_{i+1} (A) -> dK_i, dQ_i (read dS_i; dQ_i -> B)
//   -> [dQ_i drained by WG1] -> dP^T_{i+1} (B)
// so the next step's S^T is computed while WG0 still forms dS_i, and dQ's
// drain overlaps the next step's softmax work.
#include <math.h>

#include <algorithm>
#include <functional>
#include <mutex>
#include <queue>
#include <vector>

#include "host_common.h"
#include "sm100.cuh"
#include "softmax_row.cuh"

namespace ea {
namespace bwd {

template <int D_, bool CAUSAL_>
struct Cfg {
  static constexpr int D = D_;
  static constexpr bool CAUSAL = CAUSAL_;
  static constexpr int BM = 128;                   // query rows per step
  static constexpr int BN = 128;                   // keys per CTA = TMEM lanes
  static constexpr int DCH = D / 64;               // 128-byte column chunks of a tile
  static constexpr int CH = 128 * 128;             // bytes of one chunk of a 128-row tile
  static constexpr int TILE = 128 * D * 2;         // bytes of one 128-row bf16 tile
  static constexpr int DS_BYTES = BM * BN * 2;     // dS tile (A of dK K-major, A of dQ MN-major); dQ staging
  // shared memory (offsets from a 1024-byte aligned base)
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_DS = OFF_V + TILE;
  static constexpr int OFF_STAGE = OFF_DS + DS_BYTES;   // stage s: Q at +2s*TILE, dO at +(2s+1)*TILE
  static constexpr int OFF_ROWS = OFF_STAGE + 4 * TILE;  // stage s: lse2[128], drow[128] at +s*1024
  static constexpr int OFF_BAR = OFF_ROWS + 2 * 1024;
  // barriers
  static constexpr int B_KV = 0;
  static constexpr int B_QF = 1;        // [2] stage full (TMA bytes + producer arrival)
  static constexpr int B_QE = 3;        // [2] stage empty (MMA commit)
  static constexpr int B_SF = 5;        // S^T in TMEM
  static constexpr int B_DPF = 6;       // dP^T in TMEM
  static constexpr int B_DQF = 7;       // dQ in TMEM
  static constexpr int B_PR = 8;        // P^T stored (4 WG0 warps)
  static constexpr int B_DSR = 9;       // dS stored in TMEM and shared memory (4 WG0 warps)
  static constexpr int B_DQE = 10;      // dQ drained (4 WG1 warps)
  static constexpr int B_DONE = 11;     // every MMA of the CTA complete
  static constexpr int NBAR = 12;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int LAYOUT_BYTES = OFF_MISC + 16;
  static constexpr int MAX_SMEM = 227 * 1024;
  // Room for re-aligning the dynamic shared-memory base when it fits; the
  // kernel checks the alignment it got against what it was given.
  static constexpr int SMEM_BYTES = LAYOUT_BYTES + 1024 <= MAX_SMEM ? LAYOUT_BYTES + 1024 : MAX_SMEM;
  static_assert(LAYOUT_BYTES <= MAX_SMEM, "shared memory budget");
  // TMEM columns
  static constexpr int DV_COL = 0;
  static constexpr int DK_COL = D;
  static constexpr int A_COL = 2 * D;
  static constexpr int B_COL = 2 * D + 128;
  static constexpr int TMEM_COLS = 512;
  static_assert(B_COL + 128 <= TMEM_COLS, "TMEM budget");
  // Ten warps: the register file is split per SM sub-partition, so the
  // sub-partitions holding three warps cap every thread at 168 registers.
  static constexpr int THREADS = 320;
  static constexpr int PRODUCER_WARP = 8;
  static constexpr int MMA_WARP = 9;
};

struct Args {
  const float* lse;      // [B, Hq, Nq] natural log
  const float* drow;     // [B, Hq, Nq]
  __nv_bfloat16* dk;     // [B, Nk, Hkv, D]
  __nv_bfloat16* dv;     // [B, Nk, Hkv, D]
  int* status;
  int B, Hq, Hkv, Nq, Nk, group, n_qblk, n_kblk, causal_off;
  int head_group;        // heads (batch, KV head pairs) per group of the unit order
  float scale, scale_log2;
};

// Work unit u -> (key block, KV head, batch).  A head is one (batch, KV head)
// pair p = b * Hkv + hk.  Heads are taken head_group at a time, and inside a
// group the key block is the slower index, so with a causal mask the key
// blocks that see the most query blocks start first.  A group smaller than
// all heads makes the CTAs resident at once share the Q, dO and dQ
// accumulator rows of fewer heads, which then stay in L2 from one CTA to the
// next; head_group = Hkv * B is key block slowest over every head.
struct UnitPos {
  int kb, hk, b;
};
__device__ __forceinline__ UnitPos unit_pos(int u, const Args& a) {
  const int g = a.head_group;
  const int per_group = g * a.n_kblk;
  const int grp = u / per_group;
  const int r = u - grp * per_group;
  const int p0 = grp * g;
  const int gs = min(g, a.Hkv * a.B - p0);   // the last group may be smaller
  const int p = p0 + r % gs;
  return {r / gs, p % a.Hkv, p / a.Hkv};
}

constexpr float kLog2e = 1.4426950408889634f;

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dq, const Args a) {
  constexpr int D = C::D, TILE = C::TILE, CH = C::CH;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  if (base - raw + C::LAYOUT_BYTES > (uint32_t)C::SMEM_BYTES) {
    // The tiles would not fit behind the aligned base: refuse (every thread
    // takes this branch, nothing has been started yet).
    if (threadIdx.x == 0) atomicExch(a.status, ATTN_ERR_CUDA);
    return;
  }
  uint8_t* base_ptr = smem_raw + (base - raw);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::OFF_MISC + 4);
  auto bar = [&](int i) -> uint32_t { return base + C::OFF_BAR + 8u * i; };
  auto q_off = [&](int st) -> uint32_t { return base + C::OFF_STAGE + 2 * st * TILE; };
  auto do_off = [&](int st) -> uint32_t { return base + C::OFF_STAGE + (2 * st + 1) * TILE; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const UnitPos up = unit_pos(blockIdx.x, a);
  const int kb = up.kb, hk = up.hk, b = up.b;
  const int k0 = kb * C::BN;
  int qb_start = 0;
  if (C::CAUSAL) qb_start = max(0, (k0 - a.causal_off) / C::BM);   // first query block with a visible key
  const int nq = max(0, a.n_qblk - qb_start);
  const int nsteps = a.group * nq;
  // Steps walk the query blocks in order, the group's heads innermost: the
  // CTAs resident at one time (neighbouring key blocks) then work on
  // neighbouring query blocks, so the dQ accumulator rows they add into and
  // the Q / dO tiles they read stay in L2.
  auto step_head = [&](int i) { return hk * a.group + i % a.group; };
  auto step_q0 = [&](int i) { return (qb_start + i / a.group) * C::BM; };

  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_KV), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(C::B_QF + s), 1);
      mbar_init(bar(C::B_QE + s), 1);
    }
    mbar_init(bar(C::B_SF), 1);
    mbar_init(bar(C::B_DPF), 1);
    mbar_init(bar(C::B_DQF), 1);
    mbar_init(bar(C::B_PR), 4);
    mbar_init(bar(C::B_DSR), 4);
    mbar_init(bar(C::B_DQE), 4);
    mbar_init(bar(C::B_DONE), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == C::PRODUCER_WARP && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_dq);
  }
  if (warp == 0) {
    tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    if (warp == C::PRODUCER_WARP) {
      // ---------------------------------------------------------- producer
      if (nsteps > 0 && lane == 0) {
        mbar_arrive_expect_tx(bar(C::B_KV), 2 * TILE);
        for (int ch = 0; ch < C::DCH; ++ch) {
          tma_load_4d(base + C::OFF_K + ch * CH, &tm_k, bar(C::B_KV), ch * 64, hk, k0, b);
          tma_load_4d(base + C::OFF_V + ch * CH, &tm_v, bar(C::B_KV), ch * 64, hk, k0, b);
        }
      }
      int issued = 0;
      for (int j = 0; j < nsteps; ++j) {
        const int st = j & 1;
        if (!warp_wait(bar(C::B_QE + st), ((j >> 1) & 1) ^ 1, abort_flag, a.status)) break;
        const int hq = step_head(j), q0 = step_q0(j);
        float* lse_s = reinterpret_cast<float*>(base_ptr + C::OFF_ROWS + st * 1024);
        float* dr_s = lse_s + 128;
        const size_t rbase = ((size_t)b * a.Hq + hq) * a.Nq;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int c = 4 * lane + r, row = q0 + c;
          float l2 = INFINITY, d = 0.f;   // rows past Nq: p = 2^-inf = 0
          if (row < a.Nq) {
            const float l = a.lse[rbase + row];
            l2 = (l == -INFINITY) ? INFINITY : l * kLog2e;   // a row that saw no key keeps p = 0
            d = a.drow[rbase + row];
          }
          lse_s[c] = l2;
          dr_s[c] = d;
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_expect_tx(bar(C::B_QF + st), 2 * TILE);
          for (int ch = 0; ch < C::DCH; ++ch) {
            tma_load_4d(q_off(st) + ch * CH, &tm_q, bar(C::B_QF + st), ch * 64, hq, q0, b);
            tma_load_4d(do_off(st) + ch * CH, &tm_do, bar(C::B_QF + st), ch * 64, hq, q0, b);
          }
        }
        __syncwarp();
        ++issued;
      }
      // Drain: every issued copy must land before shared memory is released.
      if (lane == 0) {
        for (int j = max(0, issued - 2); j < issued; ++j) mbar_wait_drain(bar(C::B_QF + (j & 1)), (j >> 1) & 1);
        if (nsteps > 0) mbar_wait_drain(bar(C::B_KV), 0);
      }
      __syncwarp();
    } else if (warp == C::MMA_WARP) {
      // ---------------------------------------------------------- MMA issuer
      const bool leader = elect_one();
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, C::BM, false);     // S^T, dP^T: A, B K-major
      constexpr uint32_t idesc_g = idesc_bf16_f32(128, D, true);          // dV: A in TMEM; dK: A K-major; B MN-major
      constexpr uint32_t idesc_q = idesc_bf16_f32_amn(128, D, true);      // dQ: A, B MN-major
      bool ok = nsteps > 0 && warp_wait(bar(C::B_KV), 0, abort_flag, a.status);

      // S^T_i = K Q_i^T (region A) or dP^T_i = V dO_i^T (region B): both
      // operands K-major, k-steps of 16 along D.
      auto issue_kmajor = [&](uint32_t a_smem, uint32_t b_smem, uint32_t d_col, uint32_t bar_done) {
        const uint64_t adesc = sdesc_sw128(a_smem, 16, 1024);
        const uint64_t bdesc = sdesc_sw128(b_smem, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = ((ks >> 2) * CH + (ks & 3) * 32) >> 4;
          mma_ss(tmem + d_col, adesc + off, bdesc + off, idesc_s, ks > 0, leader);
        }
        mma_commit(bar_done, leader);
      };
      auto wait_stage = [&](int i) -> bool {
        if (!warp_wait(bar(C::B_QF + (i & 1)), (i >> 1) & 1, abort_flag, a.status)) return false;
        tc_fence_after();
        return true;
      };

      if (ok) ok = wait_stage(0);
      if (ok) {
        issue_kmajor(base + C::OFF_K, q_off(0), C::A_COL, bar(C::B_SF));
        issue_kmajor(base + C::OFF_V, do_off(0), C::B_COL, bar(C::B_DPF));
        __syncwarp();
      }
      for (int i = 0; ok && i < nsteps; ++i) {
        const int st = i & 1;
        if (!warp_wait(bar(C::B_PR), i & 1, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        {   // dV += P^T dO: A = P^T (TMEM, bf16), B = dO tile read MN-major
          const uint64_t bdesc = sdesc_sw128(do_off(st), CH, 1024);
#pragma unroll
          for (int ks = 0; ks < C::BM / 16; ++ks)
            mma_ts(tmem + C::DV_COL, tmem + C::A_COL + ks * 8, bdesc + ks * 128, idesc_g, (i > 0 || ks > 0) ? 1u : 0u,
                   leader);
        }
        if (i + 1 < nsteps) {
          if (!wait_stage(i + 1)) { ok = false; break; }
          issue_kmajor(base + C::OFF_K, q_off(st ^ 1), C::A_COL, bar(C::B_SF));
        }
        __syncwarp();
        if (!warp_wait(bar(C::B_DSR), i & 1, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        {   // dK += dS^T Q: A = dS^T (the dS tile read K-major: key rows, queries along K),
            // B = Q tile read MN-major
          const uint64_t adesc = sdesc_sw128(base + C::OFF_DS, 16, 1024);
          const uint64_t bdesc = sdesc_sw128(q_off(st), CH, 1024);
#pragma unroll
          for (int ks = 0; ks < C::BM / 16; ++ks) {
            const uint32_t a_off = ((ks >> 2) * (128 * 128) + (ks & 3) * 32) >> 4;
            mma_ss(tmem + C::DK_COL, adesc + a_off, bdesc + ks * 128, idesc_g, (i > 0 || ks > 0) ? 1u : 0u, leader);
          }
        }
        {   // dQ = dS K: A = dS (shared memory, MN-major), B = K tile read MN-major
          const uint64_t adesc = sdesc_sw128(base + C::OFF_DS, 128 * 128, 1024);
          const uint64_t bdesc = sdesc_sw128(base + C::OFF_K, CH, 1024);
#pragma unroll
          for (int ks = 0; ks < C::BN / 16; ++ks)
            mma_ss(tmem + C::B_COL, adesc + ks * 128, bdesc + ks * 128, idesc_q, ks > 0 ? 1u : 0u, leader);
        }
        mma_commit(bar(C::B_DQF), leader);
        mma_commit(bar(C::B_QE + st), leader);
        __syncwarp();
        if (i + 1 < nsteps) {
          if (!warp_wait(bar(C::B_DQE), i & 1, abort_flag, a.status)) { ok = false; break; }
          tc_fence_after();
          issue_kmajor(base + C::OFF_V, do_off(st ^ 1), C::B_COL, bar(C::B_DPF));
          __syncwarp();
        }
      }
      // Drain: no MMA may still run when TMEM is released (nothing was
      // issued when the CTA has no step).
      if (nsteps > 0) {
        mma_commit(bar(C::B_DONE), leader);
        __syncwarp();
        mbar_wait_drain(bar(C::B_DONE), 0);
      }
      __syncwarp();
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ WG0: P and dS
    const int kr = warp * 32 + lane;      // key row in the block = TMEM lane
    const int kk = k0 + kr;
    const bool row_valid = kk < a.Nk;
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    const uint32_t tA = tmem + lane_off + C::A_COL;
    const uint32_t tB = tmem + lane_off + C::B_COL;
    const float sl2 = a.scale_log2;
    for (int i = 0; i < nsteps; ++i) {
      const int st = i & 1, q0 = step_q0(i);
      // The stage's LSE / Drow values were stored by the producer before it
      // arrived on the stage barrier.
      if (!warp_wait(bar(C::B_QF + st), (i >> 1) & 1, abort_flag, a.status)) break;
      if (!warp_wait(bar(C::B_SF), i & 1, abort_flag, a.status)) break;
      tc_fence_after();
      const uint32_t rows_s = base + C::OFF_ROWS + st * 1024;
      // P^T row, rounded to bf16 once: the same values feed the dV product
      // and dS = P (dP - Drow) below.
      uint32_t pk[64];
      // Causal: key kk is visible to query q0 + c iff kk <= q0 + c + causal_off.
      const int cmin = row_valid ? (C::CAUSAL ? kk - a.causal_off - q0 : 0) : 128;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t s[64];
        tmem_ld64_sync(tA + half * 64, s);
#pragma unroll
        for (int j = 0; j < 64; j += 4) {
          const int c = half * 64 + j;
          uint32_t l0, l1, l2, l3;
          ld_shared_v4(rows_s + c * 4, l0, l1, l2, l3);
          const float p0 = ex2(fmaf(__uint_as_float(s[j + 0]), sl2, -__uint_as_float(l0)));
          const float p1 = ex2(fmaf(__uint_as_float(s[j + 1]), sl2, -__uint_as_float(l1)));
          const float p2 = ex2(fmaf(__uint_as_float(s[j + 2]), sl2, -__uint_as_float(l2)));
          const float p3 = ex2(fmaf(__uint_as_float(s[j + 3]), sl2, -__uint_as_float(l3)));
          pk[c / 2] = pack_bf16x2(p0, p1);
          pk[c / 2 + 1] = pack_bf16x2(p2, p3);
        }
      }
      if (cmin > 0) {
        // masked columns c < cmin: clear both halves of a pair, or only its
        // low half (column 2j) when the boundary falls inside the pair
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const uint32_t keep = (2 * j + 1 < cmin) ? 0u : (2 * j < cmin ? 0xffff0000u : 0xffffffffu);
          pk[j] &= keep;
        }
      }
      tmem_st32(tA, pk);
      tmem_st32(tA + 32, pk + 32);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_PR));

      if (!warp_wait(bar(C::B_DPF), i & 1, abort_flag, a.status)) break;
      tc_fence_after();
      const uint32_t ds_row = base + C::OFF_DS + kr * 128;
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        uint32_t dp[32];
        tmem_ld32_sync(tB + h * 32, dp);
        uint32_t ds[16];
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          uint32_t d0, d1, d2, d3;
          ld_shared_v4(rows_s + 512 + (h * 32 + c) * 4, d0, d1, d2, d3);
          const uint32_t pa = pk[(h * 32 + c) / 2], pb = pk[(h * 32 + c) / 2 + 1];
          const float x0 = __uint_as_float(pa << 16) * (__uint_as_float(dp[c + 0]) - __uint_as_float(d0));
          const float x1 = __uint_as_float(pa & 0xffff0000u) * (__uint_as_float(dp[c + 1]) - __uint_as_float(d1));
          const float x2 = __uint_as_float(pb << 16) * (__uint_as_float(dp[c + 2]) - __uint_as_float(d2));
          const float x3 = __uint_as_float(pb & 0xffff0000u) * (__uint_as_float(dp[c + 3]) - __uint_as_float(d3));
          ds[c / 2] = pack_bf16x2(x0, x1);
          ds[c / 2 + 1] = pack_bf16x2(x2, x3);
        }
        // dS tile, 128-byte swizzle: atom h/2 holds queries 64(h/2) .. +63;
        // this thread's key row is one 128-byte row of it, whose 16-byte
        // units are permuted by (key row & 7).  Read K-major it is dS^T
        // (A of dK), read MN-major it is dS (A of dQ).
        const uint32_t atom = ds_row + (h >> 1) * (128 * 128);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint32_t unit = uint32_t((h & 1) * 4 + v) ^ uint32_t(kr & 7);
          st_shared_v4(atom + unit * 16, ds[4 * v], ds[4 * v + 1], ds[4 * v + 2], ds[4 * v + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_DSR));
    }
  } else {
    // ------------------------------------------------------------ WG1: dQ drain, dK / dV out
    const int wq = warp - 4;
    const int r = wq * 32 + lane;           // TMEM lane: query row of dQ, key row of dK / dV
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const uint32_t tB = tmem + lane_off + C::B_COL;
    const uint32_t stage_s = base + C::OFF_DS;   // dS tile: free once dQ_i is in TMEM
    const bool issuer = (wq == 0 && lane == 0);
    bool ok = true;
    for (int i = 0; i < nsteps; ++i) {
      const int hq = step_head(i), q0 = step_q0(i);
      // all four warps take the same decision, so none is left at a named barrier
      ok = named_bar_and(1, 128, warp_wait(bar(C::B_DQF), i & 1, abort_flag, a.status));
      if (!ok) break;
      tc_fence_after();
      // dQ_i in rounds of 64 columns: two 32-column fp32 boxes (128 rows x
      // 128 bytes, 128-byte swizzle) staged in the dS tile, then added into
      // the accumulator by the TMA unit (rows past Nq are clipped).
#pragma unroll 1
      for (int rnd = 0; rnd < D / 64; ++rnd) {
#pragma unroll
        for (int bx = 0; bx < 2; ++bx) {
          uint32_t v[32];
          tmem_ld32_sync(tB + rnd * 64 + bx * 32, v);
          const uint32_t row_s = stage_s + bx * (128 * 128) + r * 128;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint32_t unit = uint32_t(u) ^ uint32_t(r & 7);
            st_shared_v4(row_s + unit * 16, __float_as_uint(__uint_as_float(v[4 * u]) * a.scale),
                         __float_as_uint(__uint_as_float(v[4 * u + 1]) * a.scale),
                         __float_as_uint(__uint_as_float(v[4 * u + 2]) * a.scale),
                         __float_as_uint(__uint_as_float(v[4 * u + 3]) * a.scale));
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (issuer) {
#pragma unroll
          for (int bx = 0; bx < 2; ++bx)
            tma_reduce_add_4d(&tm_dq, stage_s + bx * (128 * 128), rnd * 64 + bx * 32, hq, q0, b);
          tma_store_commit();
          tma_store_wait_read();   // the staging tile may be overwritten again
        }
        named_bar_sync(1, 128);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_DQE));
    }
    if (issuer) tma_store_wait_all();   // every reduce has landed before the CTA ends
    if (ok && nsteps > 0) {
      ok = warp_wait(bar(C::B_DONE), 0, abort_flag, a.status);
      tc_fence_after();
    }
    const int kk = k0 + r;
    // Warp-uniform: the TMEM loads below are warp-collective (.sync.aligned),
    // so every lane runs them and only the stores depend on the lane's key row.
    const bool write = __all_sync(0xffffffffu, ok && !*abort_flag);
    if (write) {
      const size_t row = (((size_t)b * a.Nk + kk) * a.Hkv + hk) * D;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* out = (which == 0 ? a.dv : a.dk) + row;
        const float mul = which == 0 ? 1.f : a.scale;
        const uint32_t col = which == 0 ? C::DV_COL : C::DK_COL;
#pragma unroll 1
        for (int h = 0; h < D / 32; ++h) {
          uint32_t v[32];
          if (nsteps > 0) {
            tmem_ld32_sync(tmem + lane_off + col + h * 32, v);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0u;
          }
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]) * mul, __uint_as_float(v[2 * j + 1]) * mul);
          if (kk < a.Nk) {
            uint4* o4 = reinterpret_cast<uint4*>(out + h * 32);
#pragma unroll
            for (int j = 0; j < 4; ++j) o4[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          }
        }
      }
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Head dimension 128: 64-query steps with dQ^T accumulated in tensor memory.
//
// The 128-query kernel above keeps dQ (128 x 128 fp32) in the TMEM columns of
// dP^T, so the next step's dP^T waits until dQ has been moved out and added
// into global memory.  With 64 queries per step the products shrink to
// N = 64, and dQ^T = K^T dS^T (M = D = 128 head dims on the TMEM lanes,
// N = 64 queries) fits beside double-buffered S^T:
//
//   TMEM   dV [0,128) | dK [128,256) | S^T/P^T x2 [256,384) | dP^T [384,448) | dQ^T [448,512)
//
// and a third warpgroup drains dQ^T into two shared-memory boxes that the
// TMA unit adds into a transposed fp32 accumulator [B, Hq, D, Nq_pad] (each
// TMEM lane is one head dim, so a box row is 32 consecutive queries of one
// dim).  dQ leaves TMEM as soon as it is loaded into registers; the adds run
// while the next steps compute.  bwd_dqt_kernel transposes the accumulator
// into dQ.
//
// Roles (448 threads):
//   warps 0-3   (WG0)  P pass: S^T -> P^T = exp2(S^T * scale * log2e - LSE2), bf16, into TMEM
//   warps 4-7   (WG1)  dS pass: P^T and dP^T from TMEM -> dS = P (dP - Drow) -> shared memory
//   warps 8-11  (WG2)  dQ^T drain -> TMA reduce-add; nothing else
//   warp 12            TMA: K, V once; three (Q, dO) stages with their LSE and Drow values
//   warp 13            tcgen05.mma issue
// At the end WG0 writes dV and WG1 writes dK.
//
// Issue order per step i, tensor pipe in issue order:
//   dV_i (P^T_i) -> dP^T_{i+1} -> dK_i, dQ^T_i (dS_i) -> S^T_{i+2}
// S^T is computed two steps ahead into the other buffer, so WG0 runs P
// passes back to back; dP^T_{i+1} is issued as soon as WG1 has loaded
// dP^T_i, so WG1 runs dS passes back to back.
template <bool CAUSAL_>
struct CfgT {
  static constexpr int D = 128;
  static constexpr bool CAUSAL = CAUSAL_;
  static constexpr int BM = 64;                    // queries per step
  static constexpr int BN = 128;                   // keys per CTA = TMEM lanes
  static constexpr int STAGES = 3;
  static constexpr int KCH = 128 * 128;            // 64-column chunk of a 128-row tile
  static constexpr int QCH = 64 * 128;             // 64-column chunk of a 64-row tile
  static constexpr int KTILE = 2 * KCH;
  static constexpr int QTILE = 2 * QCH;
  static constexpr int DS_BYTES = BN * BM * 2;     // 128 key rows x 64 queries, one 128-byte row per key
  static constexpr int BOX = 128 * 128;            // dQ^T box: 128 head dims x 32 fp32 queries
  // shared memory (offsets from a 1024-byte aligned base)
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KTILE;
  static constexpr int OFF_STAGE = OFF_V + KTILE;              // stage s: Q at +2s*QTILE, dO at +(2s+1)*QTILE
  static constexpr int OFF_DS = OFF_STAGE + STAGES * 2 * QTILE;   // two dS buffers
  static constexpr int OFF_DQS = OFF_DS + 2 * DS_BYTES;        // two dQ^T boxes
  static constexpr int OFF_ROWS = OFF_DQS + 2 * BOX;           // stage s: lse2[64], drow[64] at +s*512
  static constexpr int OFF_BAR = OFF_ROWS + STAGES * 512;
  // barriers
  static constexpr int B_KV = 0;
  static constexpr int B_QF = 1;        // [3] stage full (TMA bytes + producer arrival)
  static constexpr int B_QE = 4;        // [3] stage empty (MMA commit after dK)
  static constexpr int B_SF = 7;        // [2] S^T in TMEM buffer
  static constexpr int B_PR = 9;        // [2] P^T stored (4 WG0 warps)
  static constexpr int B_DPF = 11;      // dP^T in TMEM
  static constexpr int B_DPE = 12;      // dP^T and P^T loaded by WG1 (4 warps)
  static constexpr int B_DSR = 13;      // [2] dS in shared memory (4 WG1 warps)
  static constexpr int B_DSE = 15;      // [2] dS buffer read by dK and dQ^T (MMA commit)
  static constexpr int B_DQF = 17;      // dQ^T in TMEM
  static constexpr int B_DQE = 18;      // dQ^T loaded by WG2 (4 warps)
  static constexpr int B_DONE = 19;     // every MMA of the CTA complete
  static constexpr int NBAR = 20;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int LAYOUT_BYTES = OFF_MISC + 16;
  static constexpr int MAX_SMEM = 227 * 1024;
  static constexpr int SMEM_BYTES = LAYOUT_BYTES + 1024 <= MAX_SMEM ? LAYOUT_BYTES + 1024 : MAX_SMEM;
  static_assert(LAYOUT_BYTES <= MAX_SMEM, "shared memory budget");
  // TMEM columns
  static constexpr int DV_COL = 0;
  static constexpr int DK_COL = 128;
  static constexpr int S_COL = 256;     // buffer b at S_COL + 64 b
  static constexpr int DP_COL = 384;
  static constexpr int DQ_COL = 448;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 448;
  static constexpr int PRODUCER_WARP = 12;
  static constexpr int MMA_WARP = 13;
};

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    attn_bwd_dqt_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                        const __grid_constant__ CUtensorMap tm_dqt, const Args a) {
  constexpr int QTILE = C::QTILE, QCH = C::QCH, KCH = C::KCH, BM = C::BM;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  if (base - raw + C::LAYOUT_BYTES > (uint32_t)C::SMEM_BYTES) {
    if (threadIdx.x == 0) atomicExch(a.status, ATTN_ERR_CUDA);
    return;
  }
  uint8_t* base_ptr = smem_raw + (base - raw);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::OFF_MISC + 4);
  auto bar = [&](int i) -> uint32_t { return base + C::OFF_BAR + 8u * i; };
  auto q_off = [&](int st) -> uint32_t { return base + C::OFF_STAGE + 2 * st * QTILE; };
  auto do_off = [&](int st) -> uint32_t { return base + C::OFF_STAGE + (2 * st + 1) * QTILE; };
  auto ds_off = [&](int bf) -> uint32_t { return base + C::OFF_DS + bf * C::DS_BYTES; };
  auto rows_off = [&](int st) -> uint32_t { return base + C::OFF_ROWS + st * 512; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const UnitPos up = unit_pos(blockIdx.x, a);
  const int kb = up.kb, hk = up.hk, b = up.b;
  const int k0 = kb * C::BN;
  int qb_start = 0;
  if (C::CAUSAL) qb_start = max(0, (k0 - a.causal_off) / BM);   // first query block with a visible key
  const int nq = max(0, a.n_qblk - qb_start);
  const int nsteps = a.group * nq;
  auto step_head = [&](int i) { return hk * a.group + i % a.group; };
  auto step_q0 = [&](int i) { return (qb_start + i / a.group) * BM; };

  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_KV), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar(C::B_QF + s), 1);
      mbar_init(bar(C::B_QE + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(C::B_SF + s), 1);
      mbar_init(bar(C::B_PR + s), 4);
      mbar_init(bar(C::B_DSR + s), 4);
      mbar_init(bar(C::B_DSE + s), 1);
    }
    mbar_init(bar(C::B_DPF), 1);
    mbar_init(bar(C::B_DPE), 4);
    mbar_init(bar(C::B_DQF), 1);
    mbar_init(bar(C::B_DQE), 4);
    mbar_init(bar(C::B_DONE), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == C::PRODUCER_WARP && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_dqt);
  }
  if (warp == 0) {
    tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    if (nsteps > 0 && lane == 0) {
      mbar_arrive_expect_tx(bar(C::B_KV), 2 * C::KTILE);
      for (int ch = 0; ch < 2; ++ch) {
        tma_load_4d(base + C::OFF_K + ch * KCH, &tm_k, bar(C::B_KV), ch * 64, hk, k0, b);
        tma_load_4d(base + C::OFF_V + ch * KCH, &tm_v, bar(C::B_KV), ch * 64, hk, k0, b);
      }
    }
    int issued = 0;
    for (int j = 0; j < nsteps; ++j) {
      const int st = j % C::STAGES;
      if (!warp_wait(bar(C::B_QE + st), ((j / C::STAGES) & 1) ^ 1, abort_flag, a.status)) break;
      const int hq = step_head(j), q0 = step_q0(j);
      float* lse_s = reinterpret_cast<float*>(base_ptr + C::OFF_ROWS + st * 512);
      float* dr_s = lse_s + BM;
      const size_t rbase = ((size_t)b * a.Hq + hq) * a.Nq;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int c = 2 * lane + r, row = q0 + c;
        float l2 = INFINITY, d = 0.f;   // rows past Nq: p = 2^-inf = 0
        if (row < a.Nq) {
          const float l = a.lse[rbase + row];
          l2 = (l == -INFINITY) ? INFINITY : l * kLog2e;   // a row that saw no key keeps p = 0
          d = a.drow[rbase + row];
        }
        lse_s[c] = l2;
        dr_s[c] = d;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(C::B_QF + st), 2 * QTILE);
        for (int ch = 0; ch < 2; ++ch) {
          tma_load_4d(q_off(st) + ch * QCH, &tm_q, bar(C::B_QF + st), ch * 64, hq, q0, b);
          tma_load_4d(do_off(st) + ch * QCH, &tm_do, bar(C::B_QF + st), ch * 64, hq, q0, b);
        }
      }
      __syncwarp();
      ++issued;
    }
    // Drain: every issued copy must land before shared memory is released.
    if (lane == 0) {
      for (int j = max(0, issued - C::STAGES); j < issued; ++j)
        mbar_wait_drain(bar(C::B_QF + j % C::STAGES), (j / C::STAGES) & 1);
      if (nsteps > 0) mbar_wait_drain(bar(C::B_KV), 0);
    }
    __syncwarp();
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = elect_one();
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, BM, false);        // S^T, dP^T: A, B K-major
    constexpr uint32_t idesc_g = idesc_bf16_f32(128, C::D, true);       // dV (A in TMEM), dK: B MN-major
    constexpr uint32_t idesc_q = idesc_bf16_f32_amn(128, BM, true);     // dQ^T: A, B MN-major
    bool ok = nsteps > 0 && warp_wait(bar(C::B_KV), 0, abort_flag, a.status);

    // S^T = K Q^T or dP^T = V dO^T: both K-major, 16 head dims per k-step.
    auto issue_kmajor = [&](uint32_t a_smem, uint32_t b_smem, uint32_t d_col, uint32_t bar_done) {
      const uint64_t adesc = sdesc_sw128(a_smem, 16, 1024);
      const uint64_t bdesc = sdesc_sw128(b_smem, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < C::D / 16; ++ks) {
        const uint32_t a_off = ((ks >> 2) * KCH + (ks & 3) * 32) >> 4;
        const uint32_t b_off = ((ks >> 2) * QCH + (ks & 3) * 32) >> 4;
        mma_ss(tmem + d_col, adesc + a_off, bdesc + b_off, idesc_s, ks > 0, leader);
      }
      mma_commit(bar_done, leader);
    };
    auto wait_stage = [&](int i) -> bool {
      if (!warp_wait(bar(C::B_QF + i % C::STAGES), (i / C::STAGES) & 1, abort_flag, a.status)) return false;
      tc_fence_after();
      return true;
    };

    if (ok) ok = wait_stage(0);
    if (ok) {
      issue_kmajor(base + C::OFF_K, q_off(0), C::S_COL, bar(C::B_SF));
      issue_kmajor(base + C::OFF_V, do_off(0), C::DP_COL, bar(C::B_DPF));
      __syncwarp();
    }
    if (ok && nsteps > 1) {
      ok = wait_stage(1);
      if (ok) issue_kmajor(base + C::OFF_K, q_off(1), C::S_COL + 64, bar(C::B_SF + 1));
      __syncwarp();
    }
    for (int i = 0; ok && i < nsteps; ++i) {
      const int st = i % C::STAGES, bf = i & 1;
      // dV += P^T dO: A = P^T (TMEM, bf16 packed two per column), B = dO read MN-major
      if (!warp_wait(bar(C::B_PR + bf), (i >> 1) & 1, abort_flag, a.status)) { ok = false; break; }
      tc_fence_after();
      {
        const uint64_t bdesc = sdesc_sw128(do_off(st), QCH, 1024);
#pragma unroll
        for (int ks = 0; ks < BM / 16; ++ks)
          mma_ts(tmem + C::DV_COL, tmem + C::S_COL + 64 * bf + ks * 8, bdesc + ks * 128, idesc_g,
                 (i > 0 || ks > 0) ? 1u : 0u, leader);
      }
      __syncwarp();
      // dP^T_{i+1} once WG1 holds dP^T_i (and P^T_i) in registers
      if (i + 1 < nsteps) {
        if (!warp_wait(bar(C::B_DPE), i & 1, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        issue_kmajor(base + C::OFF_V, do_off((i + 1) % C::STAGES), C::DP_COL, bar(C::B_DPF));
        __syncwarp();
      }
      if (!warp_wait(bar(C::B_DSR + bf), (i >> 1) & 1, abort_flag, a.status)) { ok = false; break; }
      tc_fence_after();
      {   // dK += dS^T Q: A = dS^T (the dS buffer read K-major), B = Q read MN-major
        const uint64_t adesc = sdesc_sw128(ds_off(bf), 16, 1024);
        const uint64_t bdesc = sdesc_sw128(q_off(st), QCH, 1024);
#pragma unroll
        for (int ks = 0; ks < BM / 16; ++ks)
          mma_ss(tmem + C::DK_COL, adesc + ks * 2, bdesc + ks * 128, idesc_g, (i > 0 || ks > 0) ? 1u : 0u, leader);
      }
      __syncwarp();
      if (i > 0) {
        if (!warp_wait(bar(C::B_DQE), (i - 1) & 1, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
      }
      {   // dQ^T = K^T dS^T: A = K read MN-major (head dims along M), B = dS read MN-major
        const uint64_t adesc = sdesc_sw128(base + C::OFF_K, KCH, 1024);
        const uint64_t bdesc = sdesc_sw128(ds_off(bf), QCH, 1024);
#pragma unroll
        for (int ks = 0; ks < C::BN / 16; ++ks)
          mma_ss(tmem + C::DQ_COL, adesc + ks * 128, bdesc + ks * 128, idesc_q, ks > 0 ? 1u : 0u, leader);
      }
      mma_commit(bar(C::B_DQF), leader);
      mma_commit(bar(C::B_QE + st), leader);
      mma_commit(bar(C::B_DSE + bf), leader);
      __syncwarp();
      // S^T_{i+2} into this step's S buffer: dV_i was issued before it and
      // WG1 has loaded P^T_i (B_DPE above).
      if (i + 2 < nsteps) {
        if (!wait_stage(i + 2)) { ok = false; break; }
        issue_kmajor(base + C::OFF_K, q_off((i + 2) % C::STAGES), C::S_COL + 64 * bf, bar(C::B_SF + bf));
        __syncwarp();
      }
    }
    // Drain: no MMA may still run when TMEM is released.
    if (nsteps > 0) {
      mma_commit(bar(C::B_DONE), leader);
      __syncwarp();
      mbar_wait_drain(bar(C::B_DONE), 0);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------------------ WG0: P pass, then dV out
    const int kr = warp * 32 + lane;      // key row in the block = TMEM lane
    const int kk = k0 + kr;
    const bool row_valid = kk < a.Nk;
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    const float sl2 = a.scale_log2;
    bool ok = true;
    for (int i = 0; i < nsteps; ++i) {
      const int st = i % C::STAGES, bf = i & 1, q0 = step_q0(i);
      if (!warp_wait(bar(C::B_QF + st), (i / C::STAGES) & 1, abort_flag, a.status)) { ok = false; break; }
      if (!warp_wait(bar(C::B_SF + bf), (i >> 1) & 1, abort_flag, a.status)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tS = tmem + lane_off + C::S_COL + 64 * bf;
      const uint32_t rows_s = rows_off(st);
      // Causal: key kk is visible to query q0 + c iff kk <= q0 + c + causal_off.
      const int cmin = row_valid ? (C::CAUSAL ? kk - a.causal_off - q0 : 0) : BM;
      uint32_t s[64];
      tmem_ld64_sync(tS, s);
      uint32_t pk[32];
      // Pairs of columns: 5 of every 16 take 2^x on the FMA pipe (the
      // polynomial of sm100.cuh), the rest on the MUFU unit, whose throughput
      // otherwise sets this pass.  A column whose row saw no key (LSE2 = +inf)
      // gives exactly 0 either way.
      const uint64_t k2 = f2_pack(sl2, sl2);
      auto exp2_pair = [&](int c, uint64_t x, uint32_t la, uint32_t lb, float& pa, float& pb) {
        if (poly_pair(c)) {
          exp2_poly_x2(x, pa, pb);
          if (__uint_as_float(la) == INFINITY) pa = 0.f;
          if (__uint_as_float(lb) == INFINITY) pb = 0.f;
        } else {
          float xa, xb;
          f2_unpack(x, xa, xb);
          pa = ex2(xa);
          pb = ex2(xb);
        }
      };
#pragma unroll
      for (int j = 0; j < 64; j += 4) {
        uint32_t l0, l1, l2, l3;
        ld_shared_v4(rows_s + j * 4, l0, l1, l2, l3);
        const uint64_t x01 = f2_fma(f2_pack(__uint_as_float(s[j + 0]), __uint_as_float(s[j + 1])), k2,
                                    f2_pack(-__uint_as_float(l0), -__uint_as_float(l1)));
        const uint64_t x23 = f2_fma(f2_pack(__uint_as_float(s[j + 2]), __uint_as_float(s[j + 3])), k2,
                                    f2_pack(-__uint_as_float(l2), -__uint_as_float(l3)));
        float p0, p1, p2, p3;
        exp2_pair(j / 2, x01, l0, l1, p0, p1);
        exp2_pair(j / 2 + 1, x23, l2, l3, p2, p3);
        pk[j / 2] = pack_bf16x2(p0, p1);
        pk[j / 2 + 1] = pack_bf16x2(p2, p3);
      }
      if (cmin > 0) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const uint32_t keep = (2 * j + 1 < cmin) ? 0u : (2 * j < cmin ? 0xffff0000u : 0xffffffffu);
          pk[j] &= keep;
        }
      }
      tmem_st32(tS, pk);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_PR + bf));
    }
    if (ok && nsteps > 0) {
      ok = warp_wait(bar(C::B_DONE), 0, abort_flag, a.status);
      tc_fence_after();
    }
    const bool write = __all_sync(0xffffffffu, ok && !*abort_flag);
    if (write) {
      __nv_bfloat16* out = a.dv + (((size_t)b * a.Nk + kk) * a.Hkv + hk) * C::D;
#pragma unroll 1
      for (int h = 0; h < C::D / 32; ++h) {
        uint32_t v[32];
        if (nsteps > 0) {
          tmem_ld32_sync(tmem + lane_off + C::DV_COL + h * 32, v);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0u;
        }
        uint32_t o[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) o[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
        if (row_valid) {
          uint4* o4 = reinterpret_cast<uint4*>(out + h * 32);
#pragma unroll
          for (int j = 0; j < 4; ++j) o4[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
        }
      }
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ WG1: dS pass, then dK out
    const int wq = warp - 4;
    const int kr = wq * 32 + lane;
    const int kk = k0 + kr;
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    bool ok = true;
    for (int i = 0; i < nsteps; ++i) {
      const int st = i % C::STAGES, bf = i & 1;
      if (!warp_wait(bar(C::B_QF + st), (i / C::STAGES) & 1, abort_flag, a.status)) { ok = false; break; }
      if (!warp_wait(bar(C::B_PR + bf), (i >> 1) & 1, abort_flag, a.status)) { ok = false; break; }
      if (!warp_wait(bar(C::B_DPF), i & 1, abort_flag, a.status)) { ok = false; break; }
      tc_fence_after();
      uint32_t pk[32], dp[64];
      tmem_ld32_sync(tmem + lane_off + C::S_COL + 64 * bf, pk);
      tmem_ld64_sync(tmem + lane_off + C::DP_COL, dp);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_DPE));
      const uint32_t rows_s = rows_off(st) + BM * 4;
      uint32_t ds[32];
#pragma unroll
      for (int c = 0; c < 64; c += 4) {
        uint32_t d0, d1, d2, d3;
        ld_shared_v4(rows_s + c * 4, d0, d1, d2, d3);
        const uint32_t pa = pk[c / 2], pb = pk[c / 2 + 1];
        const float x0 = __uint_as_float(pa << 16) * (__uint_as_float(dp[c + 0]) - __uint_as_float(d0));
        const float x1 = __uint_as_float(pa & 0xffff0000u) * (__uint_as_float(dp[c + 1]) - __uint_as_float(d1));
        const float x2 = __uint_as_float(pb << 16) * (__uint_as_float(dp[c + 2]) - __uint_as_float(d2));
        const float x3 = __uint_as_float(pb & 0xffff0000u) * (__uint_as_float(dp[c + 3]) - __uint_as_float(d3));
        ds[c / 2] = pack_bf16x2(x0, x1);
        ds[c / 2 + 1] = pack_bf16x2(x2, x3);
      }
      // The buffer's previous tile (step i - 2) must have been read by dK and dQ^T.
      if (!warp_wait(bar(C::B_DSE + bf), ((i >> 1) & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
      // One 128-byte swizzled row per key: 16-byte unit v lands at v ^ (key row & 7).
      const uint32_t row = ds_off(bf) + kr * 128;
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const uint32_t unit = uint32_t(v) ^ uint32_t(kr & 7);
        st_shared_v4(row + unit * 16, ds[4 * v], ds[4 * v + 1], ds[4 * v + 2], ds[4 * v + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_DSR + bf));
    }
    if (ok && nsteps > 0) {
      ok = warp_wait(bar(C::B_DONE), 0, abort_flag, a.status);
      tc_fence_after();
    }
    const bool write = __all_sync(0xffffffffu, ok && !*abort_flag);
    if (write) {
      __nv_bfloat16* out = a.dk + (((size_t)b * a.Nk + kk) * a.Hkv + hk) * C::D;
#pragma unroll 1
      for (int h = 0; h < C::D / 32; ++h) {
        uint32_t v[32];
        if (nsteps > 0) {
          tmem_ld32_sync(tmem + lane_off + C::DK_COL + h * 32, v);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0u;
        }
        uint32_t o[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          o[j] = pack_bf16x2(__uint_as_float(v[2 * j]) * a.scale, __uint_as_float(v[2 * j + 1]) * a.scale);
        if (kk < a.Nk) {
          uint4* o4 = reinterpret_cast<uint4*>(out + h * 32);
#pragma unroll
          for (int j = 0; j < 4; ++j) o4[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ WG2: dQ^T drain
    const int wq = warp - 8;
    const int d = wq * 32 + lane;            // TMEM lane = head dim of dQ^T
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const bool issuer = (wq == 0 && lane == 0);
    for (int i = 0; i < nsteps; ++i) {
      const int hq = step_head(i), q0 = step_q0(i);
      // all four warps take the same decision, so none is left at a named barrier
      if (!named_bar_and(1, 128, warp_wait(bar(C::B_DQF), i & 1, abort_flag, a.status))) break;
      tc_fence_after();
      uint32_t v[64];
      tmem_ld64_sync(tmem + lane_off + C::DQ_COL, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_DQE));
#pragma unroll
      for (int bx = 0; bx < 2; ++bx) {
        // The box's previous add (one step back) must have read its source.
        if (issuer) tma_store_wait_read_n<1>();
        named_bar_sync(1, 128);
        const uint32_t row_s = base + C::OFF_DQS + bx * C::BOX + d * 128;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          const uint32_t unit = uint32_t(w) ^ uint32_t(d & 7);
          st_shared_v4(row_s + unit * 16, __float_as_uint(__uint_as_float(v[bx * 32 + 4 * w]) * a.scale),
                       __float_as_uint(__uint_as_float(v[bx * 32 + 4 * w + 1]) * a.scale),
                       __float_as_uint(__uint_as_float(v[bx * 32 + 4 * w + 2]) * a.scale),
                       __float_as_uint(__uint_as_float(v[bx * 32 + 4 * w + 3]) * a.scale));
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (issuer) {
          // A box that starts past the last query adds nothing: skip it.
          if (q0 + bx * 32 < a.Nq) tma_reduce_add_4d(&tm_dqt, base + C::OFF_DQS + bx * C::BOX, q0 + bx * 32, 0, hq, b);
          tma_store_commit();
        }
      }
    }
    if (issuer) tma_store_wait_all();   // every add has landed before the CTA ends
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Drow[b, h, i] = sum_d dO[b, i, h, d] * O[b, i, h, d] in fp32, one warp per
// (b, i, h) row; the grid also zeroes the fp32 dQ accumulator (n4 float4s,
// whatever its layout).
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ dout,
                                                       float* __restrict__ drow, float4* __restrict__ dq_acc,
                                                       long long n4, int Nq, int Hq, long long rows) {
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < n4; t += (long long)gridDim.x * blockDim.x)
    dq_acc[t] = make_float4(0.f, 0.f, 0.f, 0.f);
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  constexpr int PER = D / 32;   // 2 or 4 elements per lane
  const __nv_bfloat16* op = o + row * D + lane * PER;
  const __nv_bfloat16* dp = dout + row * D + lane * PER;
  float acc = 0.f;
  if constexpr (PER == 4) {
    const uint2 ov = *reinterpret_cast<const uint2*>(op);
    const uint2 dv = *reinterpret_cast<const uint2*>(dp);
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float2 of = __bfloat1622float2(o2[j]), df = __bfloat1622float2(d2[j]);
      acc = fmaf(of.x, df.x, acc);
      acc = fmaf(of.y, df.y, acc);
    }
  } else {
    const float2 of = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(op));
    const float2 df = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(dp));
    acc = fmaf(of.x, df.x, of.y * df.y);
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
  // row = (b * Nq + i) * Hq + h
  const long long h = row % Hq, bi = row / Hq, i = bi % Nq, bb = bi / Nq;
  if (lane == 0) drow[(bb * Hq + h) * Nq + i] = acc;
}

// dQ (bf16) from the fp32 accumulator, 8 elements per thread and step.
__global__ void __launch_bounds__(256) bwd_dq_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq,
                                                     long long n8) {
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < n8; t += (long long)gridDim.x * blockDim.x) {
    const float4 a0 = reinterpret_cast<const float4*>(acc)[2 * t];
    const float4 a1 = reinterpret_cast<const float4*>(acc)[2 * t + 1];
    reinterpret_cast<uint4*>(dq)[t] = make_uint4(pack_bf16x2(a0.x, a0.y), pack_bf16x2(a0.z, a0.w),
                                                 pack_bf16x2(a1.x, a1.y), pack_bf16x2(a1.z, a1.w));
  }
}

// dQ (bf16, [B, Nq, Hq, 128]) from the transposed fp32 accumulator
// [B, Hq, 128, nq_pad] of attn_bwd_dqt_kernel: one tile of 32 queries x 128
// head dims per iteration, read as 128 rows of 128 bytes and written as 32
// rows of 256 bytes through a padded shared-memory tile.
__global__ void __launch_bounds__(256) bwd_dqt_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq,
                                                      int Nq, int Hq, long long nq_pad, int n_qt, long long tiles) {
  __shared__ float t[128][33];
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  for (long long tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
    const int q0 = (int)(tile % n_qt) * 32;
    const long long bh = tile / n_qt;   // b * Hq + h
    const float* src = acc + bh * 128 * nq_pad + q0;
    for (int d = w; d < 128; d += 8) t[d][l] = src[d * nq_pad + l];   // q0 + l < nq_pad
    __syncthreads();
    if (q0 + l < Nq) {
      const long long h = bh % Hq, bb = bh / Hq;
      uint32_t pk[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) pk[j] = pack_bf16x2(t[w * 16 + 2 * j][l], t[w * 16 + 2 * j + 1][l]);
      uint4* o = reinterpret_cast<uint4*>(dq + ((bb * Nq + q0 + l) * Hq + h) * 128 + w * 16);
      o[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      o[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
    __syncthreads();
  }
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// ---------------------------------------------------------------- unit order
//
// The grid has one CTA per unit and one CTA fits an SM, so the block
// scheduler hands the units out in index order, each to the SM that frees
// first.  Key block slowest over all heads puts the heaviest causal units
// first (the best balance), but then the resident CTAs cover every head and
// each later wave streams the Q, dO and dQ accumulator rows of every head
// from DRAM again.  Grouping ceil(SMs / key blocks) heads keeps a wave on
// fewer heads' rows, at the risk that a late group's heaviest units end
// after everything else.  The host simulates that hand-out for both orders
// (a unit costs its query steps plus a fixed kUnitFixedSteps) and groups
// only when it costs at most 1 % more; the choice is cached per shape.
constexpr int kUnitFixedSteps = 4;
constexpr long long kMaxSimulatedUnits = 1 << 16;

long long unit_makespan(int P, int nkb, int g, const std::vector<long long>& cost, int sms) {
  std::priority_queue<long long, std::vector<long long>, std::greater<long long>> free_at;
  for (int i = 0; i < sms; ++i) free_at.push(0);
  long long end = 0;
  for (int p0 = 0; p0 < P; p0 += g) {
    const int gs = std::min(g, P - p0);
    for (int kb = 0; kb < nkb; ++kb)
      for (int j = 0; j < gs; ++j) {
        const long long t = free_at.top() + cost[kb];
        free_at.pop();
        free_at.push(t);
        end = std::max(end, t);
      }
  }
  return end;
}

int choose_head_group(int P, int nkb, int n_qblk, int group, bool causal, int causal_off, int bm, int sms) {
  if (P < 1 || nkb < 1 || sms < 1) return std::max(P, 1);
  const int g = std::min(P, (sms + nkb - 1) / nkb);
  if (g >= P || (long long)P * nkb > kMaxSimulatedUnits) return P;
  struct Entry {
    int key[8];
    int g;
  };
  static std::mutex mu;
  static Entry cache[16];
  static int n_cached = 0, next_slot = 0;
  const int key[8] = {P, nkb, n_qblk, group, (int)causal, causal ? causal_off : 0, bm, sms};
  {
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < n_cached; ++i)
      if (std::equal(key, key + 8, cache[i].key)) return cache[i].g;
  }
  std::vector<long long> cost(nkb);
  for (int kb = 0; kb < nkb; ++kb) {
    // the kernels' own count: query blocks from the first one with a visible key
    const int qb_start = causal ? std::max(0, (kb * 128 - causal_off) / bm) : 0;
    cost[kb] = (long long)group * std::max(0, n_qblk - qb_start) + kUnitFixedSteps;
  }
  const long long all_heads = unit_makespan(P, nkb, P, cost, sms);
  const long long grouped = unit_makespan(P, nkb, g, cost, sms);
  const int chosen = grouped * 100 <= all_heads * 101 ? g : P;
  std::lock_guard<std::mutex> lk(mu);
  Entry& e = cache[next_slot];
  std::copy(key, key + 8, e.key);
  e.g = chosen;
  next_slot = (next_slot + 1) % 16;
  n_cached = std::min(n_cached + 1, 16);
  return chosen;
}

// Row length of the transposed dQ accumulator: a multiple of 32 queries, so
// that its rows are 128-byte aligned for the TMA reduce-add.
inline uint64_t dqt_row(int Nq) { return ((uint64_t)Nq + 31) & ~uint64_t(31); }

inline size_t acc_bytes(int B, int Hq, int Nq, int D) {
  if (D == 128) return (size_t)B * Hq * D * dqt_row(Nq) * 4;
  return (size_t)B * Nq * Hq * D * 4;
}

size_t workspace_bytes(int B, int Hq, int Nq, int D) {
  const size_t n = (size_t)B * Nq * Hq;
  return align256(acc_bytes(B, Hq, Nq, D)) + align256(n * 4);
}

template <int D, bool CAUSAL>
int launch(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse, void* dq,
           void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nk, float scale, void* workspace,
           cudaStream_t stream) {
  // D = 128 runs the 64-query kernel with a transposed dQ accumulator; D = 64
  // the 128-query kernel with dQ rows in the output layout.
  constexpr bool kDqt = D == 128;
  constexpr int kBM = kDqt ? CfgT<CAUSAL>::BM : Cfg<D, CAUSAL>::BM;
  int* status = device_status_ptr();
  if (!status) return ATTN_ERR_CUDA;
  float* dq_acc = static_cast<float*>(workspace);
  const size_t acc_sz = acc_bytes(B, Hq, Nq, D);
  float* drow = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + align256(acc_sz));
  const long long rows = (long long)B * Nq * Hq;
  const int sms = current_sm_count();
  if (rows > 0) {
    bwd_prep_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), drow,
        reinterpret_cast<float4*>(dq_acc), (long long)(acc_sz / 16), Nq, Hq, rows);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  if (Nk > 0) {
    CUtensorMap tq, tk, tv, tdo, tdq;
    const uint64_t es = 2;
    const uint32_t kbox[4] = {64, 1, 128, 1};
    const uint32_t qbox[4] = {64, 1, (uint32_t)kBM, 1};
    {
      // With Nq == 0 no query block is ever loaded: describe a 1-row tensor at k.
      const uint64_t nq = Nq > 0 ? (uint64_t)Nq : 1;
      const void* qb = Nq > 0 ? q : k;
      const void* db = Nq > 0 ? dout : k;
      const uint64_t hq = Nq > 0 ? (uint64_t)Hq : (uint64_t)Hkv;
      const uint64_t dims[4] = {(uint64_t)D, hq, nq, Nq > 0 ? (uint64_t)B : 1};
      const uint64_t strides[3] = {D * es, hq * D * es, nq * hq * D * es};
      if (!encode_bf16_4d(&tq, qb, dims, strides, qbox)) return ATTN_ERR_CUDA;
      if (!encode_bf16_4d(&tdo, db, dims, strides, qbox)) return ATTN_ERR_CUDA;
    }
    {
      const uint64_t dims[4] = {(uint64_t)D, (uint64_t)Hkv, (uint64_t)Nk, (uint64_t)B};
      const uint64_t strides[3] = {D * es, (uint64_t)Hkv * D * es, (uint64_t)Nk * Hkv * D * es};
      if (!encode_bf16_4d(&tk, k, dims, strides, kbox)) return ATTN_ERR_CUDA;
      if (!encode_bf16_4d(&tv, v, dims, strides, kbox)) return ATTN_ERR_CUDA;
    }
    if constexpr (kDqt) {
      // transposed fp32 accumulator [B, Hq, 128, row] (row = Nq rounded up to
      // 32), boxes of 32 queries x 128 head dims; queries past Nq are clipped.
      // With Nq == 0 nothing is ever added: describe one box at k.
      const uint64_t row = Nq > 0 ? dqt_row(Nq) : 32;
      const void* base_dq = Nq > 0 ? static_cast<const void*>(dq_acc) : k;
      const uint64_t dims[4] = {Nq > 0 ? (uint64_t)Nq : 32, 128, Nq > 0 ? (uint64_t)Hq : 1, Nq > 0 ? (uint64_t)B : 1};
      const uint64_t strides[3] = {row * 4, 128 * row * 4, dims[2] * 128 * row * 4};
      const uint32_t box[4] = {32, 128, 1, 1};
      if (!encode_f32_4d(&tdq, base_dq, dims, strides, box)) return ATTN_ERR_CUDA;
    } else {
      // fp32 dQ accumulator [B, Nq, Hq, D], 32-column boxes (128 bytes);
      // with Nq == 0 nothing is ever added: describe one row at k.
      const uint64_t nq = Nq > 0 ? (uint64_t)Nq : 1;
      const void* base_dq = Nq > 0 ? static_cast<const void*>(dq_acc) : k;
      const uint64_t hq = Nq > 0 ? (uint64_t)Hq : 1;
      const uint64_t dq_dims[4] = {Nq > 0 ? (uint64_t)D : 32, hq, nq, Nq > 0 ? (uint64_t)B : 1};
      const uint64_t dq_strides[3] = {dq_dims[0] * 4, hq * dq_dims[0] * 4, nq * hq * dq_dims[0] * 4};
      const uint32_t dq_box[4] = {32, 1, 128, 1};
      if (!encode_f32_4d(&tdq, base_dq, dq_dims, dq_strides, dq_box)) return ATTN_ERR_CUDA;
    }
    Args a;
    a.lse = lse;
    a.drow = drow;
    a.dk = static_cast<__nv_bfloat16*>(dk);
    a.dv = static_cast<__nv_bfloat16*>(dv);
    a.status = status;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.Nq = Nq;
    a.Nk = Nk;
    a.group = Hq / Hkv;
    a.n_qblk = (Nq + kBM - 1) / kBM;
    a.n_kblk = (Nk + 127) / 128;
    a.causal_off = Nk - Nq;
    a.scale = scale;
    a.scale_log2 = scale * kLog2e;
    const long long units = (long long)a.n_kblk * Hkv * B;
    if (units > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    a.head_group = choose_head_group(Hkv * B, a.n_kblk, a.n_qblk, a.group, CAUSAL, a.causal_off, kBM, sms);
    if constexpr (kDqt) {
      using C = CfgT<CAUSAL>;
      static int attr_done = 0;
      const void* kfn = reinterpret_cast<const void*>(&attn_bwd_dqt_kernel<C>);
      if (int rc = ensure_smem_attr(kfn, C::SMEM_BYTES, &attr_done)) return rc;
      attn_bwd_dqt_kernel<C><<<(unsigned)units, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, tdq, a);
    } else {
      using C = Cfg<D, CAUSAL>;
      static int attr_done = 0;
      const void* kfn = reinterpret_cast<const void*>(&attn_bwd_kernel<C>);
      if (int rc = ensure_smem_attr(kfn, C::SMEM_BYTES, &attr_done)) return rc;
      attn_bwd_kernel<C><<<(unsigned)units, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, tdq, a);
    }
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  if (rows > 0) {
    if constexpr (kDqt) {
      const int n_qt = (Nq + 31) / 32;
      const long long tiles = (long long)n_qt * Hq * B;
      const unsigned grid = (unsigned)(tiles < (long long)sms * 16 ? tiles : (long long)sms * 16);
      bwd_dqt_kernel<<<grid, 256, 0, stream>>>(dq_acc, static_cast<__nv_bfloat16*>(dq), Nq, Hq,
                                               (long long)dqt_row(Nq), n_qt, tiles);
    } else {
      const long long n8 = rows * D / 8;
      const long long want = (n8 + 255) / 256;
      const unsigned grid = (unsigned)(want < (long long)sms * 8 ? want : (long long)sms * 8);
      bwd_dq_kernel<<<grid, 256, 0, stream>>>(dq_acc, static_cast<__nv_bfloat16*>(dq), n8);
    }
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

}  // namespace bwd
}  // namespace ea

extern "C" size_t attn_bwd_workspace_size(int B, int Hq, int Nq, int D) {
  if (B < 1 || Hq < 1 || Nq < 0 || (D != 64 && D != 128)) return 0;
  return ea::bwd::workspace_bytes(B, Hq, Nq, D);
}

extern "C" int attn_bwd_head_group(int B, int Hq, int Hkv, int Nq, int Nk, int D, int causal, int sm_count) {
  using namespace ea::bwd;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 0 || Nk < 1 || Hq % Hkv != 0 || sm_count < 1) return 0;
  if (D != 64 && D != 128) return 0;
  if ((long long)B * Hkv > 0x7fffffffLL) return 0;
  // the query block of the kernel that attn_bwd runs for D
  const int bm = D == 128 ? CfgT<true>::BM : Cfg<64, true>::BM;
  return choose_head_group(B * Hkv, (Nk + 127) / 128, (Nq + bm - 1) / bm, Hq / Hkv, causal != 0, Nk - Nq, bm,
                           sm_count);
}

extern "C" int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                        const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nk,
                        int D, int Dv, int causal, float scale, void* workspace, size_t workspace_bytes,
                        void* stream) {
  using namespace ea;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 0 || Nk < 0 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (Nq > 0 && (!q || !o || !dout || !lse || !dq)) return ATTN_ERR_INVALID_ARG;
  if (Nk > 0 && (!k || !v || !dk || !dv)) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4))
    return ATTN_ERR_INVALID_ARG;
  if (D != Dv) return ATTN_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if ((uint64_t)bwd::acc_bytes(B, Hq, Nq, D) >= (1ull << 40) || (uint64_t)B * Nk * Hkv * D * 2 >= (1ull << 40))
    return ATTN_ERR_UNSUPPORTED;
  if (Nq == 0 && Nk == 0) return ATTN_OK;
  const size_t need = bwd::workspace_bytes(B, Hq, Nq, D);
  if (Nq > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 256))) return ATTN_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool c = causal != 0;
  if (D == 64)
    return c ? bwd::launch<64, true>(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, scale, workspace, s)
             : bwd::launch<64, false>(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, scale, workspace, s);
  return c ? bwd::launch<128, true>(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, scale, workspace, s)
           : bwd::launch<128, false>(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, scale, workspace, s);
}
