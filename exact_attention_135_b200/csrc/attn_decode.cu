// Paged MLA decode, "MQA-absorb" form, for sm_100a (B200).
//
// What it computes: for each sequence b, one absorbed query token with Hq=128
// heads attends to the L_b cached latent rows of that sequence (pages of 64
// tokens reached through the block table; "FlashMLA" page: BF16, paged KV
// with 64-token pages, variable lengths).  Every head reads the same latent
// row ("GQLA" page, MQA-absorb path): K = the whole 576-wide row, V = its
// first 512 entries.  O = softmax(scale * q K^T) V and LSE per (b, head).
//
// Work split (split-KV): the pages of all sequences are laid end to end and
// cut into one contiguous, page-aligned range per CTA pair, so every pair
// reads the same number of pages whatever the length mix.  A range covers
// the tail of one sequence, whole sequences, and the head of another.  A
// sequence read entirely by one pair is written out directly; the pieces of
// a sequence shared by several pairs are written as fp32 partial results
// (O normalised by its own sum, plus its LSE) and merged by the LSE-combine
// kernel:  lse = ln sum_i exp(lse_i),  O = sum_i exp(lse_i - lse) O_i
// (the identity behind the running max / running sum of the online softmax,
// "FlashAttention (KO)", online softmax section).
//
// The accumulator of 128 heads x 512 fp32 fills all 512 TMEM columns of an
// SM, so the two CTAs of a pair split the 512 output columns: CTA r owns
// columns [256 r, 256 r + 256).  Each CTA computes the full 128 x 64 score
// tile per page itself.  TMEM columns per CTA:
//   [0,256) O half | [256,320) S buffer 0 | [320,384) S buffer 1 | [384,512) Q dims 320..575
// Score tiles alternate between the two S buffers, so the tile of page g+1
// is computed while the softmax still reads that of page g; P (bf16) is
// written over the first 32 columns of its own S buffer.  Q dims 0..319 sit
// in shared memory (80 KB).
//
// A page's latent rows reach shared memory in two parts with rings of their
// own, each filled by its own producer warp:
//   own part   the 4 column chunks (256 dims) of this CTA's output columns:
//              read by the score MMAs and then by the P V products;
//   rest part  the other CTA's 256 dims and the 64 RoPE dims (5 chunks): read
//              by the score MMAs only.
// The score MMAs take the rest chunks first and release them with a commit,
// then the own chunks; so a rest slot is free ~800 cycles before the score
// tile is complete, and an own part has to land only when the score MMAs reach
// it.  A whole-page stage would be held from its load until the P V product.
#include <math.h>

#include <mutex>
#include <type_traits>

#include "host_common.h"
#include "sm100.cuh"
#include "softmax_row.cuh"

namespace ea {

namespace dec {

constexpr int HQ = 128;
constexpr int DK = 576;
constexpr int DV = 512;
constexpr int PAGE = 64;
constexpr int B_MAX = 2048;
constexpr int CHUNKS = DK / 64;                 // 9 column chunks of 128 bytes
constexpr int Q_SMEM_CHUNKS = 5;                // dims 0..319 in shared memory
constexpr int Q_TMEM_DIMS = DK - 64 * Q_SMEM_CHUNKS;   // 256 dims in TMEM
constexpr int Q_CHUNK_BYTES = HQ * 128;         // 16 KB
constexpr int PAGE_CHUNK_BYTES = PAGE * 128;    // 8 KB
constexpr int Q_BYTES = Q_SMEM_CHUNKS * Q_CHUNK_BYTES;
constexpr int OWN_CHUNKS = 4;                   // this CTA's 256 output dims
constexpr int REST_CHUNKS = CHUNKS - OWN_CHUNKS;   // the other CTA's 256 dims + 64 RoPE dims
constexpr int OWN_BYTES = OWN_CHUNKS * PAGE_CHUNK_BYTES;     // 32 KB
constexpr int REST_BYTES = REST_CHUNKS * PAGE_CHUNK_BYTES;   // 40 KB
static_assert(OWN_BYTES + REST_BYTES == PAGE * DK * 2, "the two parts hold exactly one page of the pool");
// The rest part has one slot, released chunk by chunk: chunk j of page g+1 is
// asked for as soon as the score MMAs of page g have read chunk j of page g
// (a commit per chunk), so each 8 KB chunk has about one page period to land.
// Own parts are held until the P V product and get three stages.
constexpr int OWN_STAGES = 3;
constexpr int REST_STAGES = 1;
constexpr int O_COL = 0;
constexpr int S_COL = 256;                      // two buffers of PAGE columns
constexpr int Q_COL = 384;
constexpr int TMEM_COLS = 512;
constexpr int THREADS = 256;                    // 4 softmax warps, 2 producers, 2 MMA issuers
constexpr int REST_PRODUCER_WARP = 4;           // Q and the rest parts (and the L2 prefetches)
constexpr int MMA_S_WARP = 5;                   // score tiles S = Q K^T
constexpr int MMA_PV_WARP = 6;                  // products O += P V
constexpr int OWN_PRODUCER_WARP = 7;            // the own parts
// barriers
constexpr int B_QF = 0, B_QE = 1, B_QT = 2;
constexpr int B_RF = 3;                          // rest part landed (one arrival per chunk)
constexpr int B_RE = B_RF + 1;                   // rest chunk j read, one barrier per chunk
constexpr int B_OF = B_RE + REST_CHUNKS, B_OE = B_OF + OWN_STAGES;
constexpr int B_SF = B_OE + OWN_STAGES;         // score tile complete, one per S buffer
constexpr int B_SB = B_SF + 2;                   // P V product done, one per S buffer (its P is read)
constexpr int B_PF = B_SB + 2, B_OD = B_PF + 1, B_DR = B_OD + 1, B_DRS = B_DR + 1;
constexpr int NBAR = B_DRS + 1;
// shared memory
constexpr int OFF_Q = 0;
constexpr int OFF_OWN = OFF_Q + Q_BYTES;
constexpr int OFF_REST = OFF_OWN + OWN_STAGES * OWN_BYTES;
constexpr int OFF_BAR = OFF_REST + REST_STAGES * REST_BYTES;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int OFF_PREF = OFF_MISC + 16;
constexpr int SMEM_BYTES = OFF_PREF + (B_MAX + 1) * 4 + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert(OFF_OWN % 1024 == 0 && OFF_REST % 1024 == 0 && REST_BYTES % 1024 == 0, "swizzle atoms");
static_assert(REST_STAGES == 1, "the rest slot is released chunk by chunk");

// Dim chunk (64 dims) held by chunk j of the own / rest part of CTA `half`.
__device__ __forceinline__ int own_chunk_dim(int half, int j) { return OWN_CHUNKS * half + j; }
__device__ __forceinline__ int rest_chunk_dim(int half, int j) {
  return j < OWN_CHUNKS ? OWN_CHUNKS * (1 - half) + j : CHUNKS - 1;
}

// Pages the producer asks L2 for ahead of the page it loads: a page's TMA
// load is issued only when a stage frees up, and from HBM it takes ~2000
// cycles to land; prefetched, it comes from L2.  148 SMs x 2 pages x 72 KB
// (each page asked for by both CTAs of a pair) stays far below L2's 126 MB.
constexpr int PREFETCH_PAGES = 2;

constexpr float kRescaleThreshold = 8.0f;
constexpr float kLn2 = 0.6931471805599453f;

// The kernels work on query units: with s_q query tokens per sequence, unit
// u = b * s_q + i is query token i of sequence b.  The s_q tokens are the last
// s_q cached tokens, so unit u sees positions 0 .. L_b - s_q + i (the causal
// mask aligned to the bottom-right corner) of block-table row b.
struct Args {
  const __nv_bfloat16* q;        // [B * s_q, Hq, DK]
  const uint8_t* kv;             // [num_pages, PAGE, DK] (only for L2 prefetches)
  const int32_t* block_table;    // [B, max_pages]
  const int32_t* seqlens;        // [B]
  __nv_bfloat16* o;              // [B * s_q, Hq, DV]
  float* lse;                    // [B * s_q, Hq]
  int32_t* ws_pref;              // [units + 1]
  float* ws_lse;                 // [2 * pairs, Hq]
  float* ws_o;                   // [2 * pairs, Hq, DV]
  int* status;
  int B;                         // query units (sequences x s_q)
  int s_q, max_pages, num_pages, pairs;
  float scale_log2;
};

// Pages a sequence contributes (its length clamped to the block table).
__device__ __forceinline__ int seq_pages(int L, int max_pages) {
  if (L <= 0) return 0;
  const int n = (L + PAGE - 1) / PAGE;
  return n < max_pages ? n : max_pages;
}

__device__ __forceinline__ int seq_len_eff(int L, int max_pages) {
  if (L <= 0) return 0;
  const int cap = max_pages * PAGE;
  return L < cap ? L : cap;
}

// Positions unit u attends to: its sequence's length clamped to the block
// table, minus the query tokens after it.
__device__ __forceinline__ int unit_len(const Args& a, int u) {
  const int L = seq_len_eff(a.seqlens[u / a.s_q], a.max_pages) - (a.s_q - 1 - u % a.s_q);
  return L > 0 ? L : 0;
}

// First page of pair p's range: floor(p * T / pairs).
__device__ __forceinline__ int range_start(int p, int T, int pairs) {
  return (int)(((long long)p * T) / pairs);
}

// Pair whose range holds global page g (0 <= g < T).
__device__ __forceinline__ int pair_of_page(int g, int T, int pairs) {
  return (int)((((long long)g + 1) * pairs - 1) / T);
}

// Walks the segments (b, first global page, end global page) of [R0, R1).
struct SegWalk {
  const int* pref;
  int B, R0, R1, b;
  __device__ void init(const int* pref_, int B_, int R0_, int R1_) {
    pref = pref_;
    B = B_;
    R0 = R0_;
    R1 = R1_;
    // last b with pref[b] <= R0 (binary search over the prefix sums)
    int lo = 0, hi = B;   // invariant: pref[lo] <= R0, answer in [lo, hi)
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pref[mid] <= R0) lo = mid; else hi = mid;
    }
    b = lo;
  }
  // Next non-empty segment; false when the range is exhausted.
  __device__ bool next(int& sb, int& g0, int& g1) {
    while (b < B && pref[b] < R1) {
      const int s = max(R0, pref[b]), e = min(R1, pref[b + 1]);
      const int cur = b++;
      if (e > s) {
        sb = cur;
        g0 = s;
        g1 = e;
        return true;
      }
    }
    return false;
  }
};

__global__ void __launch_bounds__(THREADS, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                        const Args a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + OFF_MISC + 4);
  int* pref = reinterpret_cast<int*>(base_ptr + OFF_PREF);
  auto bar = [&](int i) -> uint32_t { return base + OFF_BAR + 8u * i; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x >> 1;
  const int half = blockIdx.x & 1;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QF), 1);
    mbar_init(bar(B_QE), 1);
    mbar_init(bar(B_QT), 4);
    mbar_init(bar(B_RF), REST_CHUNKS);
    for (int j = 0; j < REST_CHUNKS; ++j) mbar_init(bar(B_RE + j), 1);
    for (int s = 0; s < OWN_STAGES; ++s) {
      mbar_init(bar(B_OF + s), 1);
      mbar_init(bar(B_OE + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_SF + i), 1);
      mbar_init(bar(B_SB + i), 1);
    }
    mbar_init(bar(B_PF), 4);
    mbar_init(bar(B_OD), 1);
    mbar_init(bar(B_DR), 1);
    mbar_init(bar(B_DRS), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // prefix sums of pages per sequence (one pass by warp 0; B <= B_MAX)
  if (warp == 0) {
    int carry = 0;
    bool bad = false;
    for (int b0 = 0; b0 < a.B; b0 += 32) {
      const int b = b0 + lane;
      int n = 0;
      if (b < a.B) {
        const int L = a.seqlens[b / a.s_q];
        n = seq_pages(unit_len(a, b), a.max_pages);
        bad |= (L < 0) || ((long long)L > (long long)a.max_pages * PAGE);
      }
      int x = n;   // inclusive warp scan
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (b < a.B) pref[b + 1] = carry + x;
      carry += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) pref[0] = 0;
    if (__any_sync(0xffffffffu, bad) && lane == 0 && blockIdx.x == 0) atomicExch(a.status, (int)ATTN_ERR_INVALID_ARG);
  }
  if (warp == REST_PRODUCER_WARP && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_kv);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int T = pref[a.B];
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i <= a.B; i += THREADS) a.ws_pref[i] = pref[i];
  const int R0 = range_start(pair, T, a.pairs), R1 = range_start(pair + 1, T, a.pairs);

  if (warp == REST_PRODUCER_WARP) {
    // ------------------------------------------------------------ Q and rest-part producer
    if (lane == 0) {
      SegWalk w;
      w.init(pref, a.B, R0, R1);
      int sb, g0, g1, seg = 0, g = 0;
      bool ok = true;
      int issued = 0;
      int q_last = -1;
      // A second cursor runs PREFETCH_PAGES pages ahead and prefetches each
      // page it passes into L2 (one contiguous 72 KB bulk prefetch).
      SegWalk wp;
      wp.init(pref, a.B, R0, R1);
      int p_b = 0, p_g0 = 0, p_g1 = 0, p_gp = 0;
      bool p_more = wp.next(p_b, p_g0, p_g1);
      if (p_more) p_gp = p_g0;
      auto prefetch_next = [&]() {
        if (!p_more) return;
        const int page = a.block_table[(size_t)(p_b / a.s_q) * a.max_pages + (p_gp - pref[p_b])];
        if (page >= 0 && page < a.num_pages) l2_prefetch(a.kv + (size_t)page * (PAGE * DK * 2), PAGE * DK * 2);
        if (++p_gp == p_g1) {
          p_more = wp.next(p_b, p_g0, p_g1);
          if (p_more) p_gp = p_g0;
        }
      };
      for (int i = 0; i < PREFETCH_PAGES; ++i) prefetch_next();
      while (ok && w.next(sb, g0, g1)) {
        if (!mbar_wait(bar(B_QE), (seg & 1) ^ 1, abort_flag, a.status)) break;
        mbar_arrive_expect_tx(bar(B_QF), Q_BYTES);
        for (int ch = 0; ch < Q_SMEM_CHUNKS; ++ch)
          tma_load_2d(base + OFF_Q + ch * Q_CHUNK_BYTES, &tm_q, bar(B_QF), ch * 64, sb * HQ);
        q_last = seg;
        const int32_t* row = a.block_table + (size_t)(sb / a.s_q) * a.max_pages;
        for (int gp = g0; gp < g1; ++gp, ++g) {
          int page = row[gp - pref[sb]];
          if (page < 0 || page >= a.num_pages) {
            atomicExch(a.status, (int)ATTN_ERR_INVALID_ARG);
            page = 0;   // never read outside the pool; the result of this sequence is undefined
          }
          for (int j = 0; j < REST_CHUNKS && ok; ++j) {
            if (!mbar_wait(bar(B_RE + j), (g & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
            mbar_arrive_expect_tx(bar(B_RF), PAGE_CHUNK_BYTES);
            tma_load_2d(base + OFF_REST + j * PAGE_CHUNK_BYTES, &tm_kv, bar(B_RF), rest_chunk_dim(half, j) * 64,
                        page * PAGE);
          }
          if (!ok) break;
          ++issued;
          prefetch_next();
        }
        ++seg;
      }
      // the last page's chunks (a page whose loads were cut short by an abort
      // never completes its phase; the drain wait is bounded)
      if (issued > 0) mbar_wait_drain(bar(B_RF), (issued - 1) & 1);
      if (q_last >= 0) mbar_wait_drain(bar(B_QF), q_last & 1);
    }
    __syncwarp();
  } else if (warp == OWN_PRODUCER_WARP) {
    // ------------------------------------------------------------ own-part producer
    // Waits only for the P V product that frees its slot, never behind a
    // rest part, so each own part is asked for as soon as its slot is free.
    if (lane == 0) {
      SegWalk w;
      w.init(pref, a.B, R0, R1);
      int sb, g0, g1, g = 0;
      bool ok = true;
      int issued = 0;
      while (ok && w.next(sb, g0, g1)) {
        const int32_t* row = a.block_table + (size_t)(sb / a.s_q) * a.max_pages;
        for (int gp = g0; gp < g1; ++gp, ++g) {
          int page = row[gp - pref[sb]];
          if (page < 0 || page >= a.num_pages) page = 0;   // recorded by the rest producer
          const int st = g % OWN_STAGES;
          if (!mbar_wait(bar(B_OE + st), ((g / OWN_STAGES) & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(B_OF + st), OWN_BYTES);
          for (int j = 0; j < OWN_CHUNKS; ++j)
            tma_load_2d(base + OFF_OWN + st * OWN_BYTES + j * PAGE_CHUNK_BYTES, &tm_kv, bar(B_OF + st),
                        own_chunk_dim(half, j) * 64, page * PAGE);
          ++issued;
        }
      }
      for (int j = max(0, issued - OWN_STAGES); j < issued; ++j)
        mbar_wait_drain(bar(B_OF + j % OWN_STAGES), (j / OWN_STAGES) & 1);
    }
    __syncwarp();
  } else if (warp == MMA_S_WARP) {
    // ------------------------------------------------------------ score MMA issuer
    // Two warps issue MMAs, each waiting only for what its own products need:
    // this one S = Q K^T per page (page parts landed, S buffer read by the
    // softmax), the next one O += P V (P written).  A P V product therefore
    // never waits behind the next page's load.  S, P and O occupy disjoint
    // TMEM columns, so the two issue streams need no ordering between them
    // beyond those barriers.
    // The 36 k-steps of a score tile take the rest part's chunks first; a
    // commit then frees the rest slot while the own chunks are multiplied.
    // Warp-uniform schedule; one elected lane issues (predicated, no branch).
    const bool leader = elect_one();
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, PAGE, false);
    SegWalk w;
    w.init(pref, a.B, R0, R1);
    int sb, g0, g1, seg = 0, g = 0;
    bool ok = true;
    const uint64_t qdesc = sdesc_sw128(base + OFF_Q, 16, 1024);
    // The k-steps of the chunks of one part, fully unrolled for this CTA's
    // half so that every descriptor is the part's base plus a constant (the
    // issue rate of these N=64 products is what bounds the score tile).
    auto part_mmas = [&](auto half_c, auto rest_c, uint32_t d_tmem, uint64_t kdesc) {
      constexpr int H = decltype(half_c)::value;
      constexpr bool REST = decltype(rest_c)::value;
      constexpr int NCH = REST ? REST_CHUNKS : OWN_CHUNKS;
#pragma unroll
      for (int j = 0; j < NCH; ++j) {
        const int c = REST ? (j < OWN_CHUNKS ? OWN_CHUNKS * (1 - H) + j : CHUNKS - 1) : OWN_CHUNKS * H + j;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const uint32_t acc = (REST && j == 0 && k4 == 0) ? 0u : 1u;
          const uint64_t kd = kdesc + ((j * PAGE_CHUNK_BYTES + k4 * 32) >> 4);
          if (c < Q_SMEM_CHUNKS)
            mma_ss(d_tmem, qdesc + ((c * Q_CHUNK_BYTES + k4 * 32) >> 4), kd, idesc_s, acc, leader);
          else
            mma_ts(d_tmem, tmem + Q_COL + ((c - Q_SMEM_CHUNKS) * 4 + k4) * 8, kd, idesc_s, acc, leader);
        }
        if (REST) mma_commit(bar(B_RE + j), leader);   // rest chunk j may be refilled
      }
    };
    while (ok && w.next(sb, g0, g1)) {
      if (!warp_wait(bar(B_QF), seg & 1, abort_flag, a.status)) break;
      if (!warp_wait(bar(B_QT), seg & 1, abort_flag, a.status)) break;
      for (int gp = g0; gp < g1; ++gp, ++g) {
        const int os = g % OWN_STAGES, sbuf = g & 1;
        const uint32_t s_tmem = tmem + S_COL + sbuf * PAGE;
        if (!warp_wait(bar(B_RF), g & 1, abort_flag, a.status)) { ok = false; break; }
        // S buffer `sbuf` last held page g-2, whose P the P V product of page
        // g-2 reads; that product (and with it the softmax's read of S) must be
        // done.  Pages complete in order, and page g itself cannot complete
        // before this issue, so the per-buffer barrier is never two phases ahead.
        if (g >= 2 && !warp_wait(bar(B_SB + sbuf), ((g >> 1) - 1) & 1, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        const uint64_t rdesc = sdesc_sw128(base + OFF_REST, 16, 1024);
        if (half == 0) part_mmas(std::integral_constant<int, 0>(), std::true_type(), s_tmem, rdesc);
        else part_mmas(std::integral_constant<int, 1>(), std::true_type(), s_tmem, rdesc);
        __syncwarp();
        if (!warp_wait(bar(B_OF + os), (g / OWN_STAGES) & 1, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        const uint64_t odesc = sdesc_sw128(base + OFF_OWN + os * OWN_BYTES, 16, 1024);
        if (half == 0) part_mmas(std::integral_constant<int, 0>(), std::false_type(), s_tmem, odesc);
        else part_mmas(std::integral_constant<int, 1>(), std::false_type(), s_tmem, odesc);
        mma_commit(bar(B_SF + sbuf), leader);
        if (gp == g1 - 1) mma_commit(bar(B_QE), leader);   // last score tile of the segment: Q may be replaced
        __syncwarp();
      }
      ++seg;
    }
    // Drain: no MMA may still run when TMEM is released.
    mma_commit(bar(B_DRS), leader);
    __syncwarp();
    mbar_wait_drain(bar(B_DRS), 0);
    __syncwarp();
  } else if (warp == MMA_PV_WARP) {
    // ------------------------------------------------------------ P V MMA issuer
    // The P of a segment's first page is written only after the previous
    // segment's epilogue has read O (same softmax warps, in order), so the
    // overwrite of O by that page's product needs no extra barrier.  S of a
    // page is complete before its P exists, so this warp's completion of
    // P V also means the page's own part is no longer read by any MMA.
    const bool leader = elect_one();
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, 256, true);
    SegWalk w;
    w.init(pref, a.B, R0, R1);
    int sb, g0, g1, g = 0;
    bool ok = true;
    while (ok && w.next(sb, g0, g1)) {
      for (int gp = g0; gp < g1; ++gp, ++g) {
        if (!warp_wait(bar(B_PF), g & 1, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        const int os = g % OWN_STAGES;
        const uint64_t vdesc = sdesc_sw128(base + OFF_OWN + os * OWN_BYTES, PAGE_CHUNK_BYTES, 1024);
        const uint32_t p_tmem = tmem + S_COL + (g & 1) * PAGE;   // P over its page's S buffer
#pragma unroll
        for (int kk = 0; kk < PAGE / 16; ++kk)
          mma_ts(tmem + O_COL, p_tmem + kk * 8, vdesc + ((kk * 16 * 128) >> 4), idesc_o,
                 (gp == g0 && kk == 0) ? 0u : 1u, leader);
        mma_commit(bar(B_OD), leader);
        mma_commit(bar(B_SB + (g & 1)), leader);
        mma_commit(bar(B_OE + os), leader);   // the own part's slot is free
        __syncwarp();
      }
    }
    mma_commit(bar(B_DR), leader);
    __syncwarp();
    mbar_wait_drain(bar(B_DR), 0);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax (thread = head)
    const int h = warp * 32 + lane;
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    const uint32_t t_row = tmem + lane_off;
    const float sl2 = a.scale_log2;
    SegWalk w;
    w.init(pref, a.B, R0, R1);
    int sb, g0, g1, seg = 0, g = 0;
    bool ok = true;
    while (ok && w.next(sb, g0, g1)) {
      // Q dims 320..575 of this head into TMEM (the previous segment's score
      // MMAs are complete: its epilogue waited for its last P V product).
      {
        const uint4* src = reinterpret_cast<const uint4*>(a.q + ((size_t)sb * HQ + h) * DK + 64 * Q_SMEM_CHUNKS);
#pragma unroll
        for (int c = 0; c < Q_TMEM_DIMS / 64; ++c) {
          uint32_t r[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint4 u = __ldg(src + c * 8 + i);
            r[4 * i] = u.x;
            r[4 * i + 1] = u.y;
            r[4 * i + 2] = u.z;
            r[4 * i + 3] = u.w;
          }
          tmem_st32(t_row + Q_COL + c * 32, r);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_QT));
      }
      const int L = unit_len(a, sb);
      const int first_page = pref[sb];
      float m_run = -INFINITY, l_run = 0.f;
      for (int gp = g0; gp < g1; ++gp, ++g) {
        const uint32_t s_row = t_row + S_COL + (g & 1) * PAGE;   // this page's S buffer
        if (!warp_wait(bar(B_SF + (g & 1)), (g >> 1) & 1, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        uint32_t s[PAGE];
        tmem_ld64_sync(s_row, s);
        const int valid = L - (gp - first_page) * PAGE;   // tokens of this page inside the sequence
        const bool partial = valid < PAGE;
        if (partial) {
#pragma unroll
          for (int c = 0; c < PAGE; ++c)
            if (c >= valid) s[c] = __float_as_uint(-INFINITY);
        }
        const float mx = row_max<PAGE>(s);
        const float m_new = fmaxf(m_run, mx * sl2);
        const bool grow = m_new > m_run + kRescaleThreshold;
        const float m_use = grow ? m_new : m_run;
        const float alpha = grow ? ex2(m_run - m_use) : 1.f;
        const float m_eff = (m_use == -INFINITY) ? 0.f : m_use;
        uint32_t p[PAGE / 2];
        // A page cut by the sequence end uses the MUFU exp2 only (its masked
        // scores are -inf and must give exactly 0); full pages send part of
        // the work to the FMA pipe.
        const float sum = partial ? exp_row<PAGE, false>(s, p, sl2, m_eff) : exp_row<PAGE, true>(s, p, sl2, m_eff);
        l_run = l_run * alpha + sum;
        m_run = m_use;
        if (gp > g0) {
          // the previous page's P V product must be complete before O changes
          // (and before this page's P is announced: the P barrier then never
          // runs two phases ahead of the P V issuer)
          if (!warp_wait(bar(B_OD), (g - 1) & 1, abort_flag, a.status)) { ok = false; break; }
          if (__any_sync(0xffffffffu, grow)) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < 256 / 32; ++c) {
              uint32_t o[32];
              tmem_ld32_sync(t_row + O_COL + c * 32, o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(t_row + O_COL + c * 32, o);
            }
          }
        }
        tmem_st32(s_row, p);   // P over the first PAGE/2 columns of the S just read
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_PF));
      }
      if (!ok) break;
      // -------------------------------------------------------- segment epilogue
      if (!warp_wait(bar(B_OD), (g - 1) & 1, abort_flag, a.status)) { ok = false; break; }
      tc_fence_after();
      const bool full = (g0 == pref[sb]) && (g1 == pref[sb + 1]);
      const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
      const float lse = (l_run > 0.f) ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
      int slot = 2 * pair + (g0 == R0 ? 0 : 1);
#pragma unroll 1
      for (int c = 0; c < 256 / 32; ++c) {
        uint32_t o[32];
        tmem_ld32_sync(t_row + O_COL + c * 32, o);
        const int col = half * 256 + c * 32;
        if (full) {
          uint4* dst = reinterpret_cast<uint4*>(a.o + ((size_t)sb * HQ + h) * DV + col);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(o[8 * i + 0]) * inv_l, __uint_as_float(o[8 * i + 1]) * inv_l);
            u.y = pack_bf16x2(__uint_as_float(o[8 * i + 2]) * inv_l, __uint_as_float(o[8 * i + 3]) * inv_l);
            u.z = pack_bf16x2(__uint_as_float(o[8 * i + 4]) * inv_l, __uint_as_float(o[8 * i + 5]) * inv_l);
            u.w = pack_bf16x2(__uint_as_float(o[8 * i + 6]) * inv_l, __uint_as_float(o[8 * i + 7]) * inv_l);
            dst[i] = u;
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(a.ws_o + ((size_t)slot * HQ + h) * DV + col);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv_l, __uint_as_float(o[4 * i + 1]) * inv_l,
                                 __uint_as_float(o[4 * i + 2]) * inv_l, __uint_as_float(o[4 * i + 3]) * inv_l);
        }
      }
      if (half == 0) {
        if (full) a.lse[(size_t)sb * HQ + h] = lse;
        else a.ws_lse[(size_t)slot * HQ + h] = lse;
      }
      tc_fence_before();
      __syncwarp();
      ++seg;
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// One CTA per (sequence, group of 16 heads): merges the partial results of a
// sequence that several CTA pairs shared; writes O = 0, LSE = -inf for an
// empty sequence; leaves sequences written by the split kernel untouched.
constexpr int COMBINE_HEADS = 16;
constexpr int COMBINE_THREADS = 256;
constexpr int MAX_PARTS = 128;   // >= CTA pairs, so a sequence never has more pieces

__global__ void __launch_bounds__(COMBINE_THREADS)
    decode_combine_kernel(const Args a) {
  const int b = blockIdx.x;
  const int h0 = blockIdx.y * COMBINE_HEADS;
  const int tid = threadIdx.x;
  const int T = a.ws_pref[a.B];
  const int s0 = a.ws_pref[b], s1 = a.ws_pref[b + 1];
  if (s1 == s0) {
    for (int i = tid; i < COMBINE_HEADS * DV; i += COMBINE_THREADS)
      a.o[((size_t)b * HQ + h0) * DV + i] = __float2bfloat16(0.f);
    if (tid < COMBINE_HEADS) a.lse[(size_t)b * HQ + h0 + tid] = -INFINITY;
    return;
  }
  const int p_lo = pair_of_page(s0, T, a.pairs), p_hi = pair_of_page(s1 - 1, T, a.pairs);
  if (p_lo == p_hi) return;
  __shared__ float w_s[COMBINE_HEADS][MAX_PARTS];
  __shared__ int slot_s[MAX_PARTS];
  __shared__ int nparts_s;
  if (tid == 0) {
    // pairs with an empty range (fewer pages than pairs) hold no piece
    int n = 0;
    for (int p = p_lo; p <= p_hi && n < MAX_PARTS; ++p) {
      const int r0 = range_start(p, T, a.pairs);
      if (range_start(p + 1, T, a.pairs) == r0) continue;
      slot_s[n++] = 2 * p + ((p == p_lo && s0 != r0) ? 1 : 0);
    }
    nparts_s = n;
  }
  __syncthreads();
  const int nparts = nparts_s;
  if (tid < COMBINE_HEADS) {
    const int h = h0 + tid;
    float mx = -INFINITY;
    for (int i = 0; i < nparts && i < MAX_PARTS; ++i) mx = fmaxf(mx, a.ws_lse[(size_t)slot_s[i] * HQ + h]);
    float sum = 0.f;
    for (int i = 0; i < nparts && i < MAX_PARTS; ++i) {
      const float e = (mx == -INFINITY) ? 0.f : expf(a.ws_lse[(size_t)slot_s[i] * HQ + h] - mx);
      w_s[tid][i] = e;
      sum += e;
    }
    const float inv = sum > 0.f ? 1.f / sum : 0.f;
    for (int i = 0; i < nparts && i < MAX_PARTS; ++i) w_s[tid][i] *= inv;
    a.lse[(size_t)b * HQ + h] = sum > 0.f ? mx + logf(sum) : -INFINITY;
  }
  __syncthreads();
  // 16 heads x 512 columns, 4 columns per thread per step
  for (int i = tid; i < COMBINE_HEADS * DV / 4; i += COMBINE_THREADS) {
    const int hh = i / (DV / 4), c4 = i % (DV / 4);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < nparts && j < MAX_PARTS; ++j) {
      const float wgt = w_s[hh][j];
      const float4 v = *reinterpret_cast<const float4*>(a.ws_o + ((size_t)slot_s[j] * HQ + h0 + hh) * DV + c4 * 4);
      acc.x += wgt * v.x;
      acc.y += wgt * v.y;
      acc.z += wgt * v.z;
      acc.w += wgt * v.w;
    }
    __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(a.o + ((size_t)b * HQ + h0 + hh) * DV + c4 * 4);
    dst[0] = __floats2bfloat162_rn(acc.x, acc.y);
    dst[1] = __floats2bfloat162_rn(acc.z, acc.w);
  }
}

struct WsLayout {
  size_t off_pref, off_lse, off_o, total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WsLayout ws_layout(int B, int pairs) {
  WsLayout w;
  w.off_pref = 0;
  w.off_lse = align256((size_t)(B + 1) * 4);
  w.off_o = w.off_lse + align256((size_t)2 * pairs * HQ * 4);
  w.total = w.off_o + (size_t)2 * pairs * HQ * DV * 4;
  return w;
}

inline int pairs_for_sms(int sms) { return sms >= 2 ? sms / 2 : 0; }

}  // namespace dec
}  // namespace ea

extern "C" size_t attn_decode_paged_mtp_workspace_size(int B, int s_q, int Hq, int Dv, int device) {
  using namespace ea::dec;
  if (B < 1 || s_q < 1 || (long long)B * s_q > B_MAX || Hq != HQ || Dv != DV) return 0;
  const int pairs = pairs_for_sms(ea::sm_count_of(device));
  if (pairs == 0 || pairs > MAX_PARTS) return 0;
  return ws_layout(B * s_q, pairs).total;
}

extern "C" size_t attn_decode_paged_workspace_size(int B, int Hq, int Dv, int device) {
  return attn_decode_paged_mtp_workspace_size(B, 1, Hq, Dv, device);
}

extern "C" int attn_decode_paged_mtp(const void* q, const void* kv_pages, const int32_t* block_table,
                                     const int32_t* cache_seqlens, void* o, float* lse, int B, int s_q, int Hq, int Dk,
                                     int Dv, int page_size, int num_pages, int max_pages_per_seq, float scale,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  using namespace ea;
  using namespace ea::dec;
  if (!q || !kv_pages || !block_table || !cache_seqlens || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kv_pages, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(block_table, 4) || !aligned(cache_seqlens, 4))
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || s_q < 1 || num_pages < 1 || max_pages_per_seq < 1 || page_size < 1 || Hq < 1 || Dk < 1 || Dv < 1)
    return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (Hq != HQ || Dk != DK || Dv != DV || page_size != PAGE || (long long)B * s_q > B_MAX)
    return ATTN_ERR_UNSUPPORTED;
  const int units = B * s_q;
  if ((long long)num_pages * PAGE >= (1ll << 31) || (long long)B * max_pages_per_seq >= (1ll << 31))
    return ATTN_ERR_UNSUPPORTED;
  const int pairs = pairs_for_sms(current_sm_count());
  if (pairs == 0) return ATTN_ERR_CUDA;
  if (pairs > MAX_PARTS) return ATTN_ERR_UNSUPPORTED;
  const WsLayout wl = ws_layout(units, pairs);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < wl.total) return ATTN_ERR_WORKSPACE;

  static int attr_done = 0;
  if (int rc = ensure_smem_attr(reinterpret_cast<const void*>(&decode_split_kernel), SMEM_BYTES, &attr_done))
    return rc;
  int* status = device_status_ptr();
  if (!status) return ATTN_ERR_CUDA;

  CUtensorMap tq, tkv;
  {
    const uint64_t dims[2] = {(uint64_t)DK, (uint64_t)units * HQ};
    const uint64_t strides[1] = {(uint64_t)DK * 2};
    const uint32_t box[2] = {64, (uint32_t)HQ};
    if (!encode_bf16_2d(&tq, q, dims, strides, box)) return ATTN_ERR_CUDA;
  }
  {
    const uint64_t dims[2] = {(uint64_t)DK, (uint64_t)num_pages * PAGE};
    const uint64_t strides[1] = {(uint64_t)DK * 2};
    const uint32_t box[2] = {64, (uint32_t)PAGE};
    if (!encode_bf16_2d(&tkv, kv_pages, dims, strides, box)) return ATTN_ERR_CUDA;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  Args a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.kv = static_cast<const uint8_t*>(kv_pages);
  a.block_table = block_table;
  a.seqlens = cache_seqlens;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.ws_pref = reinterpret_cast<int32_t*>(ws + wl.off_pref);
  a.ws_lse = reinterpret_cast<float*>(ws + wl.off_lse);
  a.ws_o = reinterpret_cast<float*>(ws + wl.off_o);
  a.status = status;
  a.B = units;
  a.s_q = s_q;
  a.max_pages = max_pages_per_seq;
  a.num_pages = num_pages;
  a.pairs = pairs;
  a.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  decode_split_kernel<<<2 * pairs, THREADS, SMEM_BYTES, s>>>(tq, tkv, a);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  decode_combine_kernel<<<dim3(units, HQ / COMBINE_HEADS), COMBINE_THREADS, 0, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

extern "C" int attn_decode_paged(const void* q, const void* kv_pages, const int32_t* block_table,
                                 const int32_t* cache_seqlens, void* o, float* lse, int B, int Hq, int Dk, int Dv,
                                 int page_size, int num_pages, int max_pages_per_seq, float scale, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  return attn_decode_paged_mtp(q, kv_pages, block_table, cache_seqlens, o, lse, B, 1, Hq, Dk, Dv, page_size,
                               num_pages, max_pages_per_seq, scale, workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------------------
// Allocation-free variant of attn_decode_paged.
//
// Some callers cannot allocate device memory when they decode: a serving
// engine that hands the whole of HBM to its own KV-cache pool at start-up has
// no spare allocation to give a per-call workspace, and latency-critical
// decode loops are often not allowed to call the CUDA allocator at all.  For
// them the split-KV workspace lives in a fixed array of this library instead.
//
// The array below is a host-side stand-in in host code, not a device
// address: its device address is looked up once per device (with that device
// current) and cached.  The first call on each device performs that lookup,
// so make the first call on a device before any stream capture.  Every GPU
// that loads this library holds the array (kNoAllocScratchBytes) until the
// process exits.  All calls share it and it keeps the last call's contents:
// nothing in it has to start at zero (every value the kernels read is written
// earlier in the same call), but calls whose kernels overlap on the GPU (two
// streams, or two threads) race on it and must be serialised by the caller.
namespace ea {
namespace dec {

constexpr size_t kNoAllocScratchBytes = size_t(40) << 20;   // 40 MiB

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};

// Device address of the scratch array on the current device, or nullptr.
void* noalloc_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress((void**)&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_ptr[dev] = p;
  }
  return g_noalloc_ptr[dev];
}
}  // namespace

}  // namespace dec
}  // namespace ea

extern "C" size_t attn_decode_paged_noalloc_max_bytes(void) { return ea::dec::kNoAllocScratchBytes; }

extern "C" int attn_decode_paged_noalloc(const void* q, const void* kv_pages, const int32_t* block_table,
                                         const int32_t* cache_seqlens, void* o, float* lse, int B, int Hq, int Dk,
                                         int Dv, int page_size, int num_pages, int max_pages_per_seq, float scale,
                                         void* stream) {
  using namespace ea::dec;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  const size_t need = attn_decode_paged_workspace_size(B, Hq, Dv, dev);
  if (need > kNoAllocScratchBytes) return ATTN_ERR_UNSUPPORTED;   // batch too large for the fixed array
  void* scratch = noalloc_scratch();
  if (!scratch) return ATTN_ERR_CUDA;
  return attn_decode_paged(q, kv_pages, block_table, cache_seqlens, o, lse, B, Hq, Dk, Dv, page_size, num_pages,
                           max_pages_per_seq, scale, scratch, kNoAllocScratchBytes, stream);
}
