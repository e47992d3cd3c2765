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
// is computed while the softmax still reads that of page g.  P (bf16) goes to
// a shared-memory tile (the A operand of the P V product), so an S buffer is
// free again as soon as the softmax has read it.  Q dims 0..319 sit in shared
// memory (80 KB).
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
// Own parts are held until the P V product and get two stages: the own part
// of page g+2 is asked for when the P V product of page g is done, about one
// page period before the score MMAs of page g+2 reach it.
constexpr int OWN_STAGES = 2;
constexpr int REST_STAGES = 1;
constexpr int O_COL = 0;
constexpr int S_COL = 256;                      // two buffers of PAGE columns
constexpr int Q_COL = 384;
constexpr int TMEM_COLS = 512;
// Warps: two softmax groups of four (0-3 and 8-11), two producers, the score
// MMA issuer and one idle warp.  Each head's row is shared by the two groups
// (warps w and w+8 reach the same TMEM lanes): group G takes score columns
// [32G, 32G+32) and output columns [128G, 128G+128) of the CTA's half, so the
// per-page softmax latency, the rescales and the epilogue are split in two.
// The groups agree on each row's max through shared memory, and warp 0
// issues the P V product once both have written their half of P.
constexpr int THREADS = 384;
constexpr int REST_PRODUCER_WARP = 4;           // Q and the rest parts (and the L2 prefetches)
constexpr int MMA_S_WARP = 5;                   // score tiles S = Q K^T
constexpr int OWN_PRODUCER_WARP = 7;            // the own parts
constexpr int SOFTMAX_THREADS = 256;
constexpr int BAR_MAX = 1, BAR_P = 2, BAR_L = 3;   // named barriers of the two softmax groups
// barriers
constexpr int B_QF = 0, B_QE = 1, B_QT = 2;
constexpr int B_RF = 3;                          // rest part landed (one arrival per chunk)
constexpr int B_RE = B_RF + 1;                   // rest chunk j read, one barrier per chunk
constexpr int B_OF = B_RE + REST_CHUNKS, B_OE = B_OF + OWN_STAGES;
constexpr int B_SF = B_OE + OWN_STAGES;         // score tile complete, one per S buffer
constexpr int B_SB = B_SF + 2;                   // score tile read by the softmax, one per S buffer
constexpr int B_OD = B_SB + 2, B_DR = B_OD + 1, B_DRS = B_DR + 1;
constexpr int NBAR = B_DRS + 1;
// shared memory
constexpr int OFF_Q = 0;
constexpr int OFF_OWN = OFF_Q + Q_BYTES;
constexpr int OFF_REST = OFF_OWN + OWN_STAGES * OWN_BYTES;
// Per softmax warp, a 32 x 128-byte tile through which the segment epilogue
// transposes O, so that each global store writes whole row pieces.  The
// first 16 KB also hold P (128 heads x 64 tokens bf16, 128-byte swizzled
// rows): the epilogue runs only after the segment's last P V product.
constexpr int XPOSE_BYTES = 32 * 128;
constexpr int OFF_XPOSE = OFF_REST + REST_STAGES * REST_BYTES;
constexpr int OFF_P = OFF_XPOSE;
static_assert(HQ * PAGE * 2 <= 8 * XPOSE_BYTES, "P fits in the transpose tiles");
constexpr int OFF_BAR = OFF_XPOSE + 8 * XPOSE_BYTES;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int OFF_XCH = OFF_MISC + 16;          // [2][HQ] floats exchanged by the softmax groups
constexpr int OFF_PREF = OFF_XCH + 2 * HQ * 4;
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
// u = i * n_seq + b is query token i of sequence b (token-major), and its
// rows of q, o and lse are b * s_q + i.  The s_q tokens are the last s_q
// cached tokens, so unit u sees positions 0 .. L_b - s_q + i (the causal mask
// aligned to the bottom-right corner) of block-table row b.  Token-major
// order puts the s_q units of a sequence 1/s_q of the split plan apart, so
// CTA pairs that far apart walk the same pages at about the same time and
// the later read of a page comes from L2.
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
  int s_q, n_seq, max_pages, num_pages, pairs;
  float scale_log2;
};

__device__ __forceinline__ int unit_seq(const Args& a, int u) { return u % a.n_seq; }
__device__ __forceinline__ int unit_tok(const Args& a, int u) { return u / a.n_seq; }
// Row of unit u in q [B, s_q, Hq, DK], o and lse.
__device__ __forceinline__ int unit_row(const Args& a, int u) { return unit_seq(a, u) * a.s_q + unit_tok(a, u); }

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
  const int L = seq_len_eff(a.seqlens[unit_seq(a, u)], a.max_pages) - (a.s_q - 1 - unit_tok(a, u));
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

// Block-table entries of the pages of [R0, R1) in order (a page that is
// not there reads as -1).
constexpr int LOOKAHEAD = 4;
static_assert(PREFETCH_PAGES >= 1 && PREFETCH_PAGES < LOOKAHEAD, "prefetch distance within the lookahead");
struct PageCursor {
  SegWalk w;
  const int* pref;
  const int32_t* row;
  int gp, g1;
  bool more;
  __device__ void init(const int* pref_, const Args& a, int R0, int R1) {
    pref = pref_;
    w.init(pref_, a.B, R0, R1);
    int sb, g0;
    more = w.next(sb, g0, g1);
    if (more) {
      gp = g0;
      row = a.block_table + (size_t)unit_seq(a, sb) * a.max_pages - pref[sb];
    }
  }
  __device__ int next_with(const Args& a) {
    if (!more) return -1;
    const int page = row[gp];
    if (++gp == g1) {
      int sb, g0;
      more = w.next(sb, g0, g1);
      if (more) {
        gp = g0;
        row = a.block_table + (size_t)unit_seq(a, sb) * a.max_pages - pref[sb];
      }
    }
    return page;
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

  // Let the combine kernel be scheduled as this grid's CTAs retire (it waits
  // for this grid's completion before reading anything).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x >> 1;
  const int half = blockIdx.x & 1;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QF), 1);
    mbar_init(bar(B_QE), 1);
    mbar_init(bar(B_QT), 8);
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
    mbar_init(bar(B_OD), 1);
    mbar_init(bar(B_DR), 1);
    mbar_init(bar(B_DRS), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // Prefix sums of pages per query unit (B <= B_MAX): every thread loads the
  // lengths of some units at once (one memory latency), then warp 0 scans
  // them in shared memory.
  {
    bool bad = false;
    for (int u = threadIdx.x; u < a.B; u += THREADS) {
      const int L = a.seqlens[unit_seq(a, u)];
      pref[u + 1] = seq_pages(unit_len(a, u), a.max_pages);
      bad |= (L < 0) || ((long long)L > (long long)a.max_pages * PAGE);
    }
    if (bad && blockIdx.x == 0) atomicExch(a.status, (int)ATTN_ERR_INVALID_ARG);
  }
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    for (int b0 = 0; b0 < a.B; b0 += 32) {
      const int b = b0 + lane;
      int x = b < a.B ? pref[b + 1] : 0;   // inclusive warp scan
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (b < a.B) pref[b + 1] = carry + x;
      carry += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) pref[0] = 0;
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
      // A second cursor runs ahead of the loads and reads the block-table
      // entries of the next LOOKAHEAD pages into registers (independent loads,
      // so the first pages cost one memory latency, not one each); each page
      // is also prefetched into L2 when it is PREFETCH_PAGES ahead of the load.
      PageCursor cur;
      cur.init(pref, a, R0, R1);
      int ids[LOOKAHEAD];
#pragma unroll
      for (int i = 0; i < LOOKAHEAD; ++i) ids[i] = cur.next_with(a);
#pragma unroll
      for (int i = 0; i < PREFETCH_PAGES; ++i)
        if (ids[i] >= 0 && ids[i] < a.num_pages) l2_prefetch(a.kv + (size_t)ids[i] * (PAGE * DK * 2), PAGE * DK * 2);
      while (ok && w.next(sb, g0, g1)) {
        if (!mbar_wait(bar(B_QE), (seg & 1) ^ 1, abort_flag, a.status)) break;
        mbar_arrive_expect_tx(bar(B_QF), Q_BYTES);
        for (int ch = 0; ch < Q_SMEM_CHUNKS; ++ch)
          tma_load_2d(base + OFF_Q + ch * Q_CHUNK_BYTES, &tm_q, bar(B_QF), ch * 64, unit_row(a, sb) * HQ);
        q_last = seg;
        for (int gp = g0; gp < g1; ++gp, ++g) {
          int page = ids[0];
#pragma unroll
          for (int i = 0; i + 1 < LOOKAHEAD; ++i) ids[i] = ids[i + 1];
          ids[LOOKAHEAD - 1] = cur.next_with(a);
          {
            const int pf = ids[PREFETCH_PAGES - 1];   // the page PREFETCH_PAGES ahead of this one
            if (pf >= 0 && pf < a.num_pages) l2_prefetch(a.kv + (size_t)pf * (PAGE * DK * 2), PAGE * DK * 2);
          }
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
        const int32_t* row = a.block_table + (size_t)unit_seq(a, sb) * a.max_pages;
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
    // MMAs come from two warps, each waiting only for what its own products
    // need: this one issues S = Q K^T per page (page parts landed, S buffer
    // read by the softmax), softmax warp 0 issues O += P V once P is written.
    // A P V product therefore never waits behind the next page's load.  S and
    // O occupy disjoint TMEM columns and P lives in shared memory, so the two
    // issue streams need no ordering between them beyond those barriers.
    // The 36 k-steps of a score tile take the rest part's chunks first, with a
    // commit per chunk that lets the producer refill it, then the own chunks.
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
        // the whole rest part (one barrier: waiting chunk by chunk inside the
        // issue stream slows the score products more than it saves)
        if (!warp_wait(bar(B_RF), g & 1, abort_flag, a.status)) { ok = false; break; }
        // S buffer `sbuf` last held page g-2: the softmax must have read it.
        // The softmax reads tiles in order, and page g's tile cannot be read
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
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ idle warp
  } else {
    // ------------------------------------------------------------ softmax (thread = head, two groups)
    const int grp = warp >> 3;                  // 0: warps 0-3, 1: warps 8-11
    const int q4 = warp & 3;
    const int h = q4 * 32 + lane;
    const uint32_t t_row = tmem + (uint32_t(q4 * 32) << 16);
    float* xch = reinterpret_cast<float*>(base_ptr + OFF_XCH);   // [2][HQ]
    const float sl2 = a.scale_log2;
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, 256, true);
    // Q dims 320..575 of unit u's head into TMEM, half per group; the score
    // MMAs of segment s+1 wait for it (barrier QT).
    auto write_q_tmem = [&](int u) {
      const uint4* src = reinterpret_cast<const uint4*>(a.q + ((size_t)unit_row(a, u) * HQ + h) * DK + 64 * Q_SMEM_CHUNKS);
#pragma unroll
      for (int cc = 0; cc < Q_TMEM_DIMS / 128; ++cc) {
        const int c = grp * (Q_TMEM_DIMS / 128) + cc;
        uint32_t r[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v = __ldg(src + c * 8 + i);
          r[4 * i] = v.x;
          r[4 * i + 1] = v.y;
          r[4 * i + 2] = v.z;
          r[4 * i + 3] = v.w;
        }
        tmem_st32(t_row + Q_COL + c * 32, r);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_QT));
    };
    SegWalk w;
    w.init(pref, a.B, R0, R1);
    int sb, g0, g1, seg = 0, g = 0;
    bool ok = true;
    bool have = w.next(sb, g0, g1);
    if (have) write_q_tmem(sb);
    while (ok && have) {
      const int L = unit_len(a, sb);
      const int first_page = pref[sb];
      float m_run = -INFINITY, l_run = 0.f;   // l_run: this group's columns only
      for (int gp = g0; gp < g1; ++gp, ++g) {
        const uint32_t s_row = t_row + S_COL + (g & 1) * PAGE;   // this page's S buffer
        bool good = warp_wait(bar(B_SF + (g & 1)), (g >> 1) & 1, abort_flag, a.status);
        tc_fence_after();
        uint32_t s[32];
        tmem_ld32_sync(s_row + grp * 32, s);
        const int valid = L - (gp - first_page) * PAGE - grp * 32;   // tokens of this half-page in the sequence
        const bool partial = valid < 32;
        if (partial) {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c >= valid) s[c] = __float_as_uint(-INFINITY);
        }
        const float mx_own = row_max<32>(s);
        xch[grp * HQ + h] = mx_own;
        // both groups have read S (its buffer may be refilled) and agree on the max
        tc_fence_before();
        good = named_bar_and(BAR_MAX, SOFTMAX_THREADS, good);
        if (!good) { ok = false; break; }
        if (threadIdx.x == 0) {
          tc_fence_before();
          mbar_arrive(bar(B_SB + (g & 1)));   // both groups have read this page's S
        }
        const float mx = fmaxf(mx_own, xch[(1 - grp) * HQ + h]);
        const float m_new = fmaxf(m_run, mx * sl2);
        const bool grow = m_new > m_run + kRescaleThreshold;
        const float m_use = grow ? m_new : m_run;
        const float alpha = grow ? ex2(m_run - m_use) : 1.f;
        const float m_eff = (m_use == -INFINITY) ? 0.f : m_use;
        uint32_t p[16];
        // A page cut by the sequence end uses the MUFU exp2 only (its masked
        // scores are -inf and must give exactly 0); full pages send part of
        // the work to the FMA pipe.
        const float sum = partial ? exp_row<32, false>(s, p, sl2, m_eff) : exp_row<32, true>(s, p, sl2, m_eff);
        l_run = l_run * alpha + sum;
        m_run = m_use;
        if (gp > g0) {
          // the previous page's P V product must be complete before O changes
          good = warp_wait(bar(B_OD), (g - 1) & 1, abort_flag, a.status);
          if (good && __any_sync(0xffffffffu, grow)) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < 128 / 32; ++c) {
              uint32_t o[32];
              const uint32_t oc = t_row + O_COL + grp * 128 + c * 32;
              tmem_ld32_sync(oc, o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(oc, o);
            }
          }
        }
        // this group's 32 tokens of P into row h of the P tile (units 4G..4G+3
        // of the 128-byte row, XOR-swizzled by h % 8 like a TMA tile)
        {
          const uint32_t prow = base + OFF_P + (uint32_t)h * 128;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            st_shared_v4(prow + (((grp * 4 + k) ^ (h & 7)) * 16), p[4 * k], p[4 * k + 1], p[4 * k + 2], p[4 * k + 3]);
          fence_proxy_async_smem();   // visible to the tensor core's reads
        }
        tc_fence_before();
        good = named_bar_and(BAR_P, SOFTMAX_THREADS, good);
        if (!good) { ok = false; break; }
        if (warp == 0) {
          // O (+)= P V for this page: P from TMEM, V = the own part (its slot
          // is released by the same commit).  S of the page is complete, so
          // its own part has landed.
          tc_fence_after();
          const bool leader = elect_one();
          const int os = g % OWN_STAGES;
          const uint64_t vdesc = sdesc_sw128(base + OFF_OWN + os * OWN_BYTES, PAGE_CHUNK_BYTES, 1024);
          const uint64_t pdesc = sdesc_sw128(base + OFF_P, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < PAGE / 16; ++kk)
            mma_ss(tmem + O_COL, pdesc + ((kk * 32) >> 4), vdesc + ((kk * 16 * 128) >> 4), idesc_o,
                   (gp == g0 && kk == 0) ? 0u : 1u, leader);
          mma_commit(bar(B_OD), leader);
          mma_commit(bar(B_OE + os), leader);   // the own part's slot is free
          __syncwarp();
        }
      }
      if (!ok) break;
      // The next segment's Q goes into TMEM before this epilogue: the last
      // score tile of this segment is complete (its softmax has run), so the
      // next segment's first score tile can be computed during the epilogue.
      int nsb = 0, ng0 = 0, ng1 = 0;
      const bool nhave = w.next(nsb, ng0, ng1);
      if (nhave) write_q_tmem(nsb);
      // -------------------------------------------------------- segment epilogue
      bool good = warp_wait(bar(B_OD), (g - 1) & 1, abort_flag, a.status);
      tc_fence_after();
      xch[grp * HQ + h] = l_run;
      good = named_bar_and(BAR_L, SOFTMAX_THREADS, good);
      if (!good) { ok = false; break; }
      const float l_tot = l_run + xch[(1 - grp) * HQ + h];
      const bool full = (g0 == pref[sb]) && (g1 == pref[sb + 1]);
      const float inv_l = (l_tot > 0.f) ? 1.f / l_tot : 0.f;
      const float lse = (l_tot > 0.f) ? (m_run + log2f(l_tot)) * kLn2 : -INFINITY;
      int slot = 2 * pair + (g0 == R0 ? 0 : 1);
      // Each 32-column chunk of this warp's 32 rows goes through the warp's
      // transpose tile (16-byte units XOR-swizzled by row, so neither side has
      // bank conflicts); read back by rows, every store instruction then
      // writes 4 rows x 128 bytes (fp32) or 8 rows x 64 bytes (bf16) instead
      // of 32 rows x 16 bytes.
      const uint32_t xt = base + OFF_XPOSE + (uint32_t)((grp * 4 + q4) * XPOSE_BYTES);
      const int row0 = q4 * 32;   // first head of this warp
      const int orow = unit_row(a, sb);
#pragma unroll 1
      for (int c = 0; c < 128 / 32; ++c) {
        uint32_t o[32];
        tmem_ld32_sync(t_row + O_COL + grp * 128 + c * 32, o);
        const int col = half * 256 + grp * 128 + c * 32;
        if (full) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            st_shared_v4(xt + lane * 128 + ((k ^ (lane & 7)) * 16),
                         pack_bf16x2(__uint_as_float(o[8 * k + 0]) * inv_l, __uint_as_float(o[8 * k + 1]) * inv_l),
                         pack_bf16x2(__uint_as_float(o[8 * k + 2]) * inv_l, __uint_as_float(o[8 * k + 3]) * inv_l),
                         pack_bf16x2(__uint_as_float(o[8 * k + 4]) * inv_l, __uint_as_float(o[8 * k + 5]) * inv_l),
                         pack_bf16x2(__uint_as_float(o[8 * k + 6]) * inv_l, __uint_as_float(o[8 * k + 7]) * inv_l));
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int r = 8 * j + (lane >> 2), u = lane & 3;
            uint32_t v0, v1, v2, v3;
            ld_shared_v4(xt + r * 128 + ((u ^ (r & 7)) * 16), v0, v1, v2, v3);
            *reinterpret_cast<uint4*>(a.o + ((size_t)orow * HQ + row0 + r) * DV + col + 8 * u) = make_uint4(v0, v1, v2, v3);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            st_shared_v4(xt + lane * 128 + ((k ^ (lane & 7)) * 16),
                         __float_as_uint(__uint_as_float(o[4 * k + 0]) * inv_l),
                         __float_as_uint(__uint_as_float(o[4 * k + 1]) * inv_l),
                         __float_as_uint(__uint_as_float(o[4 * k + 2]) * inv_l),
                         __float_as_uint(__uint_as_float(o[4 * k + 3]) * inv_l));
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int r = 4 * j + (lane >> 3), u = lane & 7;
            uint32_t v0, v1, v2, v3;
            ld_shared_v4(xt + r * 128 + ((u ^ (r & 7)) * 16), v0, v1, v2, v3);
            *reinterpret_cast<uint4*>(a.ws_o + ((size_t)slot * HQ + row0 + r) * DV + col + 4 * u) =
                make_uint4(v0, v1, v2, v3);
          }
        }
        __syncwarp();   // the tile is rewritten by the next chunk
      }
      if (half == 0 && grp == 0) {
        if (full) a.lse[(size_t)orow * HQ + h] = lse;
        else a.ws_lse[(size_t)slot * HQ + h] = lse;
      }
      tc_fence_before();
      __syncwarp();
      ++seg;
      sb = nsb;
      g0 = ng0;
      g1 = ng1;
      have = nhave;
    }
    if (warp == 0) {
      // Drain: no P V product may still run when TMEM is released.
      const bool leader = elect_one();
      mma_commit(bar(B_DR), leader);
      __syncwarp();
      mbar_wait_drain(bar(B_DR), 0);
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

// One CTA per (sequence, group of 8 heads): merges the partial results of a
// sequence that several CTA pairs shared; writes O = 0, LSE = -inf for an
// empty sequence; leaves sequences written by the split kernel untouched.
// A long sequence in a small batch is spread over up to all CTA pairs, so
// every step is parallel over the pieces: the piece list is built by one
// thread per pair, the weights by one thread per (head, piece) and one warp
// per head, and the weighted sum issues the loads of several pieces at once.
// Two shapes (heads per CTA x pieces in flight): 8 x 2 when the batch gives
// at least two CTAs per SM, 4 x 4 for smaller batches, whose few sequences
// are spread over many pairs (a sweep of 4, 8 and 16 heads with 2 or 4
// pieces: 139.6-141.8 us for the whole decode of a 64-sequence batch, the
// lowest at 8 x 2; 40-55 us for four sequences of 70, 0, 200 and 6000
// tokens, the combine alone 20 us at 4 x 4 and 35 us at 8 x 2 under ncu).
constexpr int COMBINE_THREADS = 256;
constexpr int MAX_PARTS = 128;   // >= CTA pairs, so a sequence never has more pieces
static_assert(MAX_PARTS <= COMBINE_THREADS, "combine thread map");

template <int COMBINE_HEADS, int COMBINE_UNROLL>
__global__ void __launch_bounds__(COMBINE_THREADS)
    decode_combine_kernel(const Args a) {
  // Launched as a programmatic dependent of the split kernel: wait here until
  // that grid has completed and its writes are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int b = blockIdx.x;                 // query unit
  const int orow = unit_row(a, b);          // its row of o and lse
  const int h0 = blockIdx.y * COMBINE_HEADS;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = a.ws_pref[a.B];
  const int s0 = a.ws_pref[b], s1 = a.ws_pref[b + 1];
  if (s1 == s0) {
    for (int i = tid; i < COMBINE_HEADS * DV; i += COMBINE_THREADS)
      a.o[((size_t)orow * HQ + h0) * DV + i] = __float2bfloat16(0.f);
    if (tid < COMBINE_HEADS) a.lse[(size_t)orow * HQ + h0 + tid] = -INFINITY;
    return;
  }
  const int p_lo = pair_of_page(s0, T, a.pairs), p_hi = pair_of_page(s1 - 1, T, a.pairs);
  if (p_lo == p_hi) return;
  __shared__ float w_s[COMBINE_HEADS][MAX_PARTS];
  __shared__ int slot_s[MAX_PARTS];
  __shared__ int wcount_s[COMBINE_THREADS / 32];
  // Pieces in pair order; pairs with an empty range (fewer pages than
  // pairs) hold none.  Thread i looks at pair p_lo + i.
  const int npairs = min(p_hi - p_lo + 1, MAX_PARTS);
  bool has = false;
  int slot = 0;
  if (tid < npairs) {
    const int p = p_lo + tid;
    const int r0 = range_start(p, T, a.pairs);
    has = range_start(p + 1, T, a.pairs) > r0;
    slot = 2 * p + ((p == p_lo && s0 != r0) ? 1 : 0);
  }
  const uint32_t ballot = __ballot_sync(0xffffffffu, has);
  if (lane == 0) wcount_s[warp] = __popc(ballot);
  __syncthreads();
  int before = 0, nparts = 0;
#pragma unroll
  for (int w = 0; w < COMBINE_THREADS / 32; ++w) {
    before += (w < warp) ? wcount_s[w] : 0;
    nparts += wcount_s[w];
  }
  if (has) slot_s[before + __popc(ballot & ((1u << lane) - 1u))] = slot;
  __syncthreads();
  // LSE of every (head, piece), then one warp per head: max, weights, LSE
  for (int i = tid; i < COMBINE_HEADS * nparts; i += COMBINE_THREADS) {
    const int hh = i / nparts, j = i - hh * nparts;
    w_s[hh][j] = a.ws_lse[(size_t)slot_s[j] * HQ + h0 + hh];
  }
  __syncthreads();
  for (int hh = warp; hh < COMBINE_HEADS; hh += COMBINE_THREADS / 32) {
    float mx = -INFINITY;
    for (int j = lane; j < nparts; j += 32) mx = fmaxf(mx, w_s[hh][j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    for (int j = lane; j < nparts; j += 32) {
      const float e = (mx == -INFINITY) ? 0.f : expf(w_s[hh][j] - mx);
      w_s[hh][j] = e;
      sum += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = sum > 0.f ? 1.f / sum : 0.f;
    for (int j = lane; j < nparts; j += 32) w_s[hh][j] *= inv;
    if (lane == 0) a.lse[(size_t)orow * HQ + h0 + hh] = sum > 0.f ? mx + logf(sum) : -INFINITY;
  }
  __syncthreads();
  // COMBINE_HEADS x 512 columns as float4 groups: thread tid owns groups
  // tid + COMBINE_THREADS k (head g / 128, columns 4 (g % 128) ..).
  constexpr int OUT_PER_THREAD = COMBINE_HEADS * DV / 4 / COMBINE_THREADS;
  static_assert(OUT_PER_THREAD * COMBINE_THREADS * 4 == COMBINE_HEADS * DV, "combine output map");
  float4 acc[OUT_PER_THREAD];
  const float* src0[OUT_PER_THREAD];
  int hh_of[OUT_PER_THREAD];
#pragma unroll
  for (int k = 0; k < OUT_PER_THREAD; ++k) {
    const int g = tid + COMBINE_THREADS * k;
    hh_of[k] = g / (DV / 4);
    src0[k] = a.ws_o + ((size_t)h0 + hh_of[k]) * DV + (g % (DV / 4)) * 4;
    acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int j0 = 0; j0 < nparts; j0 += COMBINE_UNROLL) {
    float4 v[COMBINE_UNROLL][OUT_PER_THREAD];
#pragma unroll
    for (int u = 0; u < COMBINE_UNROLL; ++u) {
      const int j = j0 + u;
      const size_t off = (size_t)slot_s[j < nparts ? j : j0] * HQ * DV;
#pragma unroll
      for (int k = 0; k < OUT_PER_THREAD; ++k)
        v[u][k] = j < nparts ? *reinterpret_cast<const float4*>(src0[k] + off) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < COMBINE_UNROLL; ++u) {
      const int j = j0 + u;
      if (j >= nparts) break;
#pragma unroll
      for (int k = 0; k < OUT_PER_THREAD; ++k) {
        const float wgt = w_s[hh_of[k]][j];
        acc[k].x += wgt * v[u][k].x;
        acc[k].y += wgt * v[u][k].y;
        acc[k].z += wgt * v[u][k].z;
        acc[k].w += wgt * v[u][k].w;
      }
    }
  }
#pragma unroll
  for (int k = 0; k < OUT_PER_THREAD; ++k) {
    const int g = tid + COMBINE_THREADS * k;
    __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(a.o + ((size_t)orow * HQ + h0 + hh_of[k]) * DV + (g % (DV / 4)) * 4);
    dst[0] = __floats2bfloat162_rn(acc[k].x, acc[k].y);
    dst[1] = __floats2bfloat162_rn(acc[k].z, acc[k].w);
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

// CTA pairs of the split plan: one per two SMs, at most MAX_PARTS (the
// combine merges up to MAX_PARTS pieces of a sequence).
inline int pairs_for_sms(int sms) { return sms >= 2 ? (sms / 2 < MAX_PARTS ? sms / 2 : MAX_PARTS) : 0; }

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
  a.n_seq = B;
  a.max_pages = max_pages_per_seq;
  a.num_pages = num_pages;
  a.pairs = pairs;
  a.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  decode_split_kernel<<<2 * pairs, THREADS, SMEM_BYTES, s>>>(tq, tkv, a);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  // The combine is a programmatic dependent launch: its CTAs are scheduled as
  // the split kernel's CTAs retire and wait (griddepcontrol.wait) for that
  // grid's completion, instead of the stream's full launch gap.
  // a batch too small to give two 8-head CTAs per SM takes 4 heads per CTA
  const bool small_batch = (long long)units * (HQ / 8) < 4LL * pairs;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(units, HQ / (small_batch ? 4 : 8));
  cfg.blockDim = dim3(COMBINE_THREADS);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = small_batch ? cudaLaunchKernelEx(&cfg, decode_combine_kernel<4, 4>, a)
                                    : cudaLaunchKernelEx(&cfg, decode_combine_kernel<8, 2>, a);
  if (e != cudaSuccess) return ATTN_ERR_CUDA;
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
