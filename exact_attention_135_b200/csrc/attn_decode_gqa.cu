// GQA-path paged decode for sm_100a (B200).
//
// What it computes ("GQLA: Group-Query Latent Attention ...", key terms, GQA
// path: each group of query heads reads its own group-expanded cache;
// "FlashMLA" page: BF16, variable lengths, KV cache paged in 64-token pages;
// "FlashAttention (KO)": online softmax reaches the exact softmax):
//   for each sequence b and query head h, with g = h / (Hq / Hkv),
//   O[b,h] = softmax(scale * q[b,h] . K[b,:,g]) V[b,:,g],  LSE[b,h] = ln sum exp(...)
// over the L_b cached tokens, read through the block table.
//
// The path is memory-bound: per token and KV head it reads 2*D*2 bytes and
// does 4*G*D flops (G = query heads per KV head, <= 8), a few flops per byte.
// So it runs on the CUDA cores (packed f32x2 FMAs), and the design is about
// keeping enough bytes in flight: TMA page tiles staged in shared memory,
// grids sized to the SM count, every HBM byte read once.
//
// Work split: the (sequence, KV head) units are laid end to end, each as its
// ceil(L_b/64) pages, and the resulting page list is cut into one contiguous
// equal range per worker.  A worker is a pair of warps (four pairs per SM,
// two warps per scheduler): it owns a ring of page tiles for one KV head,
// loaded in the order they are used (K of page k, V of page k, K of page
// k+1, ...) and each released as soon as both warps are done with it; the
// first warp issues the TMA loads (lane 0).  Each warp takes 32 of the 64
// tokens of every page for both products; the pair agrees on the row max of
// the page through shared memory and merges its sums and O at the end of a
// unit.  A unit read entirely by one worker is
// written out directly; the pieces of a unit split between workers are
// written as fp32 partials (O normalised by its own sum, plus LSE) and merged
// by the LSE-combine kernel.
//
// Per page (64 tokens) a warp computes, lane = token for the scores (one of
// its 32 tokens per lane) and lane = output dims for the product:
//   s[t][h] = q[h] . k[t]   (q pre-scaled by scale*log2e, fp32 in smem)
//   warp max per head, lazy rescale (only when the max grew by > 2^8),
//   p[t][h] = 2^(s - m) -> smem, O[h][dims of this lane] += sum_t p[t][h] v[t]
#include <math.h>

#include "host_common.h"
#include "sm100.cuh"

namespace ea {
namespace gqa {

constexpr int PAGE = 64;
constexpr int B_MAX = 2048;
constexpr float kRescaleThreshold = 8.0f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D_, int G_>
struct Cfg {
  static constexpr int D = D_;
  static constexpr int G = G_;
  static constexpr int CHUNKS = D / 64;                   // 128-byte column chunks of a row
  static constexpr int CHUNK_BYTES = PAGE * 128;          // one TMA box: 64 tokens x 64 dims
  static constexpr int TILE_BYTES = CHUNKS * CHUNK_BYTES; // K (or V) rows of one page, one KV head
  // Tiles per worker: with three, K of page k+1 and V of page k+1 load while
  // the products of page k run (two tiles in flight per worker).
  static constexpr int TILES = (D == 128) ? 3 : 6;
  static constexpr int Q_BYTES = G * D * 4;               // fp32, pre-scaled by scale*log2e
  static constexpr int P_BYTES = PAGE * G * 4;            // fp32 [token][head]
  static constexpr int X_BYTES = 2 * G * 4;               // row max / sum exchange of a warp pair
  static constexpr int QPX_BYTES = (Q_BYTES + P_BYTES + X_BYTES + 15) / 16 * 16;
  // A worker is a pair of warps sharing one tile ring: four workers fill an
  // SM with two warps per scheduler.
  static constexpr int WORKERS = 4;
  static constexpr int THREADS = 64 * WORKERS;
  static constexpr int DPL = D / 32;                      // output dims per lane
  static constexpr int OFF_QPX = WORKERS * TILES * TILE_BYTES;   // tile rings first (1024-aligned)
  static constexpr int OFF_PREF = OFF_QPX + WORKERS * QPX_BYTES;
  static constexpr int OFF_BAR = (OFF_PREF + (B_MAX + 1) * 4 + 7) / 8 * 8;
  static constexpr int OFF_MISC = OFF_BAR + WORKERS * TILES * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");
};

struct Args {
  const __nv_bfloat16* q;        // [B, Hq, D]
  const int32_t* block_table;    // [B, max_pages]
  const int32_t* seqlens;        // [B]
  __nv_bfloat16* o;              // [B, Hq, D]
  float* lse;                    // [B, Hq]
  int32_t* ws_pref;              // [B + 1]
  float* ws_lse;                 // [2 * workers, G]
  float* ws_o;                   // [2 * workers, G, D]
  int* status;
  int B, Hkv, G, D, max_pages, num_pages, workers;
  float scale_log2;
};

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

// First page of worker w's range: floor(w * T / workers).
__device__ __forceinline__ int range_start(int w, int T, int workers) {
  return (int)(((long long)w * T) / workers);
}

// Worker whose range holds global page x (0 <= x < T).
__device__ __forceinline__ int worker_of_page(int x, int T, int workers) {
  return (int)((((long long)x + 1) * workers - 1) / T);
}

// Walks the units (b, g) that meet [R0, R1), in page-list order.  Unit (b, g)
// covers pages [Hkv*pref[b] + g*n_b, + n_b) with n_b = pref[b+1] - pref[b].
struct UnitWalk {
  const int* pref;
  int B, Hkv, R0, R1, b, g;
  __device__ void init(const int* pref_, int B_, int Hkv_, int R0_, int R1_) {
    pref = pref_;
    B = B_;
    Hkv = Hkv_;
    R0 = R0_;
    R1 = R1_;
    int lo = 0, hi = B;   // last b with Hkv * pref[b] <= R0
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if ((long long)Hkv * pref[mid] <= R0) lo = mid; else hi = mid;
    }
    b = lo;
    g = 0;
  }
  // Next non-empty piece: unit (sb, sg), pages [x0, x1), unit start u0.
  __device__ bool next(int& sb, int& sg, int& x0, int& x1, int& u0) {
    while (b < B) {
      const int base = Hkv * pref[b], np = pref[b + 1] - pref[b];
      if (base >= R1) return false;
      if (np == 0 || g >= Hkv) {
        ++b;
        g = 0;
        continue;
      }
      const int s0 = base + g * np, s1 = s0 + np;
      const int s = max(R0, s0), e = min(R1, s1);
      sb = b;
      sg = g;
      ++g;
      if (e > s) {
        x0 = s;
        x1 = e;
        u0 = s0;
        return true;
      }
    }
    return false;
  }
};

__device__ __forceinline__ void bf16x2_to_f2(uint32_t w, uint64_t& pair) {
  pair = f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    gqa_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const Args a) {
  constexpr int D = C::D, G = C::G, DPL = C::DPL, TILES = C::TILES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  int* pref = reinterpret_cast<int*>(base_ptr + C::OFF_PREF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::OFF_MISC);

  // Let the combine kernel be scheduled as this grid's CTAs retire (it waits
  // for this grid's completion before reading anything).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pw = warp >> 1;     // worker = pair of warps
  const int half = warp & 1;    // this warp's tokens of every page: [32 half, 32 half + 32)
  const uint32_t wbase = base + pw * TILES * C::TILE_BYTES;
  float* q_s = reinterpret_cast<float*>(base_ptr + C::OFF_QPX + pw * C::QPX_BYTES);   // [G][D]
  float* p_s = q_s + G * D;                                                              // [64][G]
  float* x_s = p_s + PAGE * G;                                                           // [2][G]
  auto full_bar = [&](int slot) -> uint32_t { return base + C::OFF_BAR + 8u * (pw * TILES + slot); };
  const int pair_bar = 1 + pw;
  auto pair_sync = [&]() { named_bar_sync(pair_bar, 64); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::WORKERS * TILES; ++i) mbar_init(base + C::OFF_BAR + 8u * i, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // prefix sums of pages per sequence (warp 0; B <= B_MAX)
  if (warp == 0) {
    int carry = 0;
    bool bad = false;
    for (int b0 = 0; b0 < a.B; b0 += 32) {
      const int b = b0 + lane;
      int n = 0;
      if (b < a.B) {
        const int L = a.seqlens[b];
        n = seq_pages(L, a.max_pages);
        bad |= (L < 0) || ((long long)L > (long long)a.max_pages * PAGE);
      }
      int x = n;
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
  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  __syncthreads();
  const int T = a.Hkv * pref[a.B];
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i <= a.B; i += C::THREADS) a.ws_pref[i] = pref[i];
  const int worker = blockIdx.x * C::WORKERS + pw;
  const int R0 = range_start(worker, T, a.workers), R1 = range_start(worker + 1, T, a.workers);
  bool ok = true;

  // ---------------------------------------------------------------- loads
  // Tile n of this worker (n = 2 * page + 0 for K, + 1 for V, pages counted in
  // range order) goes to slot n % TILES, phase n / TILES.  The first warp of
  // the pair walks the range a second time and issues the next tile whenever
  // both warps have released a slot.
  UnitWalk lw;
  lw.init(pref, a.B, a.Hkv, R0, R1);
  int l_b = 0, l_g = 0, l_x = 0, l_x1 = 0, l_u0 = 0;
  bool l_more = lw.next(l_b, l_g, l_x, l_x1, l_u0);
  int tiles = 0;   // tiles issued (meaningful in the first warp)
  auto issue_next = [&]() {
    if (half != 0 || !l_more || !ok) return;
    const int slot = tiles % TILES;
    const bool is_v = tiles & 1;
    if (lane == 0) {
      int page = a.block_table[(size_t)l_b * a.max_pages + (l_x - l_u0)];
      if (page < 0 || page >= a.num_pages) {
        if (!is_v) atomicExch(a.status, (int)ATTN_ERR_INVALID_ARG);
        page = 0;   // never read outside the pool; the result of this sequence is undefined
      }
      // the generic-proxy reads of this slot (an earlier tile) happen before the async-proxy writes
      fence_proxy_async_smem();
      const uint32_t bar = full_bar(slot);
      mbar_arrive_expect_tx(bar, C::TILE_BYTES);
      const uint32_t dst = wbase + slot * C::TILE_BYTES;
#pragma unroll
      for (int c = 0; c < C::CHUNKS; ++c)
        tma_load_3d(dst + c * C::CHUNK_BYTES, is_v ? &tm_v : &tm_k, bar, c * 64, l_g, page * PAGE);
    }
    ++tiles;
    if (is_v && ++l_x == l_x1) l_more = lw.next(l_b, l_g, l_x, l_x1, l_u0);
  };
  for (int i = 0; i < TILES; ++i) issue_next();

  // ---------------------------------------------------------------- compute
  // Both warps of the pair run the same walk and pass the same named barriers
  // in the same order.  After a failed wait a warp keeps walking without
  // touching shared tiles, so the barrier counts stay matched.
  UnitWalk w;
  w.init(pref, a.B, a.Hkv, R0, R1);
  int sb, sg, x0, x1, u0;
  int k = 0;   // pages computed (tiles 2k and 2k + 1)
  const float sl2 = a.scale_log2;
  const int t_mine = 32 * half + lane;   // this lane's token of every page (scores)
  while (w.next(sb, sg, x0, x1, u0)) {
    const int L = seq_len_eff(a.seqlens[sb], a.max_pages);
    const int np = pref[sb + 1] - pref[sb];
    // q of the group's G heads, fp32, pre-scaled; both warps load half of it
    pair_sync();   // the previous unit's reads of q_s and x_s are done
    for (int i = half * 32 + lane; i < G * D / 2; i += 64) {
      const uint32_t wq =
          reinterpret_cast<const uint32_t*>(a.q + ((size_t)sb * (a.Hkv * G) + sg * G) * D)[i];
      q_s[2 * i] = __uint_as_float(wq << 16) * sl2;
      q_s[2 * i + 1] = __uint_as_float(wq & 0xffff0000u) * sl2;
    }
    pair_sync();
    float m_run[G], l_lane[G];
    uint64_t o_acc[2][G][DPL / 2];   // two sets (even and odd tokens)
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m_run[h] = -INFINITY;
      l_lane[h] = 0.f;
#pragma unroll
      for (int j = 0; j < DPL / 2; ++j) o_acc[0][h][j] = o_acc[1][h][j] = f2_pack(0.f, 0.f);
    }
    for (int x = x0; x < x1; ++x, ++k) {
      const int nk = 2 * k, nv = 2 * k + 1;
      const uint32_t kt = wbase + (nk % TILES) * C::TILE_BYTES;
      const uint32_t vt = wbase + (nv % TILES) * C::TILE_BYTES;
      const int valid = L - (x - u0) * PAGE;   // tokens of this page inside the sequence (>= 1)
      if (ok) ok = warp_wait(full_bar(nk % TILES), (nk / TILES) & 1, abort_flag, a.status);

      // ---- scores of this lane's token against the G heads
      float s[G];
      if (ok) {
        uint64_t acc[2][G];
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
          for (int h = 0; h < G; ++h) acc[e][h] = f2_pack(0.f, 0.f);
        const int t = t_mine;
#pragma unroll 4
        for (int c = 0; c < D / 8; ++c) {
          const int cc = c >> 3, jj = c & 7;
          uint32_t k0, k1, k2, k3;
          ld_shared_v4(kt + cc * C::CHUNK_BYTES + t * 128 + ((jj ^ (t & 7)) << 4), k0, k1, k2, k3);
          uint64_t kp[4];
          bf16x2_to_f2(k0, kp[0]);
          bf16x2_to_f2(k1, kp[1]);
          bf16x2_to_f2(k2, kp[2]);
          bf16x2_to_f2(k3, kp[3]);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float4 q0 = *reinterpret_cast<const float4*>(q_s + h * D + c * 8);
            const float4 q1 = *reinterpret_cast<const float4*>(q_s + h * D + c * 8 + 4);
            acc[c & 1][h] = f2_fma(kp[0], f2_pack(q0.x, q0.y), acc[c & 1][h]);
            acc[c & 1][h] = f2_fma(kp[1], f2_pack(q0.z, q0.w), acc[c & 1][h]);
            acc[c & 1][h] = f2_fma(kp[2], f2_pack(q1.x, q1.y), acc[c & 1][h]);
            acc[c & 1][h] = f2_fma(kp[3], f2_pack(q1.z, q1.w), acc[c & 1][h]);
          }
        }
        const bool live = t < valid;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float lo, hi;
          f2_unpack(f2_add(acc[0][h], acc[1][h]), lo, hi);
          s[h] = live ? lo + hi : -INFINITY;
        }
        // this warp's max per head
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float mx = s[h];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          if (lane == 0) x_s[half * G + h] = mx;
        }
      }
      pair_sync();    // both warps are done with the K tile and have posted their maxima
      issue_next();   // refill the K tile's slot

      // ---- online softmax over the page (m, the rescale decision and alpha
      // are identical in both warps: the same two maxima, the same order)
      if (ok) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float mx = fmaxf(x_s[h], x_s[G + h]);
          const float m_new = fmaxf(m_run[h], mx);
          const bool grow = m_new > m_run[h] + kRescaleThreshold;
          const float m_use = grow ? m_new : m_run[h];
          const float m_eff = (m_use == -INFINITY) ? 0.f : m_use;
          const float p = ex2(s[h] - m_eff);
          if (grow) {
            const float alpha = ex2(m_run[h] - m_use);
            l_lane[h] *= alpha;
#pragma unroll
            for (int j = 0; j < DPL / 2; ++j) {
              o_acc[0][h][j] = f2_mul(o_acc[0][h][j], f2_pack(alpha, alpha));
              o_acc[1][h][j] = f2_mul(o_acc[1][h][j], f2_pack(alpha, alpha));
            }
          }
          l_lane[h] += p;
          m_run[h] = m_use;
          s[h] = p;
        }
        float* dst = p_s + t_mine * G;
        if constexpr (G >= 4) {
#pragma unroll
          for (int h = 0; h < G; h += 4) *reinterpret_cast<float4*>(dst + h) = make_float4(s[h], s[h + 1], s[h + 2], s[h + 3]);
        } else if constexpr (G == 2) {
          *reinterpret_cast<float2*>(dst) = make_float2(s[0], s[1]);
        } else {
          dst[0] = s[0];
        }
        __syncwarp();
        ok = warp_wait(full_bar(nv % TILES), (nv / TILES) & 1, abort_flag, a.status);
      }

      // ---- O += P V over this warp's 32 tokens, lane = output dims
      if (ok) {
        const int dim0 = DPL * lane;
        const int cc = dim0 >> 6;                 // column chunk
        const int byte_in_row = (dim0 & 63) * 2;  // within the 128-byte row
        const int unit = byte_in_row >> 4, in_unit = byte_in_row & 15;
#pragma unroll 4
        for (int tt = 0; tt < 32; ++tt) {
          const int t = 32 * half + tt;
          const uint32_t addr = vt + cc * C::CHUNK_BYTES + t * 128 + ((unit ^ (t & 7)) << 4) + in_unit;
          uint64_t vp[DPL / 2];
          if constexpr (DPL == 4) {
            uint32_t v0, v1;
            asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v0), "=r"(v1) : "r"(addr));
            bf16x2_to_f2(v0, vp[0]);
            bf16x2_to_f2(v1, vp[1]);
          } else {
            uint32_t v0;
            asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v0) : "r"(addr));
            bf16x2_to_f2(v0, vp[0]);
          }
          float pv[G];
          const float* src = p_s + t * G;
          if constexpr (G >= 4) {
#pragma unroll
            for (int h = 0; h < G; h += 4) {
              const float4 f = *reinterpret_cast<const float4*>(src + h);
              pv[h] = f.x;
              pv[h + 1] = f.y;
              pv[h + 2] = f.z;
              pv[h + 3] = f.w;
            }
          } else if constexpr (G == 2) {
            const float2 f = *reinterpret_cast<const float2*>(src);
            pv[0] = f.x;
            pv[1] = f.y;
          } else {
            pv[0] = src[0];
          }
#pragma unroll
          for (int h = 0; h < G; ++h)
#pragma unroll
            for (int j = 0; j < DPL / 2; ++j)
              o_acc[tt & 1][h][j] = f2_fma(vp[j], f2_pack(pv[h], pv[h]), o_acc[tt & 1][h][j]);
        }
      }
      pair_sync();    // both warps are done with the V tile (and with this page's maxima)
      issue_next();   // refill the V tile's slot
    }

    // ---- unit piece done: the second warp hands its sums and O to the first
    float l_w[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float l = l_lane[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      l_w[h] = l;
    }
    if (half == 1 && ok) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        if (lane == 0) x_s[h] = l_w[h];
#pragma unroll
        for (int j = 0; j < DPL / 2; ++j) {
          float lo, hi;
          f2_unpack(f2_add(o_acc[0][h][j], o_acc[1][h][j]), lo, hi);
          q_s[h * D + DPL * lane + 2 * j] = lo;       // q is no longer needed for this unit
          q_s[h * D + DPL * lane + 2 * j + 1] = hi;
        }
      }
    }
    pair_sync();
    if (half == 0 && ok && !*abort_flag) {
      const bool complete = (x0 == u0) && (x1 == u0 + np);
      const int slot = 2 * worker + (x0 == R0 ? 0 : 1);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float l = l_w[h] + x_s[h];
        const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
        const float lse = (l > 0.f) ? (m_run[h] + log2f(l)) * kLn2 : -INFINITY;
        float ov[DPL];
#pragma unroll
        for (int j = 0; j < DPL / 2; ++j) {
          f2_unpack(f2_add(o_acc[0][h][j], o_acc[1][h][j]), ov[2 * j], ov[2 * j + 1]);
          ov[2 * j] = (ov[2 * j] + q_s[h * D + DPL * lane + 2 * j]) * inv_l;
          ov[2 * j + 1] = (ov[2 * j + 1] + q_s[h * D + DPL * lane + 2 * j + 1]) * inv_l;
        }
        const int head = sg * G + h;
        if (complete) {
          __nv_bfloat16* dst = a.o + ((size_t)sb * (a.Hkv * G) + head) * D + DPL * lane;
          if constexpr (DPL == 4) {
            uint2 u;
            u.x = pack_bf16x2(ov[0], ov[1]);
            u.y = pack_bf16x2(ov[2], ov[3]);
            *reinterpret_cast<uint2*>(dst) = u;
          } else {
            *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(ov[0], ov[1]);
          }
          if (lane == 0) a.lse[(size_t)sb * (a.Hkv * G) + head] = lse;
        } else {
          float* dst = a.ws_o + ((size_t)slot * G + h) * D + DPL * lane;
          if constexpr (DPL == 4) {
            *reinterpret_cast<float4*>(dst) = make_float4(ov[0], ov[1], ov[2], ov[3]);
          } else {
            *reinterpret_cast<float2*>(dst) = make_float2(ov[0], ov[1]);
          }
          if (lane == 0) a.ws_lse[(size_t)slot * G + h] = lse;
        }
      }
    }
  }
  // Drain: every issued load must land before the CTA's shared memory goes away.
  if (half == 0 && lane == 0)
    for (int n = max(0, tiles - TILES); n < tiles; ++n) mbar_wait_drain(full_bar(n % TILES), (n / TILES) & 1);
  __syncwarp();
}

// One CTA per (sequence, KV head): merges the partial results of a unit that
// several workers shared, writes O = 0 and LSE = -inf for an empty sequence,
// leaves units written by the decode kernel untouched.  The number of pieces
// is not bounded: workers are taken in chunks of COMBINE_CHUNK, and each
// chunk's pieces, slots and weights are compacted into shared memory once, so
// the loop over output elements only reads them.
constexpr int COMBINE_THREADS = 128;
constexpr int COMBINE_CHUNK = 128;
constexpr int COMBINE_OUT = 8;   // output elements per thread: G * D <= 8 * 128

__global__ void __launch_bounds__(COMBINE_THREADS) gqa_combine_kernel(const Args a) {
  // Launched as a programmatic dependent of the decode kernel: wait here until
  // that grid has completed and its writes are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int b = blockIdx.x, g = blockIdx.y;
  const int G = a.G, D = a.D, Hq = a.Hkv * G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = a.Hkv * a.ws_pref[a.B];
  const int np = a.ws_pref[b + 1] - a.ws_pref[b];
  if (np == 0) {
    for (int i = tid; i < G * D; i += COMBINE_THREADS)
      a.o[((size_t)b * Hq + g * G) * D + i] = __float2bfloat16(0.f);
    if (tid < G) a.lse[(size_t)b * Hq + g * G + tid] = -INFINITY;
    return;
  }
  const int u0 = a.Hkv * a.ws_pref[b] + g * np, u1 = u0 + np;
  const int w_lo = worker_of_page(u0, T, a.workers), w_hi = worker_of_page(u1 - 1, T, a.workers);
  if (w_lo == w_hi) return;
  const int n = w_hi - w_lo + 1;
  // slot of worker w's piece of this unit (workers with empty ranges hold none)
  auto slot_of = [&](int w) -> int {
    const int r0 = range_start(w, T, a.workers);
    if (range_start(w + 1, T, a.workers) == r0) return -1;
    return 2 * w + ((w == w_lo && u0 != r0) ? 1 : 0);
  };
  __shared__ float s_red[COMBINE_THREADS / 32][8];
  __shared__ float s_max[8], s_inv[8];
  __shared__ int s_slot[COMBINE_CHUNK];
  __shared__ int s_cnt[COMBINE_THREADS / 32];
  __shared__ float s_w[8][COMBINE_CHUNK];

  // per-head maximum, then sum of exp(lse - max), over all pieces (in parallel over pieces)
  for (int pass = 0; pass < 2; ++pass) {
    float acc[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) acc[h] = pass == 0 ? -INFINITY : 0.f;
    for (int i = tid; i < n; i += COMBINE_THREADS) {
      const int sl = slot_of(w_lo + i);
      if (sl < 0) continue;
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        if (h >= G) break;
        const float l = a.ws_lse[(size_t)sl * G + h];
        if (pass == 0) acc[h] = fmaxf(acc[h], l);
        else if (s_max[h] != -INFINITY) acc[h] += expf(l - s_max[h]);
      }
    }
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      float v = acc[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float y = __shfl_xor_sync(0xffffffffu, v, o);
        v = pass == 0 ? fmaxf(v, y) : v + y;
      }
      if (lane == 0) s_red[warp][h] = v;
    }
    __syncthreads();
    if (tid < G) {
      float v = s_red[0][tid];
      for (int w = 1; w < COMBINE_THREADS / 32; ++w) v = pass == 0 ? fmaxf(v, s_red[w][tid]) : v + s_red[w][tid];
      if (pass == 0) {
        s_max[tid] = v;
      } else {
        s_inv[tid] = v > 0.f ? 1.f / v : 0.f;
        a.lse[(size_t)b * Hq + g * G + tid] = v > 0.f ? s_max[tid] + logf(v) : -INFINITY;
      }
    }
    __syncthreads();
  }

  // O = sum over pieces of weight * partial O, one chunk of workers at a
  // time: the chunk's pieces are first compacted (most workers of a short
  // sequence in a small batch hold none), then the loads of two pieces for
  // all of a thread's outputs are issued together.
  float out[COMBINE_OUT];
#pragma unroll
  for (int k = 0; k < COMBINE_OUT; ++k) out[k] = 0.f;
  for (int c0 = 0; c0 < n; c0 += COMBINE_CHUNK) {
    const int cn = min(COMBINE_CHUNK, n - c0);
    const int sl = tid < cn ? slot_of(w_lo + c0 + tid) : -1;
    const uint32_t ballot = __ballot_sync(0xffffffffu, sl >= 0);
    if (lane == 0) s_cnt[warp] = __popc(ballot);
    __syncthreads();
    int before = 0, m = 0;
#pragma unroll
    for (int w = 0; w < COMBINE_THREADS / 32; ++w) {
      before += (w < warp) ? s_cnt[w] : 0;
      m += s_cnt[w];
    }
    if (sl >= 0) {
      const int pos = before + __popc(ballot & ((1u << lane) - 1u));
      s_slot[pos] = sl;
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        if (h >= G) break;
        s_w[h][pos] = s_max[h] == -INFINITY ? 0.f : expf(a.ws_lse[(size_t)sl * G + h] - s_max[h]) * s_inv[h];
      }
    }
    __syncthreads();
    for (int j0 = 0; j0 < m; j0 += 2) {
      const bool two = j0 + 1 < m;
      const int j1 = two ? j0 + 1 : j0;   // v1 is 0 when there is no second piece
      const float* src0 = a.ws_o + (size_t)s_slot[j0] * G * D;
      const float* src1 = a.ws_o + (size_t)s_slot[j1] * G * D;
      float v0[COMBINE_OUT], v1[COMBINE_OUT];
#pragma unroll
      for (int k = 0; k < COMBINE_OUT; ++k) {
        const int i = tid + k * COMBINE_THREADS;
        const bool in = i < G * D;
        v0[k] = in ? src0[i] : 0.f;
        v1[k] = (in && two) ? src1[i] : 0.f;
      }
#pragma unroll
      for (int k = 0; k < COMBINE_OUT; ++k) {
        const int i = tid + k * COMBINE_THREADS;
        if (i < G * D) {
          const int h = i / D;
          out[k] += s_w[h][j0] * v0[k] + s_w[h][j1] * v1[k];
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int k = 0; k < COMBINE_OUT; ++k) {
    const int i = tid + k * COMBINE_THREADS;
    if (i >= G * D) break;
    a.o[((size_t)b * Hq + g * G) * D + i] = __float2bfloat16(out[k]);
  }
}

struct WsLayout {
  size_t off_pref, off_lse, off_o, total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline int workers_per_cta(int D) { return D == 128 ? Cfg<128, 1>::WORKERS : Cfg<64, 1>::WORKERS; }

inline WsLayout ws_layout(int B, int G, int D, int workers) {
  WsLayout w;
  w.off_pref = 0;
  w.off_lse = align256((size_t)(B + 1) * 4);
  w.off_o = w.off_lse + align256((size_t)2 * workers * G * 4);
  w.total = w.off_o + (size_t)2 * workers * G * D * 4;
  return w;
}

template <int D, int G>
int launch(const CUtensorMap& tk, const CUtensorMap& tv, const Args& a, int ctas, cudaStream_t s) {
  using C = Cfg<D, G>;
  static int attr_done = 0;
  const void* kfn = reinterpret_cast<const void*>(&gqa_decode_kernel<C>);
  if (int rc = ensure_smem_attr(kfn, C::SMEM_BYTES, &attr_done)) return rc;
  gqa_decode_kernel<C><<<ctas, C::THREADS, C::SMEM_BYTES, s>>>(tk, tv, a);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace gqa
}  // namespace ea

extern "C" size_t attn_decode_paged_gqa_workspace_size(int B, int Hq, int Hkv, int D, int device) {
  using namespace ea;
  using namespace ea::gqa;
  if (B < 1 || B > B_MAX || Hkv < 1 || Hq < 1 || Hq % Hkv != 0 || (D != 64 && D != 128)) return 0;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return 0;
  const int sms = sm_count_of(device);
  if (sms < 1) return 0;
  return ws_layout(B, G, D, sms * workers_per_cta(D)).total;
}

extern "C" int attn_decode_paged_gqa(const void* q, const void* k_pages, const void* v_pages,
                                     const int32_t* block_table, const int32_t* cache_seqlens, void* o, float* lse,
                                     int B, int Hq, int Hkv, int D, int page_size, int num_pages,
                                     int max_pages_per_seq, float scale, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  using namespace ea;
  using namespace ea::gqa;
  if (!q || !k_pages || !v_pages || !block_table || !cache_seqlens || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_pages, 16) || !aligned(v_pages, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(block_table, 4) || !aligned(cache_seqlens, 4))
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || num_pages < 1 || max_pages_per_seq < 1 || page_size < 1 || D < 1)
    return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if ((D != 64 && D != 128) || (G != 1 && G != 2 && G != 4 && G != 8) || page_size != PAGE || B > B_MAX)
    return ATTN_ERR_UNSUPPORTED;
  if ((long long)num_pages * PAGE * Hkv * D >= (1ll << 40) || (long long)B * max_pages_per_seq >= (1ll << 31) ||
      (long long)num_pages * PAGE >= (1ll << 31) || (long long)Hkv * B * max_pages_per_seq >= (1ll << 31))
    return ATTN_ERR_UNSUPPORTED;
  const int sms = current_sm_count();
  if (sms < 1) return ATTN_ERR_CUDA;
  const int workers = sms * workers_per_cta(D);
  const WsLayout wl = ws_layout(B, G, D, workers);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < wl.total) return ATTN_ERR_WORKSPACE;
  int* status = device_status_ptr();
  if (!status) return ATTN_ERR_CUDA;

  CUtensorMap tk, tv;
  {
    // [num_pages * 64 tokens][Hkv][D]: one box = 64 dims x 1 KV head x 64 tokens
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)Hkv, (uint64_t)num_pages * PAGE};
    const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)Hkv * D * 2};
    const uint32_t box[3] = {64, 1, (uint32_t)PAGE};
    if (!encode_bf16_3d(&tk, k_pages, dims, strides, box)) return ATTN_ERR_CUDA;
    if (!encode_bf16_3d(&tv, v_pages, dims, strides, box)) return ATTN_ERR_CUDA;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  Args a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.block_table = block_table;
  a.seqlens = cache_seqlens;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.ws_pref = reinterpret_cast<int32_t*>(ws + wl.off_pref);
  a.ws_lse = reinterpret_cast<float*>(ws + wl.off_lse);
  a.ws_o = reinterpret_cast<float*>(ws + wl.off_o);
  a.status = status;
  a.B = B;
  a.Hkv = Hkv;
  a.G = G;
  a.D = D;
  a.max_pages = max_pages_per_seq;
  a.num_pages = num_pages;
  a.workers = workers;
  a.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int rc;
  if (D == 128) {
    rc = G == 1 ? launch<128, 1>(tk, tv, a, sms, s)
       : G == 2 ? launch<128, 2>(tk, tv, a, sms, s)
       : G == 4 ? launch<128, 4>(tk, tv, a, sms, s)
                : launch<128, 8>(tk, tv, a, sms, s);
  } else {
    rc = G == 1 ? launch<64, 1>(tk, tv, a, sms, s)
       : G == 2 ? launch<64, 2>(tk, tv, a, sms, s)
       : G == 4 ? launch<64, 4>(tk, tv, a, sms, s)
                : launch<64, 8>(tk, tv, a, sms, s);
  }
  if (rc != ATTN_OK) return rc;
  // a programmatic dependent launch, like the MLA decode's combine
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(B, Hkv);
  cfg.blockDim = dim3(COMBINE_THREADS);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, gqa_combine_kernel, a) != cudaSuccess) return ATTN_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}
