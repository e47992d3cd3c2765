// Per-row softmax pieces shared by the prefill and decode kernels.  One
// thread owns one query row (one TMEM lane) and holds N raw fp32 scores of
// it in registers.
#pragma once

#include "sm100.cuh"

namespace ea {

// Max of the N raw scores of one row (four independent three-input chains).
template <int N>
__device__ __forceinline__ float row_max(const uint32_t* s) {
  float m0 = __uint_as_float(s[0]), m1 = __uint_as_float(s[1]);
  float m2 = __uint_as_float(s[2]), m3 = __uint_as_float(s[3]);
#pragma unroll
  for (int c = 4; c + 8 <= N; c += 8) {
    m0 = max3f(m0, __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
    m1 = max3f(m1, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
    m2 = max3f(m2, __uint_as_float(s[c + 4]), __uint_as_float(s[c + 5]));
    m3 = max3f(m3, __uint_as_float(s[c + 6]), __uint_as_float(s[c + 7]));
  }
  m0 = max3f(m0, __uint_as_float(s[N - 4]), __uint_as_float(s[N - 3]));
  m1 = max3f(m1, __uint_as_float(s[N - 2]), __uint_as_float(s[N - 1]));
  return fmaxf(max3f(m0, m1, m2), m3);
}

// Pairs of columns whose exp2 runs on the FMA pipe in full blocks: pairs
// with (c mod 16) >= T, 5 of every 16 by default, which balances the MUFU
// unit against the issue slots the polynomial costs.
__device__ __forceinline__ constexpr bool poly_pair(int c, int T = 11) { return (c & 15) >= T; }

// p = 2^(s * sl2 - m) for one row, packed to bf16 pairs; returns the fp32 sum.
template <int N, bool MIXED, int POLY_T = 11>
__device__ __forceinline__ float exp_row(const uint32_t* s, uint32_t* p, float sl2, float m) {
  const uint64_t k2 = f2_pack(sl2, sl2);
  const uint64_t nm2 = f2_pack(-m, -m);
  uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = acc0;
#pragma unroll
  for (int c = 0; c < N / 2; ++c) {
    const uint64_t x = f2_fma(f2_pack(__uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1])), k2, nm2);
    float p0, p1;
    if (MIXED && poly_pair(c, POLY_T)) {
      exp2_poly_x2(x, p0, p1);
    } else {
      float x0, x1;
      f2_unpack(x, x0, x1);
      p0 = ex2(x0);
      p1 = ex2(x1);
    }
    if (c & 1) acc1 = f2_add(acc1, f2_pack(p0, p1));
    else acc0 = f2_add(acc0, f2_pack(p0, p1));
    p[c] = pack_bf16x2(p0, p1);
  }
  float a0, a1, b0, b1;
  f2_unpack(acc0, a0, a1);
  f2_unpack(acc1, b0, b1);
  return (a0 + b0) + (a1 + b1);
}

// The same with p packed four to a word as e4m3 bytes (column 4w + i in
// byte i of word w), the layout of an 8-bit A operand in tensor memory.
template <int N, bool MIXED, int POLY_T = 11>
__device__ __forceinline__ float exp_row_e4m3(const uint32_t* s, uint32_t* p, float sl2, float m) {
  const uint64_t k2 = f2_pack(sl2, sl2);
  const uint64_t nm2 = f2_pack(-m, -m);
  uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = acc0;
#pragma unroll
  for (int c = 0; c < N / 2; ++c) {
    const uint64_t x = f2_fma(f2_pack(__uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1])), k2, nm2);
    float p0, p1;
    if (MIXED && poly_pair(c, POLY_T)) {
      exp2_poly_x2(x, p0, p1);
    } else {
      float x0, x1;
      f2_unpack(x, x0, x1);
      p0 = ex2(x0);
      p1 = ex2(x1);
    }
    if (c & 1) acc1 = f2_add(acc1, f2_pack(p0, p1));
    else acc0 = f2_add(acc0, f2_pack(p0, p1));
    const uint32_t pair = pack_e4m3x2(p0, p1);
    if (c & 1) p[c / 2] |= pair << 16;
    else p[c / 2] = pair;
  }
  float a0, a1, b0, b1;
  f2_unpack(acc0, a0, a1);
  f2_unpack(acc1, b0, b1);
  return (a0 + b0) + (a1 + b1);
}

}  // namespace ea
