// Row-softmax building blocks for one thread holding one 128-column row of S:
// a 3-input max tree, packed fp32x2 arithmetic, and 2^x split between the
// MUFU unit (ex2.approx) and a polynomial on the FMA pipe, so that neither
// unit alone limits the softmax while the tensor core runs the other tile.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

#ifndef CALIBATT_PACKED_F32X2
#define CALIBATT_PACKED_F32X2 1
#endif

namespace calibatt {

// fp32x2 arithmetic: one packed instruction on sm_100 (or two scalar ones).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
#if CALIBATT_PACKED_F32X2
  return __ffma2_rn(a, b, c);
#else
  return make_float2(__fmaf_rn(a.x, b.x, c.x), __fmaf_rn(a.y, b.y, c.y));
#endif
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
#if CALIBATT_PACKED_F32X2
  return __fadd2_rn(a, b);
#else
  return make_float2(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y));
#endif
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// max over 128 values: 8 independent chains of 3-input maxima, then a tree.
__device__ __forceinline__ float row_max128(const float (&s)[128]) {
  float a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = s[i];
#pragma unroll
  for (int k = 8; k < 128; k += 16) {
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = max3f(a[i], s[k + i], s[k + 8 + i]);
  }
  return fmaxf(max3f(a[0], a[1], a[2]), fmaxf(max3f(a[3], a[4], a[5]), max3f(a[6], a[7], a[7])));
}

// 2^x for a pair, on the FMA pipe (Cody-Waite additive range reduction with
// round-to-nearest: x = n + f, |f| <= 1/2; 2^f by a minimax polynomial; n
// added to the exponent field). Inputs below -120 are clamped (2^-120 is
// below anything the softmax sums can resolve). Coefficients: Remez exchange
// for the relative error on [-1/2, 1/2] (see gen_exp2_poly.py): degree 3 has
// max relative error 7.5e-5, degree 5 2.3e-7 (fp32 Horner).
__device__ __forceinline__ uint32_t exp_insert(uint32_t t, uint32_t p) {
  uint32_t r;
  asm("mad.lo.u32 %0, %1, 8388608, %2;" : "=r"(r) : "r"(t), "r"(p));
  return r;
}

template <int DEG>
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: adding it rounds to an integer
  x.x = fmaxf(x.x, -120.f);
  x.y = fmaxf(x.y, -120.f);
  const float2 t = fadd2(x, make_float2(kMagic, kMagic));
  const float2 n = fadd2(t, make_float2(-kMagic, -kMagic));
  const float2 f = ffma2(n, make_float2(-1.f, -1.f), x);
  float2 p;
  if (DEG == 3) {
    p = make_float2(5.517166853e-02f, 5.517166853e-02f);
    p = ffma2(p, f, make_float2(2.426111251e-01f, 2.426111251e-01f));
    p = ffma2(p, f, make_float2(6.932609677e-01f, 6.932609677e-01f));
    p = ffma2(p, f, make_float2(9.999280572e-01f, 9.999280572e-01f));
  } else {
    p = make_float2(1.327647245e-03f, 1.327647245e-03f);
    p = ffma2(p, f, make_float2(9.675540961e-03f, 9.675540961e-03f));
    p = ffma2(p, f, make_float2(5.550713092e-02f, 5.550713092e-02f));
    p = ffma2(p, f, make_float2(2.402212024e-01f, 2.402212024e-01f));
    p = ffma2(p, f, make_float2(6.931469440e-01f, 6.931469440e-01f));
    p = ffma2(p, f, make_float2(1.000000119e+00f, 1.000000119e+00f));
  }
  // low bits of t hold n (two's complement); n * 2^23 + bits(p) puts it in the
  // exponent field with one integer multiply-add
  p.x = __uint_as_float(exp_insert(__float_as_uint(t.x), __float_as_uint(p.x)));
  p.y = __uint_as_float(exp_insert(__float_as_uint(t.y), __float_as_uint(p.y)));
  return p;
}

__device__ __forceinline__ float2 exp2_mufu2(float2 x) {
  float2 r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r.x) : "f"(x.x));
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r.y) : "f"(x.y));
  return r;
}

// Pair i of a row goes to the FMA pipe when EmuMask has bit (i % 8) set.
template <int DEG, unsigned EmuMask>
__device__ __forceinline__ float2 exp2_pair(int i, float2 x) {
  return ((EmuMask >> (i & 7)) & 1u) ? exp2_poly2<DEG>(x) : exp2_mufu2(x);
}

__device__ __forceinline__ uint32_t pack_bf16x2f(float2 v) {
  __nv_bfloat162 b = __float22bfloat162_rn(v);
  return *reinterpret_cast<uint32_t*>(&b);
}

}  // namespace calibatt
