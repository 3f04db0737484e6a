// bimath.cuh -- the library's own exp and log for log_softmax.
//
// CUDA's expf/logf (and any vendor math library) are not correctly rounded
// and their bits cannot be reproduced elsewhere.  A batch-invariant
// log_softmax needs exp/log whose every operation is fixed, so that the
// result is the same bits on any IEEE-754 machine that follows the method.
// These are textbook methods written out here:
//
// bi_exp(x): Cody-Waite reduction.  n = rint(x * log2 e) (nearest, ties to
//   even); r = x - n*ln2 with ln2 split into a head (ln2 with its low 8
//   mantissa bits cleared, 0x3f317200) and a tail (ln2 - head, rounded to
//   fp32), each subtracted with one fused multiply-add; e^r by its Taylor
//   series through r^7 in Horner form with fused multiply-adds (coefficients
//   1/k! rounded to fp32); the result is scaled by 2^n built from exponent
//   bits (exact, in two steps below 2^-126).  x < -103 returns +0.
// bi_log(x), x > 0 normal: x = 2^e * m with m in [sqrt(1/2), sqrt(2));
//   f = (m-1)/(m+1); log m = 2f + 2f * f^2 * (1/3 + f^2/5 + f^4/7 + f^6/9)
//   (bracket in Horner form, coefficients 1/(2k+1) rounded to fp32, the
//   leading 2f added by a final fused multiply-add);
//   log x = fma(e, ln2_head, fma(e, ln2_tail, log m)).
#pragma once

#include "common.cuh"

namespace bi {

BI_DEV float pow2_exact(int n) { return __uint_as_float((unsigned)(n + 127) << 23); }

BI_DEV float bi_exp(float x) {
  const float log2e = (float)1.4426950408889634074;
  const float ln2_head = 0.693145751953125f;
  const float ln2_tail = (float)(0.693147180559945309417 - 0.693145751953125);
  if (x < -103.0f) return 0.0f;
  const float n = rintf(__fmul_rn(x, log2e));
  float r = __fmaf_rn(-n, ln2_head, x);
  r = __fmaf_rn(-n, ln2_tail, r);
  float p = (float)(1.0 / 5040.0);
  p = __fmaf_rn(p, r, (float)(1.0 / 720.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 120.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 24.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 6.0));
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const int ni = (int)n;
  if (ni > 127) return __fmul_rn(__fmul_rn(p, pow2_exact(ni - 1)), 2.0f);
  if (ni < -126) return __fmul_rn(__fmul_rn(p, pow2_exact(ni + 100)), pow2_exact(-100));
  return __fmul_rn(p, pow2_exact(ni));
}

// bi_exp for -87 <= x <= 88: the same operations and the same bits as
// bi_exp there, with the rounding to an integer done by adding and
// subtracting 1.5 * 2^23 (nearest, ties to even -- what rint does for
// |t| < 2^22) and the integer read from the sum's low bits; the scale 2^n is
// a normal number over the whole range, so the result is one multiply.
BI_DEV float bi_exp_fast(float x) {
  const float log2e = (float)1.4426950408889634074;
  const float ln2_head = 0.693145751953125f;
  const float ln2_tail = (float)(0.693147180559945309417 - 0.693145751953125);
  const float magic = 12582912.0f;                    // 1.5 * 2^23
  const float sh = __fadd_rn(__fmul_rn(x, log2e), magic);
  const float n = __fsub_rn(sh, magic);
  const int ni = __float_as_int(sh) - __float_as_int(magic);
  float r = __fmaf_rn(-n, ln2_head, x);
  r = __fmaf_rn(-n, ln2_tail, r);
  float p = (float)(1.0 / 5040.0);
  p = __fmaf_rn(p, r, (float)(1.0 / 720.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 120.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 24.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 6.0));
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  return __fmul_rn(p, __int_as_float((ni + 127) << 23));
}

// Two lanes at once: sm_100's packed fp32 instructions (sub/mul/fma
// .rn.f32x2) round each lane exactly as the scalar instruction does, so
// bi_exp_fast2 gives bi_exp_fast's bits for both lanes in about half the
// issued instructions.  fma(-n, c, r) is computed as fma(n, -c, r): the
// product is the same exact value, so the rounding is the same.
BI_DEV uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
BI_DEV float2 upk2(uint64_t r) {
  float2 v;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
  return v;
}
BI_DEV uint64_t fma2_rn(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
BI_DEV uint64_t sub2_rn(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
BI_DEV uint64_t mul2_rn(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
BI_DEV uint64_t splat2(float a) { return pk2(a, a); }

// bi_exp_fast on both lanes of x; both must lie in [-87, 88].  The
// rounding to an integer stays on scalar instructions: a packed multiply
// followed by a packed add was measured to round once, like a fused
// multiply-add (x = -81.4447937: x * log2 e rounds to the tie -117.5, which
// must then round to -118), so the packed forms start at n.
BI_DEV uint64_t bi_exp_fast2(uint64_t x) {
  const float magic = 12582912.0f;                    // 1.5 * 2^23
  const float log2e = (float)1.4426950408889634074;
  const float2 xv = upk2(x);
  const uint64_t sh = pk2(__fadd_rn(__fmul_rn(xv.x, log2e), magic), __fadd_rn(__fmul_rn(xv.y, log2e), magic));
  const uint64_t n = sub2_rn(sh, splat2(magic));
  uint64_t r = fma2_rn(n, splat2(-0.693145751953125f), x);
  r = fma2_rn(n, splat2(-(float)(0.693147180559945309417 - 0.693145751953125)), r);
  uint64_t p = splat2((float)(1.0 / 5040.0));
  p = fma2_rn(p, r, splat2((float)(1.0 / 720.0)));
  p = fma2_rn(p, r, splat2((float)(1.0 / 120.0)));
  p = fma2_rn(p, r, splat2((float)(1.0 / 24.0)));
  p = fma2_rn(p, r, splat2((float)(1.0 / 6.0)));
  p = fma2_rn(p, r, splat2(0.5f));
  p = fma2_rn(p, r, splat2(1.0f));
  p = fma2_rn(p, r, splat2(1.0f));
  const float2 s = upk2(sh);
  const int na = __float_as_int(s.x) - __float_as_int(magic);
  const int nb = __float_as_int(s.y) - __float_as_int(magic);
  return mul2_rn(p, pk2(__int_as_float((na + 127) << 23), __int_as_float((nb + 127) << 23)));
}

BI_DEV float bi_log(float x) {
  const float ln2_head = 0.693145751953125f;
  const float ln2_tail = (float)(0.693147180559945309417 - 0.693145751953125);
  const float sqrt2 = (float)1.4142135623730950488;
  const unsigned b = __float_as_uint(x);
  int e = (int)((b >> 23) & 0xffu) - 127;
  float m = __uint_as_float((b & 0x007fffffu) | 0x3f800000u);
  if (m > sqrt2) {
    m = __fmul_rn(m, 0.5f);
    e += 1;
  }
  const float f2 = __fmul_rn(2.0f, __fdiv_rn(__fsub_rn(m, 1.0f), __fadd_rn(m, 1.0f)));
  const float s = __fmul_rn(__fmul_rn(f2, f2), 0.25f);
  float q = (float)(1.0 / 9.0);
  q = __fmaf_rn(q, s, (float)(1.0 / 7.0));
  q = __fmaf_rn(q, s, (float)(1.0 / 5.0));
  q = __fmaf_rn(q, s, (float)(1.0 / 3.0));
  const float lm = __fmaf_rn(__fmul_rn(f2, s), q, f2);
  const float ef = (float)e;
  return __fmaf_rn(ef, ln2_head, __fmaf_rn(ef, ln2_tail, lm));
}

}  // namespace bi
