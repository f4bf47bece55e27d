// Block quantisation rounding shared by the kernels: codes = rne(x / s) of
// one 16-byte chunk of fp16 values, bit-identical to the IEEE definition.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace tilemix {

// rne(f / s) without a division on the common path.  y = f * rcp_rn(s) is
// within 2^-15 of the correctly rounded quotient (|f / s| <= 127, two
// roundings of 2^-24 relative each), so whenever y lies more than 2^-12 from
// every half-integer both round to the same integer; inside that band the
// quotient is taken with the IEEE division itself.  Rounding to an integer
// adds 1.5 * 2^23 (for |y| < 2^22 the sum's unit in the last place is 1, so
// round-to-nearest-even of the addition is rne of y, and the integer n sits
// in the low mantissa bits: the sum's bit pattern is 0x4B400000 + n, whose low
// byte is the two's-complement byte of n).  No clamp is needed: |f| <= a and
// s = fl(a / 127) give |y| < 127.0001, so rne(y) already lies in [-127, 127].
constexpr float kRoundShift = 12582912.0f;  // 1.5 * 2^23
constexpr float kBandEdge = 0.5f - 0x1p-12f;

__device__ __forceinline__ float shifted_code_exact(float f, float s, float r) {
  const float y = __fmul_rn(f, r);
  const float t = __fadd_rn(y, kRoundShift);
  const float e = __fsub_rn(y, __fsub_rn(t, kRoundShift));  // y - rne(y), exact
  return fabsf(e) > kBandEdge ? __fadd_rn(__fdiv_rn(f, s), kRoundShift) : t;
}

// Two-lane fp32 arithmetic (sm_100 packed instructions: one issue for both
// lanes, each lane rounded exactly as the scalar IEEE operation).
__device__ __forceinline__ unsigned long long f2_bits(float x, float y) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(x), "f"(y));
  return r;
}
__device__ __forceinline__ float2 bits_f2(unsigned long long r) {
  float2 v;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
  return v;
}
__device__ __forceinline__ unsigned long long mul2_rn(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ unsigned long long add2_rn(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ unsigned long long sub2_rn(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Codes of the eight fp16 values of one 16-byte chunk, as eight bytes in
// order.  The band test is taken for the whole chunk at once (the largest
// distance from an integer), so the common path has no per-element branch;
// its arithmetic runs on value pairs.
__device__ __forceinline__ uint2 quant_chunk(const uint4& u, float s, float r) {
  const __half2* hv = reinterpret_cast<const __half2*>(&u);
  const unsigned long long rr = f2_bits(r, r);
  const unsigned long long shift = f2_bits(kRoundShift, kRoundShift);
  float2 f[4], t[4];
  float emax = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    f[k] = __half22float2(hv[k]);
    const unsigned long long y = mul2_rn(f2_bits(f[k].x, f[k].y), rr);
    const unsigned long long ts = add2_rn(y, shift);
    const float2 e = bits_f2(sub2_rn(y, sub2_rn(ts, shift)));  // y - rne(y), exact
    t[k] = bits_f2(ts);
    emax = fmaxf(emax, fmaxf(fabsf(e.x), fabsf(e.y)));
  }
  if (emax > kBandEdge) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      t[k].x = shifted_code_exact(f[k].x, s, r);
      t[k].y = shifted_code_exact(f[k].y, s, r);
    }
  }
  uint32_t b[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    b[2 * k] = static_cast<uint32_t>(__float_as_int(t[k].x));
    b[2 * k + 1] = static_cast<uint32_t>(__float_as_int(t[k].y));
  }
  return make_uint2(__byte_perm(__byte_perm(b[0], b[1], 0x3340u), __byte_perm(b[2], b[3], 0x3340u), 0x5410u),
                    __byte_perm(__byte_perm(b[4], b[5], 0x3340u), __byte_perm(b[6], b[7], 0x3340u), 0x5410u));
}

}  // namespace tilemix
