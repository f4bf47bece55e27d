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

// Codes of the eight fp16 values of one 16-byte chunk, as eight bytes in
// order.  The band test is taken for the whole chunk at once, so the common
// path has no per-element branch.
__device__ __forceinline__ uint2 quant_chunk(const uint4& u, float s, float r) {
  const __half2* hv = reinterpret_cast<const __half2*>(&u);
  float f[8], t[8];
  bool near_half = false;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 v = __half22float2(hv[k]);
    f[2 * k] = v.x;
    f[2 * k + 1] = v.y;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float y = __fmul_rn(f[e], r);
    t[e] = __fadd_rn(y, kRoundShift);
    near_half |= fabsf(__fsub_rn(y, __fsub_rn(t[e], kRoundShift))) > kBandEdge;
  }
  if (near_half) {
#pragma unroll
    for (int e = 0; e < 8; ++e) t[e] = shifted_code_exact(f[e], s, r);
  }
  uint32_t b[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) b[e] = static_cast<uint32_t>(__float_as_int(t[e]));
  return make_uint2(__byte_perm(__byte_perm(b[0], b[1], 0x3340u), __byte_perm(b[2], b[3], 0x3340u), 0x5410u),
                    __byte_perm(__byte_perm(b[4], b[5], 0x3340u), __byte_perm(b[6], b[7], 0x3340u), 0x5410u));
}

}  // namespace tilemix
