// NVFP4 encoding of one group of 16 values (the Q/K/V quantisation kernels
// and the decode kernel's query row): scale = E4M3_rn(fl32(amax / 6)),
// code = E2M1_rn(x / scale), a zero scale encoding the group as +0.
//
// x / scale must be rounded exactly like a correctly rounded division: for
// fp16 x and an E4M3 scale the quotient is either exactly an E2M1 rounding
// tie or at least 2^-12 (relative) away from one.  The division follows
// Markstein's correction of a reciprocal-multiply quotient (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990): q1 = x * (1/s) is within
// 1.5 ulp of x/s; the residual e = x - q1*s is exact by FMA, and
// q = q1 + e*(1/s) lands exactly on the quotient whenever the quotient is
// representable (the tie case) and within an ulp otherwise, which cannot move
// it across a tie.  The scale uses the correctly rounded division amax/6.
#pragma once
#include "ptx.cuh"

namespace thrift {

struct Group16 {
  uint32_t lo, hi;   // 16 E2M1 codes, element 2k in the low nibble of byte k
  uint32_t scale;    // E4M3 byte
};

// The quotient keeps the sign of x (so -0 stays -0 and encodes as code 8).
__device__ __forceinline__ float quotient(float x, float s, float r) {
  const float q1 = x * r;
  const float e = fmaf(-q1, s, x);
  return copysignf(fmaf(e, r, q1), x);
}

__device__ __forceinline__ Group16 encode16(const float (&x)[16]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  const uint32_t sbyte = cvt_e4m3x2(__fdiv_rn(amax, 6.0f), 0.f) & 0xFFu;
  const float s = e4m3_to_f32(sbyte);
  Group16 g{0u, 0u, sbyte};
  if (s > 0.f) {
    const float r = __frcp_rn(s);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      const uint32_t pair = cvt_e2m1x2(quotient(x[i], s, r), quotient(x[i + 1], s, r));
      w[i / 8] |= pair << ((i % 8) * 4);
    }
    g.lo = w[0];
    g.hi = w[1];
  }
  return g;
}

}  // namespace thrift
