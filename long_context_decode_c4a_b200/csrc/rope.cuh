// rope.cuh -- cos/sin of a rotary angle pos * inv_freq for positions up to 2^31.
#pragma once

namespace csa {

// The angle is formed and reduced modulo 2*pi in double precision (two-term Cody-Waite reduction
// with 2*pi split into its double rounding and the remainder), so the absolute angle error stays
// near 1e-16 * |angle|; the reduced angle, within [-pi, pi], then goes through single-precision
// sincosf. inv_freq = rope_base^(-2i/rope_dim) is formed on the host in double precision.
__device__ __forceinline__ void rope_cos_sin(long long pos, double inv_freq, float* c, float* s) {
  constexpr double kTwoPiHi = 6.283185307179586;            // 2*pi rounded to double
  constexpr double kTwoPiLo = 2.4492935982947064e-16;       // 2*pi - kTwoPiHi
  constexpr double kInvTwoPi = 0.15915494309189535;
  const double a = (double)pos * inv_freq;
  const double k = rint(a * kInvTwoPi);
  const double red = fma(-k, kTwoPiLo, fma(-k, kTwoPiHi, a));
  sincosf((float)red, s, c);
}

}  // namespace csa
