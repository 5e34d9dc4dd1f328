// Rotary position encoding on the sliding-window branch ("Simple linear
// attention language models balance the recall-throughput tradeoff", proposed
// method: rotary encoding on the window attention, none on the linear branch).
// Reading: the RoFormer rotation with rotate-half pairs; for i < d/2 the pair
// (x[i], x[i + d/2]) at absolute position p turns by p * theta_i, theta_i =
// base^(-2i/d).  theta_i comes from the host in fp64 (RopeTable).
//
// The angle p * theta_i reaches 1e5 rad at long positions, where an fp32
// product alone would be off by about 1e-2 rad, so it is formed in fp64 and
// reduced to [-pi, pi] by Cody-Waite reduction with a two-part 2*pi (the fma
// keeps k * hi exact) before the fast fp32 sine/cosine, accurate on [-pi, pi].
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace swa {

__device__ __forceinline__ void rope_cos_sin(int p, double theta, float& c, float& s) {
  constexpr double kInv2Pi = 0.15915494309189533577;      // 1 / (2 pi)
  constexpr double kTwoPiHi = 6.283185307179586232;       // 2 pi rounded to double
  constexpr double kTwoPiLo = 2.4492935982947064e-16;     // 2 pi - kTwoPiHi
  const double a = static_cast<double>(p) * theta;
  const double k = rint(a * kInv2Pi);
  double r = fma(-k, kTwoPiHi, a);
  r = fma(-k, kTwoPiLo, r);
  __sincosf(static_cast<float>(r), &s, &c);     // |r| <= pi: abs error below 2^-21
}

// Rotate the 8 pairs (lo[e], hi[e]) of two 16-byte bf16 chunks whose element
// index in the low half is i0 + e; the rotated values are rounded to bf16 (RNE).
template <typename Theta>
__device__ __forceinline__ void rope_rotate_chunks(uint4& lo, uint4& hi, int p, int i0, const Theta& theta) {
  uint32_t* l = reinterpret_cast<uint32_t*>(&lo);
  uint32_t* h = reinterpret_cast<uint32_t*>(&hi);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float xl[2] = {__uint_as_float(l[q] << 16), __uint_as_float(l[q] & 0xffff0000u)};
    float xh[2] = {__uint_as_float(h[q] << 16), __uint_as_float(h[q] & 0xffff0000u)};
    float yl[2], yh[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float c, s;
      rope_cos_sin(p, theta[i0 + 2 * q + u], c, s);
      yl[u] = fmaf(xl[u], c, -xh[u] * s);
      yh[u] = fmaf(xl[u], s, xh[u] * c);
    }
    __nv_bfloat162 a = __floats2bfloat162_rn(yl[0], yl[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(yh[0], yh[1]);
    l[q] = *reinterpret_cast<uint32_t*>(&a);
    h[q] = *reinterpret_cast<uint32_t*>(&b);
  }
}

}  // namespace swa
