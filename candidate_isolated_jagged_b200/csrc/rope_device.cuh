// Right-anchored rotary position embedding, device arithmetic shared by the rotation pre-pass, the
// cosine/sine tables and the attention kernel's in-tile rotation (候选隔离注意力掩码, section
// 位置编码：候选共用一个位置). Every path forms cos/sin of p * theta_j the same way, so a tensor
// rotated by the pre-pass and a tile rotated inside the attention kernel hold the same bf16 values.
//
// theta_j = base^(-2j/d) for the pair (j, j + d/2). The angle p * theta_j reaches thousands of
// radians at the low frequencies; it is split as p = 128 q + r (0 <= r < 128):
//   cos(p theta) = cos(128 q theta) cos(r theta) - sin(128 q theta) sin(r theta)
//   sin(p theta) = sin(128 q theta) cos(r theta) + cos(128 q theta) sin(r theta)
// and each factor is evaluated by rope_cs: angle formed and reduced to [-pi, pi] in fp64, sine and
// cosine by the fast intrinsics on the reduced fp32 argument (accurate to about 2^-21 there). The
// attention kernel reads the factors from two small tables (128 q multiples of the positions in
// use, and r = 0..127) instead of evaluating them per element.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace jca {

constexpr int kRopeFine = 128;   // positions per coarse step (p = 128 q + r)

__host__ __device__ inline double rope_inv_freq(int j, int d, double log2_base) {
  return exp2(-(double)(2 * j) / (double)d * log2_base);
}

// (cos, sin) of p * inv_freq: fp64 angle and reduction, fast fp32 sine and cosine.
__device__ __forceinline__ float2 rope_cs(double p, double inv_freq) {
  constexpr double kTwoPi = 6.283185307179586476925286766559;
  constexpr double kInvTwoPi = 0.15915494309189533576888376337251;
  const double ang = p * inv_freq;
  const double red = ang - kTwoPi * rint(ang * kInvTwoPi);
  float sn, cs;
  __sincosf((float)red, &sn, &cs);
  return make_float2(cs, sn);
}

// Coarse and fine indices of position p (floor division by 128 for negative positions too).
__device__ __forceinline__ void rope_split(int64_t p, int64_t& q, int& r) {
  q = p >= 0 ? p / kRopeFine : -((-p + kRopeFine - 1) / kRopeFine);
  r = (int)(p - q * kRopeFine);
}

// (cos, sin) of (128 q + r) theta from the factors of 128 q and r.
__device__ __forceinline__ float2 rope_compose(float2 coarse, float2 fine) {
  return make_float2(__fmaf_rn(coarse.x, fine.x, -__fmul_rn(coarse.y, fine.y)),
                     __fmaf_rn(coarse.y, fine.x, __fmul_rn(coarse.x, fine.y)));
}

// (a, b) rotated by the angle whose (cos, sin) is cs, in fp32.
__device__ __forceinline__ void rope_rotate(float a, float b, float2 cs, float& oa, float& ob) {
  oa = __fmaf_rn(a, cs.x, -__fmul_rn(b, cs.y));
  ob = __fmaf_rn(a, cs.y, __fmul_rn(b, cs.x));
}

}  // namespace jca
