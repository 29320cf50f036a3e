// rope_math.cuh - the rotation of one adjacent pair by angle phi, shared by the
// stand-alone rotary-embedding pass and the rotation phase of the fused
// attention kernel, so both give the same bits:
//   x'_2i   = x_2i cos phi - x_2i+1 sin phi
//   x'_2i+1 = x_2i sin phi + x_2i+1 cos phi
// The rounding is spelled out (one product rounded, then a fused multiply-add)
// so that the compiler's choice of contraction, which may differ between the
// two call sites, cannot change the result.
#pragma once

namespace ajvp {

__device__ __forceinline__ void rope_rotate_pair(float& x0, float& x1, float c, float s) {
  const float a = x0, b = x1;
  x0 = __fmaf_rn(a, c, -__fmul_rn(b, s));
  x1 = __fmaf_rn(a, s, __fmul_rn(b, c));
}

}  // namespace ajvp
