// rope_math.cuh - the rotation of one adjacent pair by angle phi, shared by the
// stand-alone rotary-embedding pass and the rotation phase of the fused
// attention kernel, so both give the same bits:
//   x'_2i   = x_2i cos phi - x_2i+1 sin phi
//   x'_2i+1 = x_2i sin phi + x_2i+1 cos phi
#pragma once

namespace ajvp {

__device__ __forceinline__ void rope_rotate_pair(float& x0, float& x1, float c, float s) {
  const float a = x0, b = x1;
  x0 = a * c - b * s;
  x1 = a * s + b * c;
}

}  // namespace ajvp
