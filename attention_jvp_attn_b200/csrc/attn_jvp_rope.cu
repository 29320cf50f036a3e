// attn_jvp_rope.cu - rotary position embedding of Q, K and their tangents
// tQ, tK ahead of the attention JVP, and its C ABI (attn_jvp_rope).
//
// The pages name RoPE as the positional treatment of queries and keys, one of
// the neighbours of the attention inside the layer-level JVP (Causal-rCM
// summary page, section 3, "KV Cache": pre- and post-RoPE caching; "JVP and
// distributed attention"). They give no formula; this is the standard rotary
// embedding on adjacent pairs with per-token angles phi [L, d/2] supplied by
// the caller as cos and sin tables (1-D or 3-D positions, the packed
// clean|noisy order: all of it lives in the tables):
//
//   x'_2i   = x_2i cos phi_ti - x_2i+1 sin phi_ti
//   x'_2i+1 = x_2i sin phi_ti + x_2i+1 cos phi_ti
//
// The rotation does not depend on its input, so the tangent of a rotated
// query (key) is the rotated tangent: the same kernel turns tQ and tK.
//
// One pass over HBM: each thread moves 16 bytes of one of the four tensors
// per step (8 bf16 or 4 fp32 values, whole pairs, one token), reads the
// matching cos/sin entries (L2-resident: L * d/2 * 8 bytes) and writes the
// result; grid-stride loop, gridDim.y = the four tensors. An output may be
// its own input (in place): every element is read and then written by the
// same thread.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "attn_jvp.h"
#include "rope_math.cuh"

namespace ajvp_rope {

constexpr int kThreads = 256;

struct RopeParams {
  const void* in[4];  // q, k, tq, tk: [B, L, H, d]
  void* out[4];
  const float* cos;   // [L, d/2]
  const float* sin;   // [L, d/2]
  int64_t n_vec;      // 16-byte vectors per tensor
  int L, H, d;
};

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;  // elements per 16 bytes
};
template <>
struct Vec<float> {
  static constexpr int N = 4;
};

__device__ __forceinline__ void unpack(const uint4& u, float* x, __nv_bfloat16) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
    const float2 f = __bfloat1622float2(h);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void unpack(const uint4& u, float* x, float) {
  x[0] = __uint_as_float(u.x);
  x[1] = __uint_as_float(u.y);
  x[2] = __uint_as_float(u.z);
  x[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ uint4 pack(const float* x, __nv_bfloat16) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ uint4 pack(const float* x, float) {
  return make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]),
                    __float_as_uint(x[3]));
}

template <typename T>
__global__ void __launch_bounds__(kThreads) rope_kernel(const __grid_constant__ RopeParams p) {
  constexpr int N = Vec<T>::N;
  constexpr int NP = N / 2;  // pairs per vector
  const int which = blockIdx.y;
  const uint4* src = static_cast<const uint4*>(p.in[which]);
  uint4* dst = static_cast<uint4*>(p.out[which]);
  const int vec_per_row = p.d / N;          // vectors per (token, head) row
  const int64_t vec_per_token = int64_t(p.H) * vec_per_row;
  const int half = p.d / 2;
  for (int64_t v = int64_t(blockIdx.x) * kThreads + threadIdx.x; v < p.n_vec;
       v += int64_t(gridDim.x) * kThreads) {
    const int t = static_cast<int>((v / vec_per_token) % p.L);
    const int col = static_cast<int>(v % vec_per_row) * N;  // first element of the vector
    const int64_t a = int64_t(t) * half + col / 2;        // first pair's angle
    float x[N], c[NP], s[NP];
    unpack(src[v], x, T());
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      c[i] = p.cos[a + i];
      s[i] = p.sin[a + i];
    }
#pragma unroll
    for (int i = 0; i < NP; ++i) ajvp::rope_rotate_pair(x[2 * i], x[2 * i + 1], c[i], s[i]);
    dst[v] = pack(x, T());
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace ajvp_rope

extern "C" {

int attn_jvp_rope(const attn_jvp_shape* shape, const void* q, const void* k, const void* tq,
                  const void* tk, const float* cos, const float* sin, void* q_out, void* k_out,
                  void* tq_out, void* tk_out, void* stream) {
  using namespace ajvp_rope;
  if (!shape) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  const attn_jvp_shape& s = *shape;
  if (s.B < 1 || s.H < 1 || s.L < 1) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  if (s.dtype != ATTN_JVP_BF16 && s.dtype != ATTN_JVP_F32) return ATTN_JVP_ERR_UNSUPPORTED;
  if (s.d != 64 && s.d != 128) return ATTN_JVP_ERR_UNSUPPORTED;
  if (s.L > (int64_t(1) << 30) || s.H > 65535 || s.B > 65535) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  const void* ptrs[] = {q, k, tq, tk, cos, sin, q_out, k_out, tq_out, tk_out};
  for (const void* ptr : ptrs) {
    if (!ptr) return ATTN_JVP_ERR_INVALID_ARGUMENT;
    if (!aligned16(ptr)) return ATTN_JVP_ERR_MISALIGNED;
  }
  int dev = -1, major = 0, minor = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return ATTN_JVP_ERR_NO_DEVICE;
  }
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_JVP_ERR_CUDA;
  }
  if (major != 10 || minor != 0) return ATTN_JVP_ERR_NO_DEVICE;
  RopeParams p;
  p.in[0] = q;
  p.in[1] = k;
  p.in[2] = tq;
  p.in[3] = tk;
  p.out[0] = q_out;
  p.out[1] = k_out;
  p.out[2] = tq_out;
  p.out[3] = tk_out;
  p.cos = cos;
  p.sin = sin;
  p.L = static_cast<int>(s.L);
  p.H = static_cast<int>(s.H);
  p.d = static_cast<int>(s.d);
  const int per_vec = s.dtype == ATTN_JVP_BF16 ? Vec<__nv_bfloat16>::N : Vec<float>::N;
  p.n_vec = s.B * s.L * s.H * s.d / per_vec;
  // enough CTAs to fill every SM several times over; the loop strides the rest
  const int64_t want = (p.n_vec + kThreads - 1) / kThreads;
  const int64_t cap = int64_t(sms) * 8;
  const dim3 grid(static_cast<unsigned>(want < cap ? want : cap), 4);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.dtype == ATTN_JVP_BF16)
    rope_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(p);
  else
    rope_kernel<float><<<grid, kThreads, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? ATTN_JVP_OK : ATTN_JVP_ERR_CUDA;
}

}  // extern "C"
