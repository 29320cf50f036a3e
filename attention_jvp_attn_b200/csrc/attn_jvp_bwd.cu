// attn_jvp_bwd.cu - backward (vector-Jacobian product) of the masked primal
// attention on CUDA cores, and its C ABI (attn_jvp_bwd, attn_jvp_bwd_groups).
// bf16 problems the tensor-core kernels take (attn_jvp_bwd_tc.cu) go there;
// the kernels in this file serve fp32 and bf16 sequences too short for them.
//
// The fused forward returns LSE so that a backward pass can rebuild P without
// a second softmax pass (Causal-rCM summary page, App. B, last item); the
// pages describe no backward kernel. This one computes the plain gradient of
// O = softmax(s Q K^T + M) V, and optionally of LSE, under the same mask:
//
//   P_ij  = exp(s q_i.k_j - LSE_i) on admissible pairs, 0 elsewhere
//   dP_ij = dO_i . v_j
//   D_i   = dO_i . O_i - dLSE_i          (= rowsum(P * dP) - dLSE_i)
//   dS_ij = P_ij (dP_ij - D_i)
//   dV_j  = sum_i P_ij dO_i,   dK_j = s sum_i dS_ij q_i,   dQ_i = s sum_j dS_ij k_j
//
// Two kernels, so that every output row has exactly one writer (no atomics;
// the same bits on every run):
//   * attn_bwd_dq_kernel: one CTA per 32 query rows of a (batch, head); it
//     walks the key tiles of the mask's block-sparse schedule (the same
//     schedule as the forward kernels).
//   * attn_bwd_dkdv_kernel: one CTA per 32 keys; it walks the query blocks
//     whose schedule lists that key tile.
// Arithmetic is fp32 from bf16 or fp32 inputs; dQ, dK, dV are written in the
// input type (bf16 rounded to nearest even).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn_jvp.h"
#include "kernels.cuh"
#include "mask_schedule.cuh"

namespace ajvp_bwd {

using ajvp::GroupRange;
using ajvp::MaskSpec;
using ajvp::RowRange;
using ajvp::TileSched;

constexpr int kBlock = 32;                         // query rows per dQ CTA, keys per dK/dV CTA
constexpr int kThreads = 256;                      // 8 warps
constexpr int kPerWarp = kBlock / (kThreads / 32); // 4 rows (or keys) per warp
constexpr float kLog2e = 1.4426950408889634f;

struct BwdParams {
  const void *q, *k, *v, *o, *dout;  // [B, L, H, d] of the element type
  const float* lse;                  // [B, H, L]
  const float* dlse;                 // [B, H, L] or null (no LSE cotangent)
  void *dq, *dk, *dv;                // [B, L, H, d] of the element type
  int B, H, L;
  MaskSpec mask;
  float scale, scale_log2;
  GroupRange groups[ajvp::kMaxGroups];  // mask.mode == kModeGroups: the row groups
};

__device__ __forceinline__ float ld(const float* p, size_t i) { return p[i]; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p, size_t i) {
  return __bfloat162float(p[i]);
}
__device__ __forceinline__ void st(float* p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void st(__nv_bfloat16* p, size_t i, float x) {
  p[i] = __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// D_i and LSE_i * log2(e) of the block's rows [r0, r0 + 32): warp w takes
// rows w*4 .. w*4+3; rows past L get 0 (their P is 0).
template <int D, typename T>
__device__ __forceinline__ void row_stats(const BwdParams& p, size_t base, size_t lbase, int r0,
                                          float* sDelta, float* sLse) {
  const T* dO = static_cast<const T*>(p.dout);
  const T* O = static_cast<const T*>(p.o);
  const size_t rs = static_cast<size_t>(p.H) * D;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll 1
  for (int i = 0; i < kPerWarp; ++i) {
    const int r = warp * kPerWarp + i;
    const int t = r0 + r;
    float acc = 0.f;
    if (t < p.L) {
      const size_t g = base + static_cast<size_t>(t) * rs;
      for (int x = lane; x < D; x += 32) acc = fmaf(ld(dO, g + x), ld(O, g + x), acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) {
      if (t < p.L) {
        sDelta[r] = acc - (p.dlse ? p.dlse[lbase + t] : 0.f);
        sLse[r] = p.lse[lbase + t] * kLog2e;
      } else {
        sDelta[r] = 0.f;
        sLse[r] = 0.f;
      }
    }
  }
}

template <int D>
struct Smem {
  static constexpr int KP = D + 1;  // padded pitch: a lane walking its own row hits its own bank
  static constexpr size_t BYTES = sizeof(float) * (2 * kBlock * D + 2 * kBlock * KP);
};

template <int D, typename T>
__global__ void __launch_bounds__(kThreads) attn_bwd_dq_kernel(const __grid_constant__ BwdParams p) {
  constexpr int KP = Smem<D>::KP, CPL = D / 32;
  extern __shared__ float sm[];
  float* sQ = sm;                  // [32][D] query rows (read as broadcasts)
  float* sdO = sQ + kBlock * D;    // [32][D]
  float* sK = sdO + kBlock * D;    // [32][KP] keys (lane j walks key j)
  float* sV = sK + kBlock * KP;    // [32][KP]
  __shared__ float sDelta[kBlock], sLse[kBlock];

  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  MaskSpec mask = p.mask;
  mask.groups = p.groups;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = p.L;
  const size_t rs = static_cast<size_t>(p.H) * D;
  const size_t base = (static_cast<size_t>(b) * L * p.H + h) * D;
  const size_t lbase = (static_cast<size_t>(b) * p.H + h) * L;
  const T* Q = static_cast<const T*>(p.q);
  const T* K = static_cast<const T*>(p.k);
  const T* V = static_cast<const T*>(p.v);
  const T* dO = static_cast<const T*>(p.dout);
  const int r0 = qt * kBlock;

  for (int e = threadIdx.x; e < kBlock * D; e += kThreads) {
    const int r = e / D, x = e - r * D;
    const int t = r0 + r;
    const bool in = t < L;
    const size_t g = base + static_cast<size_t>(in ? t : 0) * rs + x;
    sQ[e] = in ? ld(Q, g) : 0.f;
    sdO[e] = in ? ld(dO, g) : 0.f;
  }
  row_stats<D, T>(p, base, lbase, r0, sDelta, sLse);

  RowRange rr[kPerWarp];
  float acc[kPerWarp][CPL];
#pragma unroll
  for (int i = 0; i < kPerWarp; ++i) {
    const int t = r0 + warp * kPerWarp + i;
    rr[i] = ajvp::row_range(mask, t < L ? t : L - 1);
#pragma unroll
    for (int u = 0; u < CPL; ++u) acc[i][u] = 0.f;
  }

  const TileSched sch = ajvp::make_tile_sched(mask, qt, kBlock, kBlock);
  const int cnt = sch.count();
  for (int idx = 0; idx < cnt; ++idx) {
    const int k0 = sch.tile(idx) * kBlock;
    __syncthreads();  // previous tile consumed (and, first time round, row stats written)
    for (int e = threadIdx.x; e < kBlock * D; e += kThreads) {
      const int r = e / D, x = e - r * D;
      const int t = k0 + r;
      const bool in = t < L;
      const size_t g = base + static_cast<size_t>(in ? t : 0) * rs + x;
      sK[r * KP + x] = in ? ld(K, g) : 0.f;
      sV[r * KP + x] = in ? ld(V, g) : 0.f;
    }
    __syncthreads();
    const int key = k0 + lane;
#pragma unroll  // register-resident accumulators
    for (int i = 0; i < kPerWarp; ++i) {
      const int r = warp * kPerWarp + i;
      const int t = r0 + r;
      const float* qr = sQ + r * D;
      const float* dor = sdO + r * D;
      const float* kr = sK + lane * KP;
      const float* vr = sV + lane * KP;
      float s = 0.f, dp = 0.f;
#pragma unroll 8
      for (int x = 0; x < D; ++x) {
        s = fmaf(qr[x], kr[x], s);
        dp = fmaf(dor[x], vr[x], dp);
      }
      const bool allowed = t < L && key < L && ajvp::row_allows(rr[i], key);
      const float pj = allowed ? exp2f(s * p.scale_log2 - sLse[r]) : 0.f;
      const float dsj = pj * (dp - sDelta[r]);
#pragma unroll 4
      for (int jj = 0; jj < kBlock; ++jj) {
        const float db = __shfl_sync(0xffffffffu, dsj, jj);
        const float* kj = sK + jj * KP + lane;
#pragma unroll
        for (int u = 0; u < CPL; ++u) acc[i][u] = fmaf(db, kj[32 * u], acc[i][u]);
      }
    }
  }

  T* dQ = static_cast<T*>(p.dq);
#pragma unroll
  for (int i = 0; i < kPerWarp; ++i) {
    const int t = r0 + warp * kPerWarp + i;
    if (t >= L) continue;
    const size_t g = base + static_cast<size_t>(t) * rs + lane;
#pragma unroll
    for (int u = 0; u < CPL; ++u) st(dQ, g + 32 * u, acc[i][u] * p.scale);
  }
}

template <int D, typename T>
__global__ void __launch_bounds__(kThreads) attn_bwd_dkdv_kernel(const __grid_constant__ BwdParams p) {
  constexpr int KP = Smem<D>::KP, CPL = D / 32;
  extern __shared__ float sm[];
  float* sK = sm;                  // [32][D] keys (read as broadcasts)
  float* sV = sK + kBlock * D;     // [32][D]
  float* sQ = sV + kBlock * D;     // [32][KP] query rows (lane r walks row r)
  float* sdO = sQ + kBlock * KP;   // [32][KP]
  __shared__ float sDelta[kBlock], sLse[kBlock];

  const int kt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  MaskSpec mask = p.mask;
  mask.groups = p.groups;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = p.L;
  const size_t rs = static_cast<size_t>(p.H) * D;
  const size_t base = (static_cast<size_t>(b) * L * p.H + h) * D;
  const size_t lbase = (static_cast<size_t>(b) * p.H + h) * L;
  const T* Q = static_cast<const T*>(p.q);
  const T* K = static_cast<const T*>(p.k);
  const T* V = static_cast<const T*>(p.v);
  const T* dO = static_cast<const T*>(p.dout);
  const int k0 = kt * kBlock;

  for (int e = threadIdx.x; e < kBlock * D; e += kThreads) {
    const int r = e / D, x = e - r * D;
    const int t = k0 + r;
    const bool in = t < L;
    const size_t g = base + static_cast<size_t>(in ? t : 0) * rs + x;
    sK[e] = in ? ld(K, g) : 0.f;
    sV[e] = in ? ld(V, g) : 0.f;
  }

  float dk[kPerWarp][CPL], dv[kPerWarp][CPL];
#pragma unroll
  for (int i = 0; i < kPerWarp; ++i)
#pragma unroll
    for (int u = 0; u < CPL; ++u) dk[i][u] = dv[i][u] = 0.f;

  const int n_qt = ajvp::cdiv(L, kBlock);
  for (int qt = 0; qt < n_qt; ++qt) {
    // the same test in every thread: the branch is uniform over the CTA
    const TileSched sch = ajvp::make_tile_sched(mask, qt, kBlock, kBlock);
    const bool hit = (kt >= sch.t1_begin && kt < sch.t1_end) ||
                     (kt >= sch.t2_begin && kt < sch.t2_end);
    if (!hit) continue;
    const int r0 = qt * kBlock;
    __syncthreads();  // previous query block consumed
    for (int e = threadIdx.x; e < kBlock * D; e += kThreads) {
      const int r = e / D, x = e - r * D;
      const int t = r0 + r;
      const bool in = t < L;
      const size_t g = base + static_cast<size_t>(in ? t : 0) * rs + x;
      sQ[r * KP + x] = in ? ld(Q, g) : 0.f;
      sdO[r * KP + x] = in ? ld(dO, g) : 0.f;
    }
    row_stats<D, T>(p, base, lbase, r0, sDelta, sLse);
    __syncthreads();
    const int t = r0 + lane;
    const RowRange rr = ajvp::row_range(mask, t < L ? t : L - 1);
    const float* qr = sQ + lane * KP;
    const float* dor = sdO + lane * KP;
    const float lse_t = sLse[lane], delta_t = sDelta[lane];
#pragma unroll  // register-resident accumulators
    for (int i = 0; i < kPerWarp; ++i) {
      const int j = warp * kPerWarp + i;
      const int key = k0 + j;
      const float* kr = sK + j * D;
      const float* vr = sV + j * D;
      float s = 0.f, dp = 0.f;
#pragma unroll 8
      for (int x = 0; x < D; ++x) {
        s = fmaf(qr[x], kr[x], s);
        dp = fmaf(dor[x], vr[x], dp);
      }
      const bool allowed = t < L && key < L && ajvp::row_allows(rr, key);
      const float pt = allowed ? exp2f(s * p.scale_log2 - lse_t) : 0.f;
      const float dst = pt * (dp - delta_t);
#pragma unroll 4
      for (int r2 = 0; r2 < kBlock; ++r2) {
        const float pb = __shfl_sync(0xffffffffu, pt, r2);
        const float db = __shfl_sync(0xffffffffu, dst, r2);
        const float* dorow = sdO + r2 * KP + lane;
        const float* qrow = sQ + r2 * KP + lane;
#pragma unroll
        for (int u = 0; u < CPL; ++u) {
          dv[i][u] = fmaf(pb, dorow[32 * u], dv[i][u]);
          dk[i][u] = fmaf(db, qrow[32 * u], dk[i][u]);
        }
      }
    }
  }

  T* dK = static_cast<T*>(p.dk);
  T* dV = static_cast<T*>(p.dv);
#pragma unroll
  for (int i = 0; i < kPerWarp; ++i) {
    const int key = k0 + warp * kPerWarp + i;
    if (key >= L) continue;
    const size_t g = base + static_cast<size_t>(key) * rs + lane;
#pragma unroll
    for (int u = 0; u < CPL; ++u) {
      st(dK, g + 32 * u, dk[i][u] * p.scale);
      st(dV, g + 32 * u, dv[i][u]);
    }
  }
}

template <int D, typename T>
cudaError_t prepare_one() {
  const int bytes = static_cast<int>(Smem<D>::BYTES);
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_dq_kernel<D, T>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(attn_bwd_dkdv_kernel<D, T>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int D, typename T>
cudaError_t launch(const BwdParams& p, cudaStream_t stream) {
  const dim3 grid(ajvp::cdiv(p.L, kBlock), p.H, p.B);
  attn_bwd_dq_kernel<D, T><<<grid, kThreads, Smem<D>::BYTES, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_bwd_dkdv_kernel<D, T><<<grid, kThreads, Smem<D>::BYTES, stream>>>(p);
  return cudaGetLastError();
}

// ---- host side -------------------------------------------------------------

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxSeq = int64_t(1) << 30;
std::mutex g_mu;
bool g_ready[kMaxDevices];

// Once per device: check it is sm_100 and raise the kernels' shared-memory limit.
int device_ready() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return ATTN_JVP_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_ready[dev]) return ATTN_JVP_OK;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_JVP_ERR_CUDA;
  }
  if (major != 10 || minor != 0) return ATTN_JVP_ERR_NO_DEVICE;  // built for sm_100a only
  if (prepare_one<64, float>() != cudaSuccess || prepare_one<128, float>() != cudaSuccess ||
      prepare_one<64, __nv_bfloat16>() != cudaSuccess ||
      prepare_one<128, __nv_bfloat16>() != cudaSuccess || ajvp::bwd_tc_prepare() != cudaSuccess) {
    cudaGetLastError();
    return ATTN_JVP_ERR_CUDA;
  }
  g_ready[dev] = true;
  return ATTN_JVP_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(const attn_jvp_shape* s) {
  if (!s) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  if (s->B < 1 || s->H < 1 || s->L < 1) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  if (s->dtype != ATTN_JVP_BF16 && s->dtype != ATTN_JVP_F32) return ATTN_JVP_ERR_UNSUPPORTED;
  if (s->d != 64 && s->d != 128) return ATTN_JVP_ERR_UNSUPPORTED;
  if (!(s->scale <= 0.f || std::isfinite(s->scale))) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  if (s->L > kMaxSeq || s->B > 65535 || s->H > 65535) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  return ATTN_JVP_OK;
}

int check_pointers(const void* const* ptrs, int n, const float* dlse) {
  for (int i = 0; i < n; ++i) {
    if (!ptrs[i]) return ATTN_JVP_ERR_INVALID_ARGUMENT;
    if (!aligned16(ptrs[i])) return ATTN_JVP_ERR_MISALIGNED;
  }
  if (dlse && !aligned16(dlse)) return ATTN_JVP_ERR_MISALIGNED;
  return ATTN_JVP_OK;
}

int check_mode_mask(const attn_jvp_shape* s, attn_jvp_mask m) {
  if (m.mode != ATTN_JVP_MASK_TEACHER_FORCING && m.mode != ATTN_JVP_MASK_BLOCK_CAUSAL)
    return ATTN_JVP_ERR_INVALID_ARGUMENT;
  if (m.chunk_tokens < 1 || m.n_chunks < 1) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  const int64_t per = (m.mode == ATTN_JVP_MASK_TEACHER_FORCING) ? 2 : 1;
  if (per * int64_t(m.n_chunks) * int64_t(m.chunk_tokens) != s->L)
    return ATTN_JVP_ERR_INVALID_ARGUMENT;
  return ATTN_JVP_OK;
}

int check_groups(const attn_jvp_shape* s, const attn_jvp_group* g, int32_t n) {
  if (!g || n < 1) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  if (n > ATTN_JVP_MAX_GROUPS) return ATTN_JVP_ERR_UNSUPPORTED;
  int64_t prev = 0;
  for (int32_t i = 0; i < n; ++i) {
    const attn_jvp_group& x = g[i];
    if (x.row_end <= prev) return ATTN_JVP_ERR_INVALID_ARGUMENT;
    if (x.k0_begin < 0 || x.k0_begin > x.k0_end || x.k0_end > x.k1_begin ||
        x.k1_begin > x.k1_end || x.k1_end > s->L)
      return ATTN_JVP_ERR_INVALID_ARGUMENT;
    if (x.k0_end - x.k0_begin + x.k1_end - x.k1_begin <= 0) return ATTN_JVP_ERR_INVALID_ARGUMENT;
    prev = x.row_end;
  }
  return prev == s->L ? ATTN_JVP_OK : ATTN_JVP_ERR_INVALID_ARGUMENT;
}

int run(const attn_jvp_shape* s, BwdParams& p, void* stream) {
  const int rc = device_ready();
  if (rc != ATTN_JVP_OK) return rc;
  p.B = static_cast<int>(s->B);
  p.H = static_cast<int>(s->H);
  p.L = static_cast<int>(s->L);
  p.mask.L = p.L;
  p.scale = s->scale > 0.f ? s->scale : 1.0f / std::sqrt(static_cast<float>(s->d));
  p.scale_log2 = p.scale * kLog2e;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s->dtype == ATTN_JVP_BF16 && ajvp::bwd_tc_supported(s->B, s->L, s->H, s->d)) {
    ajvp::BwdTcArgs a;
    a.q = p.q;
    a.k = p.k;
    a.v = p.v;
    a.o = p.o;
    a.dout = p.dout;
    a.lse = p.lse;
    a.dlse = p.dlse;
    a.dq = p.dq;
    a.dk = p.dk;
    a.dv = p.dv;
    a.B = s->B;
    a.L = s->L;
    a.H = s->H;
    a.d = s->d;
    a.mask = p.mask;
    a.mask.groups = p.mask.mode == ajvp::kModeGroups ? p.groups : nullptr;
    a.scale = p.scale;
    return ajvp::bwd_tc_launch(a, st);
  }
  cudaError_t e;
  if (s->dtype == ATTN_JVP_BF16)
    e = s->d == 128 ? launch<128, __nv_bfloat16>(p, st) : launch<64, __nv_bfloat16>(p, st);
  else
    e = s->d == 128 ? launch<128, float>(p, st) : launch<64, float>(p, st);
  return e == cudaSuccess ? ATTN_JVP_OK : ATTN_JVP_ERR_CUDA;
}

void set_buffers(BwdParams& p, const void* q, const void* k, const void* v, const void* o,
                 const void* dout, const float* lse, const float* dlse, void* dq, void* dk,
                 void* dv) {
  p.q = q;
  p.k = k;
  p.v = v;
  p.o = o;
  p.dout = dout;
  p.lse = lse;
  p.dlse = dlse;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
}

}  // namespace ajvp_bwd

extern "C" {

int attn_jvp_bwd(const attn_jvp_shape* shape, const void* q, const void* k, const void* v,
                 const void* o, const void* dout, const float* lse, const float* dlse,
                 attn_jvp_mask mask, void* dq, void* dk, void* dv, void* stream) {
  using namespace ajvp_bwd;
  int rc = check_shape(shape);
  if (rc != ATTN_JVP_OK) return rc;
  rc = check_mode_mask(shape, mask);
  if (rc != ATTN_JVP_OK) return rc;
  const void* ptrs[] = {q, k, v, o, dout, lse, dq, dk, dv};
  rc = check_pointers(ptrs, 9, dlse);
  if (rc != ATTN_JVP_OK) return rc;
  static thread_local BwdParams p;
  set_buffers(p, q, k, v, o, dout, lse, dlse, dq, dk, dv);
  p.mask.mode = mask.mode;
  p.mask.c = mask.chunk_tokens;
  p.mask.n = mask.n_chunks;
  p.mask.n_groups = 0;
  p.mask.groups = nullptr;
  return run(shape, p, stream);
}

int attn_jvp_bwd_groups(const attn_jvp_shape* shape, const void* q, const void* k,
                        const void* v, const void* o, const void* dout, const float* lse,
                        const float* dlse, const attn_jvp_group* groups, int32_t n_groups,
                        void* dq, void* dk, void* dv, void* stream) {
  using namespace ajvp_bwd;
  int rc = check_shape(shape);
  if (rc != ATTN_JVP_OK) return rc;
  rc = check_groups(shape, groups, n_groups);
  if (rc != ATTN_JVP_OK) return rc;
  const void* ptrs[] = {q, k, v, o, dout, lse, dq, dk, dv};
  rc = check_pointers(ptrs, 9, dlse);
  if (rc != ATTN_JVP_OK) return rc;
  static thread_local BwdParams p;
  set_buffers(p, q, k, v, o, dout, lse, dlse, dq, dk, dv);
  for (int32_t i = 0; i < n_groups; ++i)
    p.groups[i] = GroupRange{groups[i].row_end, groups[i].k0_begin, groups[i].k0_end,
                             groups[i].k1_begin, groups[i].k1_end};
  p.mask.mode = ajvp::kModeGroups;
  p.mask.c = 1;
  p.mask.n = 1;
  p.mask.n_groups = n_groups;
  p.mask.groups = nullptr;  // the kernels read the table from their own parameters
  return run(shape, p, stream);
}

}  // extern "C"
