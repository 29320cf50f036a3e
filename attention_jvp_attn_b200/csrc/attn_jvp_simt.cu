// attn_jvp_simt.cu - fp32 custom-mask attention forward fused with its JVP on
// CUDA cores.
//
// Same method as the tensor-core kernel (Causal-rCM summary page, App. B: one
// online-softmax pass, primal and tangent accumulators rescaled together,
// the block-sparse schedule of the mask, masked entries carrying no tangent)
// in plain fp32 arithmetic, for callers that need fp32 accuracy (TF32 tensor
// cores keep only 10 mantissa bits).
//
// CTA = 32 query rows of one (batch, head), 8 warps x 4 rows. Per admissible
// key tile of 32 keys (K, tK, V, tV staged in shared memory), lane j of a
// warp scores key j for the warp's row; the running max is exact (rescaled
// every tile); each lane accumulates d/32 output columns of A = sum p v and
// T = sum (u v + p tv), u = p s tS'.
#include "kernels.cuh"

namespace ajvp {

template <int D>
struct SimtCfg {
  static constexpr int BQ = kSimtBlockQ;
  static constexpr int BK = kSimtBlockK;
  static constexpr int NW = kSimtThreads / 32;
  static constexpr int RPW = BQ / NW;  // rows per warp
  static constexpr int KP = D + 1;     // padded row pitch of K / tK (conflict-free column walk)
  static constexpr int CPL = D / 32;   // output columns per lane
  static constexpr size_t BYTES = sizeof(float) * (2 * BK * KP + 2 * BK * D + 2 * BQ * D);
};

template <int D>
__global__ void __launch_bounds__(kSimtThreads) attn_jvp_simt_kernel(const __grid_constant__ SimtParams p) {
  using C = SimtCfg<D>;
  extern __shared__ float sm[];
  float* sK = sm;
  float* sTK = sK + C::BK * C::KP;
  float* sV = sTK + C::BK * C::KP;
  float* sTV = sV + C::BK * D;
  float* sQ = sTV + C::BK * D;
  float* sTQ = sQ + C::BQ * D;

  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  MaskSpec mask = p.mask;  // with the group table (if any) from this launch's parameters
  mask.groups = p.groups;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = p.L, H = p.H;
  const size_t rs = static_cast<size_t>(H) * D;  // row stride of [B, L, H, d]
  const size_t base = (static_cast<size_t>(b) * L * H + h) * D;

  for (int e = threadIdx.x; e < C::BQ * D; e += kSimtThreads) {
    const int r = e / D, x = e - r * D;
    const int t = qt * C::BQ + r;
    const bool in = t < L;
    sQ[e] = in ? p.q[base + t * rs + x] : 0.f;
    sTQ[e] = in ? p.tq[base + t * rs + x] : 0.f;
  }

  float m[C::RPW], l[C::RPW], ds[C::RPW], A[C::RPW][C::CPL], T[C::RPW][C::CPL];
  RowRange rr[C::RPW];
#pragma unroll
  for (int i = 0; i < C::RPW; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
    ds[i] = 0.f;
#pragma unroll
    for (int u = 0; u < C::CPL; ++u) A[i][u] = T[i][u] = 0.f;
    rr[i] = row_range(mask, qt * C::BQ + warp * C::RPW + i);
  }

  const TileSched sch = make_tile_sched(mask, qt, C::BQ, C::BK);
  const int cnt = sch.count();
  for (int idx = 0; idx < cnt; ++idx) {
    const int k0 = sch.tile(idx) * C::BK;
    __syncthreads();
    for (int e = threadIdx.x; e < C::BK * D; e += kSimtThreads) {
      const int r = e / D, x = e - r * D;
      const int t = k0 + r;
      const bool in = t < L;
      const size_t g = base + t * rs + x;
      sK[r * C::KP + x] = in ? p.k[g] : 0.f;
      sTK[r * C::KP + x] = in ? p.tk[g] : 0.f;
      sV[e] = in ? p.v[g] : 0.f;
      sTV[e] = in ? p.tv[g] : 0.f;
    }
    __syncthreads();
    const int key = k0 + lane;
#pragma unroll 1
    for (int i = 0; i < C::RPW; ++i) {
      const int r = warp * C::RPW + i;
      const float* q = sQ + r * D;
      const float* tq = sTQ + r * D;
      const float* kr = sK + lane * C::KP;
      const float* tkr = sTK + lane * C::KP;
      float s = 0.f, ts = 0.f;
#pragma unroll 8
      for (int x = 0; x < D; ++x) {
        const float kx = kr[x];
        s = fmaf(q[x], kx, s);
        ts = fmaf(tq[x], kx, ts);
        ts = fmaf(q[x], tkr[x], ts);
      }
      const bool allowed = key < L && row_allows(rr[i], key);
      const float xs = allowed ? s * p.scale_log2 : -INFINITY;
      float mt = xs;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
      const float m_new = fmaxf(m[i], mt);
      const float alpha = (m[i] == -INFINITY) ? 0.f : exp2f(m[i] - m_new);
      const float mb = (m_new == -INFINITY) ? 0.f : m_new;
      const float pj = allowed ? exp2f(xs - mb) : 0.f;
      const float uj = pj * p.scale * ts;
      float ps = pj, us = uj;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        ps += __shfl_xor_sync(0xffffffffu, ps, o);
        us += __shfl_xor_sync(0xffffffffu, us, o);
      }
      l[i] = alpha * l[i] + ps;
      ds[i] = alpha * ds[i] + us;
      m[i] = m_new;
#pragma unroll
      for (int u = 0; u < C::CPL; ++u) {
        A[i][u] *= alpha;
        T[i][u] *= alpha;
      }
#pragma unroll 4
      for (int jj = 0; jj < C::BK; ++jj) {
        const float pb = __shfl_sync(0xffffffffu, pj, jj);
        const float ub = __shfl_sync(0xffffffffu, uj, jj);
        const float* vr = sV + jj * D + lane;
        const float* tvr = sTV + jj * D + lane;
#pragma unroll
        for (int u = 0; u < C::CPL; ++u) {
          const float vv = vr[32 * u];
          A[i][u] = fmaf(pb, vv, A[i][u]);
          T[i][u] = fmaf(ub, vv, T[i][u]);
          T[i][u] = fmaf(pb, tvr[32 * u], T[i][u]);
        }
      }
    }
  }

#pragma unroll
  for (int i = 0; i < C::RPW; ++i) {
    const int t = qt * C::BQ + warp * C::RPW + i;
    if (t >= L) continue;
    const float inv_l = 1.f / l[i];
    const float mu = ds[i] * inv_l;
    const size_t g = base + t * rs;
#pragma unroll
    for (int u = 0; u < C::CPL; ++u) {
      const float o = A[i][u] * inv_l;
      p.o[g + lane + 32 * u] = o;
      p.to[g + lane + 32 * u] = T[i][u] * inv_l - mu * o;
    }
    if (lane == 0) {
      const float mb = (m[i] == -INFINITY) ? 0.f : m[i];
      p.lse[(static_cast<size_t>(b) * H + h) * L + t] = (mb + log2f(l[i])) * 0.69314718055994530942f;
    }
  }
}

size_t simt_smem_bytes(int d) { return d == 128 ? SimtCfg<128>::BYTES : SimtCfg<64>::BYTES; }

cudaError_t simt_prepare(int d) {
  if (d == 128)
    return cudaFuncSetAttribute(attn_jvp_simt_kernel<128>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(SimtCfg<128>::BYTES));
  return cudaFuncSetAttribute(attn_jvp_simt_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(SimtCfg<64>::BYTES));
}

cudaError_t simt_launch(int d, const SimtParams& p, cudaStream_t stream) {
  const dim3 grid((p.L + kSimtBlockQ - 1) / kSimtBlockQ, p.H, p.B);
  if (d == 128)
    attn_jvp_simt_kernel<128><<<grid, kSimtThreads, SimtCfg<128>::BYTES, stream>>>(p);
  else
    attn_jvp_simt_kernel<64><<<grid, kSimtThreads, SimtCfg<64>::BYTES, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace ajvp
