// attn_jvp_tc.cu - bf16 custom-mask attention forward fused with its JVP on
// sm_100a tensor cores (tcgen05 MMA, TMEM accumulators, TMA tile loads).
//
// Causal-rCM summary page, App. B: one online-softmax pass computes the primal
// output and the tangent output with shared rescaling; masked entries get no
// tangent; the same sparse (query tile x key range) schedule drives the primal
// and tangent scores; queries and keys are tiled; outputs are O, LSE and tO.
//
// Per query tile (128 rows, one TMEM lane per row) and admissible key tile j
// (128 keys), with s the softmax scale and x = s log2(e) Q K^T:
//   MMA   S_j   = Q K_j^T                      (TMEM cols [0,128),   fp32)
//   MMA   tS'_j = tQ K_j^T + Q tK_j^T          (TMEM cols [128,256), fp32)
//   warps p = 2^(x - m), l += sum p, written back over S as bf16 P
//         u = p * s * tS', D += sum u,  written back over tS' as bf16 U
//   MMA   A += P V_j                           (TMEM cols [256,256+d))
//   MMA   T += U V_j + P tV_j                  (TMEM cols [256+d,256+2d))
//   end   O = A/l, mu = D/l, tO = T/l - mu O, LSE = (m + log2 l) ln 2
// which is tO = sum_j P_ij (tS_ij - mu_i) v_j + sum_j P_ij tv_j with
// tS = s (tQ K^T + Q tK^T), i.e. tP V + P tV, tP = P (tS - rowsum(P tS)).
//
// The running max m is only raised (and A, T, l, D rescaled by 2^(m_old -
// m_new)) when a tile's max exceeds it by more than kRescaleTau: every p stays
// <= 2^kRescaleTau and the final normalisation by l is exact.
//
// Warp roles (192 threads, one CTA per SM, persistent over work items):
//   warps 0-3  softmax + epilogue, thread i owns query row / TMEM lane i
//   warp  4    TMA producer (one thread): Q,tQ per item; K,tK,V,tV per key tile
//   warp  5    MMA issuer (one thread), TMEM allocator
// Work items (batch, head, query tile) are ordered head-major so that CTAs
// running at the same time share one head's keys in L2, and, within a head,
// longest first; CTA c takes items c, 2G-1-c, 2G+c, ... of that list.
// No TMA multicast is used anywhere: each CTA loads its own tiles.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace ajvp {

constexpr float kRescaleTau = 8.0f;
constexpr float kLn2 = 0.69314718055994530942f;

template <int D>
struct TcCfg {
  static constexpr int BM = kTcBlockM;
  static constexpr int BN = kTcBlockN;
  static constexpr int CH = D / 64;               // 128-byte swizzle chunks per row
  static constexpr int TILE = BN * D * 2;         // bytes of one K/V-type tile
  static constexpr int QBYTES = BM * D * 2;       // bytes of the Q (or tQ) tile
  static constexpr int NSLOT = (D == 128) ? 5 : 10;
  static constexpr int DATA = 2 * QBYTES + NSLOT * TILE;
  static constexpr int NBAR = 2 * NSLOT + 8;
  static constexpr int BYTES = 1024 + DATA + NBAR * 8 + 16;
  static constexpr uint32_t TM_S = 0;
  static constexpr uint32_t TM_TS = 128;
  static constexpr uint32_t TM_A = 256;
  static constexpr uint32_t TM_T = 256 + D;
  static constexpr uint32_t TM_COLS = 512;
  static_assert(BYTES <= 232448, "shared memory budget");
  static_assert(TM_T + D <= TM_COLS, "TMEM budget");
};

// K-major operand (rows of 64-element / 128-byte swizzled chunks, chunk c of
// a `rows`-row tile at c * rows * 128 bytes): k-step kk covers elements
// [16 kk, 16 kk + 16) of the contraction dimension.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t base, int rows, int kk) {
  const uint32_t addr = base + (kk >> 2) * rows * 128 + (kk & 3) * 32;
  return smem_desc_sw128(addr, 16, 1024);
}

// MN-major operand: a V tile [BN keys x D] read as B[K = keys, N = d]; k-step
// ks covers keys [16 ks, 16 ks + 16). 64-element N blocks sit BN*128 bytes
// apart (LBO), 8-key groups 1024 bytes apart (SBO).
template <int BN>
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t base, int ks) {
  return smem_desc_sw128(base + ks * 16 * 128, BN * 128, 1024);
}

struct WorkItem {
  int b, h, qt;
};

__device__ __forceinline__ int item_position(int k, int cta, int G) {
  return (k & 1) ? k * G + (G - 1 - cta) : k * G + cta;
}

__device__ __forceinline__ WorkItem decode_item(const TcParams& p, int pos) {
  const int bh = pos / p.n_qtiles;
  const int r = pos - bh * p.n_qtiles;
  WorkItem w;
  w.qt = p.order_len ? static_cast<int>(p.order[r]) : (p.n_qtiles - 1 - r);
  w.b = bh / p.H;
  w.h = bh - w.b * p.H;
  return w;
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1) attn_jvp_tc_kernel(const __grid_constant__ TcParams p) {
  using C = TcCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sTQ = smem + C::QBYTES;
  uint8_t* sRing = smem + 2 * C::QBYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::DATA);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::NSLOT;
  uint64_t* q_full = bars + 2 * C::NSLOT + 0;
  uint64_t* q_empty = bars + 2 * C::NSLOT + 1;
  uint64_t* s_full = bars + 2 * C::NSLOT + 2;
  uint64_t* ts_full = bars + 2 * C::NSLOT + 3;
  uint64_t* p_full = bars + 2 * C::NSLOT + 4;
  uint64_t* u_full = bars + 2 * C::NSLOT + 5;
  uint64_t* acc_full = bars + 2 * C::NSLOT + 6;
  uint64_t* drain = bars + 2 * C::NSLOT + 7;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int cta = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(ts_full, 1);
    mbar_init(p_full, 4);
    mbar_init(u_full, 4);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, C::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.map_q);
      tma_prefetch_desc(&p.map_k);
      tma_prefetch_desc(&p.map_v);
      tma_prefetch_desc(&p.map_tq);
      tma_prefetch_desc(&p.map_tk);
      tma_prefetch_desc(&p.map_tv);
      const uint64_t keep = l2_policy_evict_last();
      const CUtensorMap* kv_maps[4] = {&p.map_k, &p.map_tk, &p.map_v, &p.map_tv};
      uint32_t ctr = 0, q_issued = 0, q_ph = 0;
      bool ok = true;
      for (int k = 0; ok && k * G < p.n_items; ++k) {
        const int pos = item_position(k, cta, G);
        if (pos >= p.n_items) continue;
        const WorkItem w = decode_item(p, pos);
        if (q_issued > 0) {
          if (!mbar_wait(q_empty, q_ph, abort_flag, p.status)) { ok = false; break; }
          q_ph ^= 1;
        }
        mbar_arrive_expect_tx(q_full, 2 * C::QBYTES);
#pragma unroll
        for (int c = 0; c < C::CH; ++c) {
          tma_load_4d(sQ + c * C::BM * 128, &p.map_q, q_full, c * 64, w.h, w.qt * C::BM, w.b);
          tma_load_4d(sTQ + c * C::BM * 128, &p.map_tq, q_full, c * 64, w.h, w.qt * C::BM, w.b);
        }
        ++q_issued;
        const TileSched sch = make_tile_sched(p.mask, w.qt, C::BM, C::BN);
        const int cnt = sch.count();
        for (int idx = 0; ok && idx < cnt; ++idx) {
          const int kt = sch.tile(idx);
#pragma unroll 1
          for (int u = 0; u < 4; ++u) {
            const uint32_t slot = ctr % C::NSLOT;
            const uint32_t ph = (ctr / C::NSLOT) & 1;
            if (!mbar_wait(&empty[slot], ph ^ 1, abort_flag, p.status)) { ok = false; break; }
            mbar_arrive_expect_tx(&full[slot], C::TILE);
            uint8_t* dst = sRing + slot * C::TILE;
#pragma unroll
            for (int c = 0; c < C::CH; ++c)
              tma_load_4d_hint(dst + c * C::BN * 128, kv_maps[u], &full[slot], c * 64, w.h,
                               kt * C::BN, w.b, keep);
            ++ctr;
          }
        }
      }
      if (!ok) {
        // Abort: let every copy already issued land before the CTA exits.
        for (uint32_t s = 0; s < C::NSLOT && s < ctr; ++s) {
          const uint32_t last = ctr - 1 - ((ctr - 1 + C::NSLOT - s) % C::NSLOT);
          mbar_wait_drain(&full[s], (last / C::NSLOT) & 1, 200000000ull);
        }
        if (q_issued > 0) mbar_wait_drain(q_full, (q_issued - 1) & 1, 200000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(C::BM, C::BN, 0);
      const uint32_t idesc_v = idesc_bf16_f32(C::BM, D, 1);
      const uint32_t aQ = smem_u32(sQ), aTQ = smem_u32(sTQ), aRing = smem_u32(sRing);
      uint32_t ctr = 0, q_ph = 0, p_ph = 0, u_ph = 0;
      bool ok = true;
      for (int k = 0; ok && k * G < p.n_items; ++k) {
        const int pos = item_position(k, cta, G);
        if (pos >= p.n_items) continue;
        const WorkItem w = decode_item(p, pos);
        if (!mbar_wait(q_full, q_ph, abort_flag, p.status)) { ok = false; break; }
        q_ph ^= 1;
        tc_fence_after();
        const TileSched sch = make_tile_sched(p.mask, w.qt, C::BM, C::BN);
        const int cnt = sch.count();
        for (int idx = 0; idx < cnt; ++idx, ctr += 4) {
          const uint32_t sK = ctr % C::NSLOT, sTK = (ctr + 1) % C::NSLOT;
          const uint32_t sV = (ctr + 2) % C::NSLOT, sTV = (ctr + 3) % C::NSLOT;
          const uint32_t aK = aRing + sK * C::TILE, aTK = aRing + sTK * C::TILE;
          const uint32_t aV = aRing + sV * C::TILE, aTV = aRing + sTV * C::TILE;
          // S = Q K^T
          if (!mbar_wait(&full[sK], (ctr / C::NSLOT) & 1, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_ss(tmem + C::TM_S, desc_kmajor(aQ, C::BM, kk), desc_kmajor(aK, C::BN, kk), idesc_s,
                    kk > 0);
          umma_commit(s_full);
          // tS' = tQ K^T + Q tK^T
          if (!mbar_wait(&full[sTK], ((ctr + 1) / C::NSLOT) & 1, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_ss(tmem + C::TM_TS, desc_kmajor(aTQ, C::BM, kk), desc_kmajor(aK, C::BN, kk),
                    idesc_s, kk > 0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_ss(tmem + C::TM_TS, desc_kmajor(aQ, C::BM, kk), desc_kmajor(aTK, C::BN, kk),
                    idesc_s, 1);
          umma_commit(ts_full);
          umma_commit(&empty[sK]);
          umma_commit(&empty[sTK]);
          if (idx == cnt - 1) umma_commit(q_empty);
          // A += P V
          if (!mbar_wait(p_full, p_ph, abort_flag, p.status)) { ok = false; break; }
          p_ph ^= 1;
          tc_fence_after();
          if (!mbar_wait(&full[sV], ((ctr + 2) / C::NSLOT) & 1, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < C::BN / 16; ++ks)
            umma_ts(tmem + C::TM_A, tmem + C::TM_S + ks * 8, desc_mnmajor<C::BN>(aV, ks), idesc_v,
                    (idx > 0 || ks > 0) ? 1u : 0u);
          // T += U V + P tV
          if (!mbar_wait(u_full, u_ph, abort_flag, p.status)) { ok = false; break; }
          u_ph ^= 1;
          tc_fence_after();
          if (!mbar_wait(&full[sTV], ((ctr + 3) / C::NSLOT) & 1, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < C::BN / 16; ++ks)
            umma_ts(tmem + C::TM_T, tmem + C::TM_TS + ks * 8, desc_mnmajor<C::BN>(aV, ks), idesc_v,
                    (idx > 0 || ks > 0) ? 1u : 0u);
#pragma unroll
          for (int ks = 0; ks < C::BN / 16; ++ks)
            umma_ts(tmem + C::TM_T, tmem + C::TM_S + ks * 8, desc_mnmajor<C::BN>(aTV, ks), idesc_v, 1u);
          umma_commit(&empty[sV]);
          umma_commit(&empty[sTV]);
          if (idx == cnt - 1) umma_commit(acc_full);
        }
      }
      // Every MMA issued so far completes before TMEM is released.
      umma_commit(drain);
      mbar_wait_drain(drain, 0, 1000000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::TM_S;
    const uint32_t tTS = tmem + lane_off + C::TM_TS;
    const uint32_t tA = tmem + lane_off + C::TM_A;
    const uint32_t tT = tmem + lane_off + C::TM_T;
    const float scale_log2 = p.scale_log2;
    const float scale = p.scale;
    uint32_t s_ph = 0, ts_ph = 0, acc_ph = 0;
    bool ok = true;
    for (int k = 0; ok && k * G < p.n_items; ++k) {
      const int pos = item_position(k, cta, G);
      if (pos >= p.n_items) continue;
      const WorkItem w = decode_item(p, pos);
      const int t = w.qt * C::BM + warp * 32 + lane;  // this thread's query row
      const RowRange rr = row_range(p.mask, t);
      const TileSched sch = make_tile_sched(p.mask, w.qt, C::BM, C::BN);
      const int cnt = sch.count();
      float m_use = -INFINITY, l = 0.f, dsum = 0.f;
      for (int idx = 0; idx < cnt; ++idx) {
        const int kt = sch.tile(idx);
        const bool full_tile = sch.full(kt);
        const int k0 = kt * C::BN;
        if (!warp_wait(s_full, s_ph, abort_flag, p.status)) { ok = false; break; }
        s_ph ^= 1;
        tc_fence_after();
        uint32_t sr[C::BN];
#pragma unroll
        for (int c = 0; c < C::BN / 32; ++c)
          tmem_ld32(tS + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
        tmem_wait_ld();
        float x[C::BN];
        float mt = -INFINITY;
#pragma unroll
        for (int j = 0; j < C::BN; ++j) {
          x[j] = __uint_as_float(sr[j]) * scale_log2;
          if (!full_tile && !row_allows(rr, k0 + j)) x[j] = -INFINITY;
          mt = fmaxf(mt, x[j]);
        }
        bool resc = false;
        float alpha = 1.f;
        if (m_use == -INFINITY) {
          m_use = mt;  // nothing accumulated for this row yet (its A, T rows are zero)
        } else if (mt > m_use + kRescaleTau) {
          alpha = ex2_approx(m_use - mt);
          m_use = mt;
          l *= alpha;
          dsum *= alpha;
          resc = true;
        }
        if (__any_sync(0xffffffffu, resc)) {
          // All value MMAs of earlier tiles are complete (S of this tile was
          // issued after them), so A and T can be rescaled in place.
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t a[32], tt[32];
            tmem_ld32(tA + 32 * c, a);
            tmem_ld32(tT + 32 * c, tt);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              a[j] = __float_as_uint(__uint_as_float(a[j]) * alpha);
              tt[j] = __float_as_uint(__uint_as_float(tt[j]) * alpha);
            }
            tmem_st32(tA + 32 * c, a);
            tmem_st32(tT + 32 * c, tt);
          }
        }
        const float mb = (m_use == -INFINITY) ? 0.f : m_use;
        uint32_t pk[C::BN / 2];
        float lsum = 0.f;
#pragma unroll
        for (int j = 0; j < C::BN / 2; ++j) {
          const float p0 = ex2_approx(x[2 * j] - mb);
          const float p1 = ex2_approx(x[2 * j + 1] - mb);
          lsum += p0 + p1;
          pk[j] = pack_bf16x2(p0, p1);
        }
        l += lsum;
#pragma unroll
        for (int c = 0; c < C::BN / 64; ++c)
          tmem_st32(tS + 32 * c, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32 * c]));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);

        if (!warp_wait(ts_full, ts_ph, abort_flag, p.status)) { ok = false; break; }
        ts_ph ^= 1;
        tc_fence_after();
        float ds = 0.f;
#pragma unroll
        for (int c = 0; c < C::BN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tTS + 32 * c, v);
          tmem_wait_ld();
          uint32_t uk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const uint32_t pp = pk[16 * c + j];
            const float u0 = bf16lo_to_f32(pp) * scale * __uint_as_float(v[2 * j]);
            const float u1 = bf16hi_to_f32(pp) * scale * __uint_as_float(v[2 * j + 1]);
            ds += u0 + u1;
            uk[j] = pack_bf16x2(u0, u1);
          }
          tmem_st16(tTS + 16 * c, uk);
        }
        dsum += ds;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(u_full);
      }
      if (!ok) break;
      // ---------------- epilogue: O = A/l, tO = T/l - (D/l) O, LSE
      if (!warp_wait(acc_full, acc_ph, abort_flag, p.status)) { ok = false; break; }
      acc_ph ^= 1;
      tc_fence_after();
      const bool valid = t < p.L;
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
      const float mu = dsum * inv_l;
      const size_t row_off = ((static_cast<size_t>(w.b) * p.L + (valid ? t : 0)) * p.H + w.h) * D;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + row_off;
      __nv_bfloat16* torow = reinterpret_cast<__nv_bfloat16*>(p.to) + row_off;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t a[32], tt[32];
        tmem_ld32(tA + 32 * c, a);
        tmem_ld32(tT + 32 * c, tt);
        tmem_wait_ld();
        uint32_t ob[16], tb[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float o0 = __uint_as_float(a[2 * j]) * inv_l;
          const float o1 = __uint_as_float(a[2 * j + 1]) * inv_l;
          const float t0 = __uint_as_float(tt[2 * j]) * inv_l - mu * o0;
          const float t1 = __uint_as_float(tt[2 * j + 1]) * inv_l - mu * o1;
          ob[j] = pack_bf16x2(o0, o1);
          tb[j] = pack_bf16x2(t0, t1);
        }
        if (valid) {
          uint4* od = reinterpret_cast<uint4*>(orow + 32 * c);
          uint4* td = reinterpret_cast<uint4*>(torow + 32 * c);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            od[q] = make_uint4(ob[4 * q], ob[4 * q + 1], ob[4 * q + 2], ob[4 * q + 3]);
            td[q] = make_uint4(tb[4 * q], tb[4 * q + 1], tb[4 * q + 2], tb[4 * q + 3]);
          }
        }
      }
      if (valid) {
        const float mb = (m_use == -INFINITY) ? 0.f : m_use;
        p.lse[(static_cast<size_t>(w.b) * p.H + w.h) * p.L + t] = (mb + __log2f(l)) * kLn2;
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, C::TM_COLS);
}

size_t tc_smem_bytes(int d) { return d == 128 ? TcCfg<128>::BYTES : TcCfg<64>::BYTES; }

cudaError_t tc_prepare(int d) {
  if (d == 128)
    return cudaFuncSetAttribute(attn_jvp_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                TcCfg<128>::BYTES);
  return cudaFuncSetAttribute(attn_jvp_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              TcCfg<64>::BYTES);
}

cudaError_t tc_launch(int d, const TcParams& p, int grid, cudaStream_t stream) {
  if (d == 128)
    attn_jvp_tc_kernel<128><<<grid, kTcThreads, TcCfg<128>::BYTES, stream>>>(p);
  else
    attn_jvp_tc_kernel<64><<<grid, kTcThreads, TcCfg<64>::BYTES, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace ajvp
