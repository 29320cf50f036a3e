// attn_jvp_bwd_tc.cu - backward (vector-Jacobian product) of the masked primal
// attention for bf16 inputs on sm_100a tensor cores: tcgen05 MMAs with TMEM
// accumulators, TMA tile loads, warp-specialised roles.
//
// The fused forward returns LSE so that a backward pass can rebuild P without
// a second softmax pass (Causal-rCM summary page, App. B, last item). With
// s the softmax scale, on admissible pairs (0 elsewhere):
//   P_ij  = exp(s q_i.k_j - LSE_i) = 2^(s log2(e) q_i.k_j - LSE_i log2(e))
//   dP_ij = dO_i . v_j,   D_i = dO_i . O_i - dLSE_i,   dS_ij = P_ij (dP_ij - D_i)
//   dV = P^T dO,   dK = s dS^T Q,   dQ = s dS K
// Every product is a dense bf16 contraction with fp32 accumulation; P and dS
// are rounded to bf16 before they enter the dV, dK and dQ products.
//
// Three launches on the caller's stream. Each output element has one writer
// (no atomics: repeated calls give the same bits) and nothing is allocated:
//   1. bwd_prep_kernel: D_i and LSE_i log2(e) as fp32 rows of Lp = 128 ceil(L/128)
//      entries per (batch, head), written into the caller's dq buffer, which
//      serves as scratch until launch 3 overwrites it. Padded rows i >= L get
//      D = 0 and LSE = +inf, so their P is exactly 0.
//   2. bwd_dkdv_tc_kernel: one CTA per 128 keys of a (batch, head). dK and dV
//      stay in TMEM while the CTA streams the 128-row query tiles whose
//      key-tile schedule lists this key tile (the forward's schedule,
//      transposed), from separate Q and dO rings:
//        S^T = K Q^T, dP^T = V dO^T            (SS MMAs, K and V resident)
//        P^T, dS^T in registers (bf16 copies back to TMEM over dP^T)
//        dV += P^T dO, dK += dS^T Q            (A operand read from TMEM)
//   3. bwd_dq_tc_kernel: one CTA per 128 query rows, over the key tiles of the
//      forward's schedule, from separate K and V rings:
//        S = Q K^T, dP = dO V^T (two dP buffers), dS in registers,
//        dQ += dS K                            (A operand read from TMEM)
//      It forms D_i itself from O and dO, since it overwrites the scratch.
// Warp roles (320 threads): warps 0-7 two "softmax" warpgroups (each owns 64
// of a tile's 128 columns), warp 8 TMA producer, warp 9 MMA issuer and TMEM
// allocator. Every wait is bounded (see ptx.cuh).
#include <cuda_bf16.h>

#include <cmath>

#include "attn_jvp.h"
#include "kernels.cuh"
#include "ptx.cuh"
#include "tiles.cuh"

namespace ajvp {

namespace {

constexpr int kBB = 128;        // keys per dK/dV item, query rows per dQ item, tile size
constexpr int kBwdThreads = 320;
constexpr float kLog2eF = 1.4426950408889634f;

struct BwdTcParams {
  CUtensorMap map_q, map_k, map_v, map_do;  // [B, L, H, d] bf16, boxes of 64 columns x 128 rows
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;
  const float* lse;
  const float* dlse;  // or null
  float* scratch;     // the dq buffer as fp32: D [B H][Lp], then LSE log2(e) [B H][Lp]
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  unsigned int* status;
  int B, H, L, Lp, n_qt, n_kt;
  MaskSpec mask;
  float scale, scale_log2;
  GroupRange groups[kMaxGroups];  // mask.mode == kModeGroups: the row groups
};

// ---------------------------------------------------------------- prep
// One warp per (batch, head, row) of the padded length Lp.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __grid_constant__ BwdTcParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t total = static_cast<int64_t>(p.B) * p.H * p.Lp;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  float* d_out = p.scratch;
  float* l_out = p.scratch + total;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       r < total; r += warps) {
    const int64_t bh = r / p.Lp;
    const int i = static_cast<int>(r - bh * p.Lp);
    float dsum = 0.f, l2 = INFINITY;
    if (i < p.L) {
      const int b = static_cast<int>(bh / p.H), h = static_cast<int>(bh - int64_t(b) * p.H);
      const size_t off = ((static_cast<size_t>(b) * p.L + i) * p.H + h) * D;
      float acc = 0.f;
      if constexpr (D == 128) {
        const uint2 a = reinterpret_cast<const uint2*>(p.dout + off)[lane];
        const uint2 c = reinterpret_cast<const uint2*>(p.o + off)[lane];
        acc = bf16lo_to_f32(a.x) * bf16lo_to_f32(c.x) + bf16hi_to_f32(a.x) * bf16hi_to_f32(c.x) +
              bf16lo_to_f32(a.y) * bf16lo_to_f32(c.y) + bf16hi_to_f32(a.y) * bf16hi_to_f32(c.y);
      } else {
        const uint32_t a = reinterpret_cast<const uint32_t*>(p.dout + off)[lane];
        const uint32_t c = reinterpret_cast<const uint32_t*>(p.o + off)[lane];
        acc = bf16lo_to_f32(a) * bf16lo_to_f32(c) + bf16hi_to_f32(a) * bf16hi_to_f32(c);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      const size_t li = static_cast<size_t>(bh) * p.L + i;
      dsum = acc - (p.dlse ? p.dlse[li] : 0.f);
      l2 = p.lse[li] * kLog2eF;
    }
    if (lane == 0) {
      d_out[r] = dsum;
      l_out[r] = l2;
    }
  }
}

// ---------------------------------------------------------------- schedules
// Query tiles whose key-tile schedule (make_tile_sched, 128 x 128) lists key
// tile kt, in increasing order. The whole warp scans 32 query tiles at a
// time, one per lane, and keeps the visited and full ones as bit masks.
struct ColScan {
  int kt, n_qt, base;
  uint32_t vis, full;
};

// bq: rows of a query tile (the key tiles are kBB wide)
__device__ __forceinline__ void col_scan_load(const MaskSpec& m, ColScan& cs, int bq) {
  const int qt = cs.base + static_cast<int>(threadIdx.x & 31);
  bool v = false, f = false;
  if (qt < cs.n_qt) {
    const TileSched s = make_tile_sched(m, qt, bq, kBB);
    v = (cs.kt >= s.t1_begin && cs.kt < s.t1_end) || (cs.kt >= s.t2_begin && cs.kt < s.t2_end);
    f = v && s.full(cs.kt);
  }
  cs.vis = __ballot_sync(0xffffffffu, v);
  cs.full = __ballot_sync(0xffffffffu, f);
}

__device__ __forceinline__ void col_scan_start(const MaskSpec& m, ColScan& cs, int kt, int n_qt,
                                               int bq) {
  // Only the query tiles the mask can admit for this key tile: without the
  // bounds every warp scanned all query tiles of the sequence (tens of
  // microseconds per CTA).
  int lo, hi;
  key_tile_query_bounds(m, kt, kBB, n_qt, bq, lo, hi);
  cs.kt = kt;
  cs.n_qt = hi + 1;
  cs.base = lo;
  col_scan_load(m, cs, bq);
}

// The next visited query tile and whether every pair in it is admissible.
__device__ __forceinline__ bool col_next(const MaskSpec& m, ColScan& cs, int& qt, bool& full,
                                         int bq) {
  while (cs.vis == 0) {
    cs.base += 32;
    if (cs.base >= cs.n_qt) return false;
    col_scan_load(m, cs, bq);
  }
  const int bit = __ffs(cs.vis) - 1;
  qt = cs.base + bit;
  full = (cs.full >> bit) & 1u;
  cs.vis &= cs.vis - 1;
  return true;
}

// Per-lane bit masks of the admissible columns [c0, c0 + 64) of one row
// whose admissible set is [a0, a1) U [b0, b1).
__device__ __forceinline__ uint32_t bits_in(int s, int e, int q) {
  auto low = [](int n) -> uint32_t {
    return n <= 0 ? 0u : (n >= 32 ? 0xffffffffu : ((1u << n) - 1u));
  };
  return low(e - 32 * q) & ~low(s - 32 * q);
}

__device__ __forceinline__ void store_row_bf16(__nv_bfloat16* dst, const uint32_t (&pk)[16]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) d4[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
}

// ---------------------------------------------------------------- dK, dV
// Query tiles of 128 rows, as in the forward: the score MMAs are N = 128 wide
// (at N = 64 the tensor core takes about as long for half the work), and TMEM
// holds one S^T and one dP^T tile beside dV and dK (128 + 128 + 2 d columns).
// As in the forward, the softmax writes bf16 P^T and dS^T over dP^T (each
// warpgroup: P^T over the first 32 of its 64 columns, dS^T over the second
// 32), so S^T is free as soon as the softmax has read it, and S^T_{g+1} runs
// while the softmax finishes tile g.
template <int D>
struct DkdvCfg {
  static constexpr int CH = D / 64;
  static constexpr int TILE = kBB * D * 2;            // bytes of a [128 x D] bf16 tile
  static constexpr int QSLOT = TILE + 1024;           // Q, then LSE log2 e [128] and D [128]
  static constexpr int NQ = D == 128 ? 2 : 4;         // Q ring slots (released after dK)
  static constexpr int ND = D == 128 ? 2 : 4;         // dO ring slots (released after dV)
  static constexpr int DATA = 2 * TILE + NQ * QSLOT + ND * TILE;
  static constexpr int NBAR = 2 * NQ + 2 * ND + 10;
  static constexpr int BYTES = 1024 + DATA + NBAR * 8 + 16;
  // TMEM columns: S^T, dP^T (bf16 P^T and dS^T over it), dV, dK
  static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_P = TM_DP, TM_DS = TM_DP + 32;
  static constexpr uint32_t TM_DV = 256, TM_DK = 256 + D, TM_COLS = 512;
  static_assert(QSLOT % 1024 == 0 && TILE % 1024 == 0, "1024-byte aligned swizzled tiles");
  static_assert(BYTES <= 232448, "shared memory budget");
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_dkdv_tc_kernel(const __grid_constant__ BwdTcParams p) {
  using C = DkdvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sK = smem;
  uint8_t* sV = smem + C::TILE;
  uint8_t* sQ = smem + 2 * C::TILE;                  // [NQ] Q slots
  uint8_t* sDO = sQ + C::NQ * C::QSLOT;              // [ND] dO slots
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::DATA);
  uint64_t* q_full = bars;                           // [NQ]
  uint64_t* q_empty = bars + C::NQ;                  // [NQ]
  uint64_t* do_full = bars + 2 * C::NQ;              // [ND]
  uint64_t* do_empty = do_full + C::ND;              // [ND]
  uint64_t* kv_full = do_empty + C::ND;
  uint64_t* s_full = kv_full + 1;    // S^T of the current tile
  uint64_t* s_free = kv_full + 2;    // the softmax has read it
  uint64_t* dp_full = kv_full + 3;   // dP^T
  uint64_t* p_full = kv_full + 4;    // P^T (bf16) written
  uint64_t* ds_full = kv_full + 5;   // dS^T (bf16) written
  uint64_t* acc_full = kv_full + 6;  // dK, dV complete
  uint64_t* drain = kv_full + 7;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = warp_uniform(static_cast<int>(threadIdx.x >> 5));
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x / p.n_kt;
  const int kt = blockIdx.x - bh * p.n_kt;
  const int b = bh / p.H, h = bh - b * p.H;
  MaskSpec mask = p.mask;
  mask.groups = p.groups;
  auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
    return warp_wait(bar, parity, abort_flag, p.status);
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NQ; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < C::ND; ++i) {
      mbar_init(&do_full[i], 1);
      mbar_init(&do_empty[i], 1);
    }
    mbar_init(kv_full, 1);
    mbar_init(s_full, 1);
    mbar_init(s_free, 8);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 8);
    mbar_init(ds_full, 8);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, C::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(warp_uniform(static_cast<int>(*tmem_slot)));

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    // K and V of the block, then per visited query tile g: Q_g with its LSE
    // and D rows (Q ring), dO_g (dO ring).
    tma_prefetch_desc(&p.map_q);
    tma_prefetch_desc(&p.map_k);
    tma_prefetch_desc(&p.map_v);
    tma_prefetch_desc(&p.map_do);
    const uint64_t keep = l2_policy_evict_last();   // Q, dO: read by every key block of the head
    const uint64_t once = l2_policy_evict_first();  // K, V: this CTA only
    if (elect_one()) {
      mbar_arrive_expect_tx(kv_full, 2 * C::TILE);
#pragma unroll
      for (int c = 0; c < C::CH; ++c) {
        tma_load_4d_hint(sK + c * kBB * 128, &p.map_k, kv_full, c * 64, h, kt * kBB, b, once);
        tma_load_4d_hint(sV + c * kBB * 128, &p.map_v, kv_full, c * 64, h, kt * kBB, b, once);
      }
    }
    __syncwarp();
    const size_t total = static_cast<size_t>(p.B) * p.H * p.Lp;
    const float* d_row = p.scratch + static_cast<size_t>(bh) * p.Lp;
    const float* l_row = p.scratch + total + static_cast<size_t>(bh) * p.Lp;
    ColScan cs;
    col_scan_start(mask, cs, kt, p.n_qt, kBB);
    int qn = 0, dn = 0;  // Q and dO tiles issued
    bool ok = true;
    int qt;
    bool fl;
    while (col_next(mask, cs, qt, fl, kBB)) {
      const int g = qn;
      const uint32_t sq = g % C::NQ, sd = g % C::ND;
      if (!wwait(&q_empty[sq], ((g / C::NQ) & 1) ^ 1)) { ok = false; break; }
      uint8_t* qs = sQ + sq * C::QSLOT;
      if (elect_one()) {
        mbar_arrive_expect_tx(&q_full[sq], C::TILE + 2 * kBB * 4);
#pragma unroll
        for (int c = 0; c < C::CH; ++c)
          tma_load_4d_hint(qs + c * kBB * 128, &p.map_q, &q_full[sq], c * 64, h, qt * kBB, b, keep);
        bulk_load(qs + C::TILE, l_row + qt * kBB, kBB * 4, &q_full[sq]);
        bulk_load(qs + C::TILE + kBB * 4, d_row + qt * kBB, kBB * 4, &q_full[sq]);
      }
      __syncwarp();
      qn = g + 1;
      if (!wwait(&do_empty[sd], ((g / C::ND) & 1) ^ 1)) { ok = false; break; }
      if (elect_one()) {
        mbar_arrive_expect_tx(&do_full[sd], C::TILE);
#pragma unroll
        for (int c = 0; c < C::CH; ++c)
          tma_load_4d_hint(sDO + sd * C::TILE + c * kBB * 128, &p.map_do, &do_full[sd], c * 64, h,
                           qt * kBB, b, keep);
      }
      __syncwarp();
      dn = g + 1;
    }
    if (!ok && lane == 0) {
      // Abort: let every copy already issued land before the CTA exits.
      mbar_wait_drain(kv_full, 0, 200000000ull);
      for (int j = qn - 1; j >= 0 && j >= qn - C::NQ; --j)
        mbar_wait_drain(&q_full[j % C::NQ], (j / C::NQ) & 1, 200000000ull);
      for (int j = dn - 1; j >= 0 && j >= dn - C::ND; --j)
        mbar_wait_drain(&do_full[j % C::ND], (j / C::ND) & 1, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // Per tile g (all single TMEM buffers):
    //   C: S^T_{g+1} = K Q_{g+1}^T   once the softmax has read S^T_g (s_free)
    //   A: dV += P^T_g dO_g          after P^T_g (p_full)
    //   B: dK += dS^T_g Q_g          after dS^T_g (ds_full)
    //   E: dP^T_{g+1} = V dO_{g+1}^T over the columns of P^T_g and dS^T_g:
    //      one thread's tcgen05.mma execute in order, so it follows A and B.
    // The softmax releases S^T_g before P^T_g is ready, so waiting for s_free
    // first never delays A and B.
    const uint32_t idesc_s = idesc_bf16_f32(128, kBB, 0);
    const uint32_t idesc_v = idesc_bf16_f32(128, D, 1);
    const uint32_t aK = smem_u32(sK), aV = smem_u32(sV);
    const uint32_t aQ0 = smem_u32(sQ), aD0 = smem_u32(sDO);
    auto q_addr = [&](int g) { return aQ0 + (g % C::NQ) * C::QSLOT; };
    auto do_addr = [&](int g) { return aD0 + (g % C::ND) * C::TILE; };
    auto issue_s = [&](int j) -> bool {
      if (!wwait(&q_full[j % C::NQ], (j / C::NQ) & 1)) return false;
      tc_fence_after();
      mma_scores<D, kBB, kBB, false>(tmem + C::TM_S, aK, q_addr(j), idesc_s, false);
      umma_commit(s_full);
      return true;
    };
    auto issue_dp = [&](int j) -> bool {
      if (!wwait(&do_full[j % C::ND], (j / C::ND) & 1)) return false;
      tc_fence_after();
      mma_scores<D, kBB, kBB, false>(tmem + C::TM_DP, aV, do_addr(j), idesc_s, false);
      umma_commit(dp_full);
      return true;
    };
    ColScan cs;
    col_scan_start(mask, cs, kt, p.n_qt, kBB);
    int qt;
    bool fl;
    bool ok = wwait(kv_full, 0);
    bool has = ok && col_next(mask, cs, qt, fl, kBB);
    if (has) ok = issue_s(0) && issue_dp(0);
    for (int g = 0; ok && has; ++g) {
      const uint32_t ph = g & 1;
      const bool next = col_next(mask, cs, qt, fl, kBB);
      // C
      if (next && (!wwait(s_free, ph) || !issue_s(g + 1))) break;
      // A
      if (!wwait(p_full, ph)) break;
      tc_fence_after();
      mma_values_split<kBB, false>(tmem + C::TM_DV, tmem + C::TM_P, do_addr(g), idesc_v, g > 0);
      umma_commit(&do_empty[g % C::ND]);
      // B
      if (!wwait(ds_full, ph)) break;
      tc_fence_after();
      mma_values_split<kBB, false>(tmem + C::TM_DK, tmem + C::TM_DS, q_addr(g), idesc_v, g > 0);
      umma_commit(&q_empty[g % C::NQ]);
      if (!next) {
        umma_commit(acc_full);
        break;
      }
      // E
      if (!issue_dp(g + 1)) break;
    }
    // Every MMA issued so far completes before TMEM is released.
    umma_commit(drain);
    if (lane == 0) mbar_wait_drain(drain, 0, 1000000000ull);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // Thread (wg, sub, lane) owns key row 32 sub + lane (its TMEM lane) and the
    // query columns [64 wg, 64 wg + 64) of every 128-row query tile.
    const int wg = warp >> 2, sub = warp & 3;
    const int row = sub * 32 + lane;
    const int key = kt * kBB + row;
    const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::TM_S + 64 * wg;
    const uint32_t tDP = tmem + lane_off + C::TM_DP + 64 * wg;
    const uint32_t tDV = tmem + lane_off + C::TM_DV + (D / 2) * wg;
    const uint32_t tDK = tmem + lane_off + C::TM_DK + (D / 2) * wg;
    const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
    ColScan cs;
    col_scan_start(mask, cs, kt, p.n_qt, kBB);
    int g = 0;
    bool ok = true;
    int qt;
    bool fl;
    while (col_next(mask, cs, qt, fl, kBB)) {
      const uint32_t ph = g & 1;
      const float* lse2 =
          reinterpret_cast<const float*>(sQ + (g % C::NQ) * C::QSLOT + C::TILE) + 64 * wg;
      const float* dd = lse2 + kBB;
      // the tile's LSE and D are read from shared memory: observe its copies
      if (!wwait(&q_full[g % C::NQ], (g / C::NQ) & 1)) { ok = false; break; }
      if (!wwait(s_full, ph)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      // S^T_g is in registers: the MMA warp may write S^T_{g+1}
      tc_fence_before();
      __syncwarp();
      mbar_arrive_if(s_free, lane == 0);
      if (!fl) {
        // Admissible query columns of this key: the rows of the warpgroup's
        // 64 columns fall into a few row groups (rows with one admissible key
        // set); each group admits this key for all its rows or for none. Every
        // step advances at least one row (past the last row group, as for the
        // padding rows beyond L, the next group start does not advance), so
        // the loop ends after at most 64 steps.
        const int i0 = qt * kBB + 64 * wg;
        uint32_t m0 = 0u, m1 = 0u;
#pragma unroll 1
        for (int i = i0; i < i0 + 64;) {
          const RowRange rr = row_range(mask, i);
          const int e = max(min(next_group_start(mask, i), i0 + 64), i + 1);
          if (row_allows(rr, key)) {
            m0 |= bits_in(i - i0, e - i0, 0);
            m1 |= bits_in(i - i0, e - i0, 1);
          }
          i = e;
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (!((m0 >> j) & 1u)) sr[j] = __float_as_uint(-INFINITY);
          if (!((m1 >> j) & 1u)) sr[32 + j] = __float_as_uint(-INFINITY);
        }
      }
      // P^T = 2^(S^T s log2 e - LSE_i log2 e): 0 where masked or past L
      uint32_t pk[32];
#pragma unroll
      for (int j = 0; j < 64; j += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(lse2 + j);
        const float2 x01 = __ffma2_rn(make_float2(__uint_as_float(sr[j]), __uint_as_float(sr[j + 1])),
                                      sc2, make_float2(-l4.x, -l4.y));
        const float2 x23 = __ffma2_rn(make_float2(__uint_as_float(sr[j + 2]), __uint_as_float(sr[j + 3])),
                                      sc2, make_float2(-l4.z, -l4.w));
        const float p0 = ex2_approx(x01.x), p1 = ex2_approx(x01.y);
        const float p2 = ex2_approx(x23.x), p3 = ex2_approx(x23.y);
        sr[j] = __float_as_uint(p0);
        sr[j + 1] = __float_as_uint(p1);
        sr[j + 2] = __float_as_uint(p2);
        sr[j + 3] = __float_as_uint(p3);
        pk[j / 2] = pack_bf16x2(p0, p1);
        pk[j / 2 + 1] = pack_bf16x2(p2, p3);
      }
      // dS^T = P^T (dP^T - D_i) on pairs of floats, in two halves of 32
      // queries: P^T goes over the first half of this warpgroup's dP^T columns
      // once it is read, dS^T over the second.
      if (!wwait(dp_full, ph)) { ok = false; break; }
      tc_fence_after();
      uint32_t dk[32];
      auto ds_half = [&](int hq, const uint32_t (&v)[32]) {
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float2 d2 = *reinterpret_cast<const float2*>(dd + 32 * hq + j);
          const float2 ds = __fmul2_rn(
              make_float2(__uint_as_float(sr[32 * hq + j]), __uint_as_float(sr[32 * hq + j + 1])),
              __fadd2_rn(make_float2(__uint_as_float(v[j]), __uint_as_float(v[j + 1])),
                         make_float2(-d2.x, -d2.y)));
          dk[16 * hq + j / 2] = pack_bf16x2(ds.x, ds.y);
        }
      };
      {
        uint32_t v[32];
        tmem_ld32(tDP, v);
        tmem_wait_ld();
        ds_half(0, v);
      }
      tmem_st32(tDP, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      mbar_arrive_if(p_full, lane == 0);
      {
        uint32_t v[32];
        tmem_ld32(tDP + 32, v);
        tmem_wait_ld();
        ds_half(1, v);
      }
      tmem_st32(tDP + 32, dk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      mbar_arrive_if(ds_full, lane == 0);
      ++g;
    }
    // ---------------- epilogue: dV, s dK of this key (zero if no query sees it)
    if (ok) {
      const bool any = g > 0;
      if (any && !wwait(acc_full, 0)) ok = false;
      if (ok) {
        tc_fence_after();
        const bool valid = key < p.L;
        const size_t off = ((static_cast<size_t>(b) * p.L + (valid ? key : 0)) * p.H + h) * D +
                           (D / 2) * wg;
#pragma unroll 1
        for (int c = 0; c < D / 64; ++c) {
          uint32_t a[32], t[32];
          if (any) {
            tmem_ld32(tDV + 32 * c, a);
            tmem_ld32(tDK + 32 * c, t);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) a[j] = t[j] = 0u;
          }
          uint32_t pv[16], pkk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            pv[j] = pack_bf16x2(__uint_as_float(a[2 * j]), __uint_as_float(a[2 * j + 1]));
            pkk[j] = pack_bf16x2(__uint_as_float(t[2 * j]) * p.scale,
                                 __uint_as_float(t[2 * j + 1]) * p.scale);
          }
          if (valid) {
            store_row_bf16(p.dv + off + 32 * c, pv);
            store_row_bf16(p.dk + off + 32 * c, pkk);
          }
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, C::TM_COLS);
}

// ---------------------------------------------------------------- dQ
template <int D>
struct DqCfg {
  static constexpr int CH = D / 64;
  static constexpr int TILE = kBB * D * 2;
  // Two rings: K_j is read by S_j (early) and dQ_j (late), V_j only by dP_j
  // (early), so each ring is released at its own pace and a V load need not
  // wait for a K slot.
  static constexpr int NK = D == 128 ? 3 : 4;         // K ring slots
  static constexpr int NV = D == 128 ? 2 : 4;         // V ring slots
  static constexpr int NP = NK + NV;
  static constexpr int DATA = 2 * TILE + NP * TILE;   // Q, dO resident, then the rings
  static constexpr int XCH = 2 * kBB * 4;             // partial dO.O exchange [2][128]
  static constexpr int NBAR = 2 * NP + 9 + 4;
  static constexpr int BYTES = 1024 + DATA + XCH + NBAR * 8 + 16;
  // TMEM columns: S, dP (two buffers; dS over the first half of each
  // warpgroup's slice), dQ
  static constexpr uint32_t TM_S = 0, TM_DP0 = 128, TM_DQ = 256, TM_DP1 = 384, TM_COLS = 512;
  static_assert(BYTES <= 232448, "shared memory budget");
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_dq_tc_kernel(const __grid_constant__ BwdTcParams p) {
  using C = DqCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sDO = smem + C::TILE;
  uint8_t* sRing = smem + 2 * C::TILE;
  float* xch = reinterpret_cast<float*>(smem + C::DATA);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::DATA + C::XCH);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::NP;
  uint64_t* q_full = bars + 2 * C::NP;
  uint64_t* s_full = q_full + 1;
  uint64_t* s_free = q_full + 2;
  // dp_full and ds_full come one per dP buffer: the MMA warp issues
  // dP_{j+1} before it waits for dS_j, so the softmax may finish tile j+1
  // before that wait; with one barrier its phase could then run two ahead.
  uint64_t* dp_full = q_full + 3;   // [2]
  uint64_t* ds_full = q_full + 5;   // [2]
  uint64_t* acc_full = q_full + 7;
  uint64_t* drain = q_full + 8;
  uint64_t* xa = q_full + 9;        // [4] partial-D exchange (once per CTA)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = warp_uniform(static_cast<int>(threadIdx.x >> 5));
  const int lane = threadIdx.x & 31;
  // Items in reverse query-tile order within a head: under causal masks the
  // last query tiles see the most keys, so the longest items start first.
  const int bh = blockIdx.x / p.n_qt;
  const int qt = p.n_qt - 1 - (blockIdx.x - bh * p.n_qt);
  const int b = bh / p.H, h = bh - b * p.H;
  MaskSpec mask = p.mask;
  mask.groups = p.groups;
  const TileSched sch = warp_uniform(make_tile_sched(mask, qt, kBB, kBB));
  const int cnt = sch.count();
  auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
    return warp_wait(bar, parity, abort_flag, p.status);
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NP; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(s_full, 1);
    mbar_init(s_free, 8);
    mbar_init(&dp_full[0], 1);
    mbar_init(&dp_full[1], 1);
    mbar_init(&ds_full[0], 8);
    mbar_init(&ds_full[1], 8);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&xa[i], 64);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, C::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(warp_uniform(static_cast<int>(*tmem_slot)));

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    // Ring elements in order of first use: K_j, then V_j, per key tile j.
    tma_prefetch_desc(&p.map_q);
    tma_prefetch_desc(&p.map_k);
    tma_prefetch_desc(&p.map_v);
    tma_prefetch_desc(&p.map_do);
    const uint64_t keep = l2_policy_evict_last();   // K, V: read by every query block of the head
    const uint64_t once = l2_policy_evict_first();  // Q, dO: this CTA only
    if (cnt > 0 && elect_one()) {
      mbar_arrive_expect_tx(q_full, 2 * C::TILE);
#pragma unroll
      for (int c = 0; c < C::CH; ++c) {
        tma_load_4d_hint(sQ + c * kBB * 128, &p.map_q, q_full, c * 64, h, qt * kBB, b, once);
        tma_load_4d_hint(sDO + c * kBB * 128, &p.map_do, q_full, c * 64, h, qt * kBB, b, once);
      }
    }
    __syncwarp();
    // ring slot of K_j: j % NK; of V_j: NK + j % NV
    int k_issued = 0, v_issued = 0;
    bool ok = true;
    for (int idx = 0; ok && idx < cnt; ++idx) {
      const int kt = sch.tile(idx);
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const int n = which == 0 ? C::NK : C::NV;
        const uint32_t el = (which == 0 ? 0 : C::NK) + idx % n;
        if (!wwait(&empty[el], ((idx / n) & 1) ^ 1)) { ok = false; break; }
        if (elect_one()) {
          mbar_arrive_expect_tx(&full[el], C::TILE);
          const CUtensorMap* map = which == 0 ? &p.map_k : &p.map_v;
#pragma unroll
          for (int c = 0; c < C::CH; ++c)
            tma_load_4d_hint(sRing + el * C::TILE + c * kBB * 128, map, &full[el], c * 64, h,
                             kt * kBB, b, keep);
        }
        __syncwarp();
        if (which == 0)
          k_issued = idx + 1;
        else
          v_issued = idx + 1;
      }
    }
    if (!ok && lane == 0) {
      // Abort: let every copy already issued land before the CTA exits.
      if (cnt > 0) mbar_wait_drain(q_full, 0, 200000000ull);
      for (int j = k_issued - 1; j >= 0 && j >= k_issued - C::NK; --j)
        mbar_wait_drain(&full[j % C::NK], (j / C::NK) & 1, 200000000ull);
      for (int j = v_issued - 1; j >= 0 && j >= v_issued - C::NV; --j)
        mbar_wait_drain(&full[C::NK + j % C::NV], (j / C::NV) & 1, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // Per key tile j: once the softmax has read S_j, S_{j+1} and dP_{j+1}
    // (into the other dP buffer); then dQ += dS_j K_j. dP_{j+1} overwrites
    // the buffer that dQ_{j-1} read, which was issued before it.
    const uint32_t idesc_s = idesc_bf16_f32(128, kBB, 0);
    const uint32_t idesc_v = idesc_bf16_f32(128, D, 1);
    const uint32_t aQ = smem_u32(sQ), aDO = smem_u32(sDO), aRing = smem_u32(sRing);
    // K_j in slot j % NK, V_j in slot NK + j % NV
    auto k_slot = [&](int j) { return static_cast<uint32_t>(j % C::NK); };
    auto v_slot = [&](int j) { return static_cast<uint32_t>(C::NK + j % C::NV); };
    auto k_ph = [&](int j) { return static_cast<uint32_t>((j / C::NK) & 1); };
    auto v_ph = [&](int j) { return static_cast<uint32_t>((j / C::NV) & 1); };
    auto el_addr = [&](uint32_t slot) { return aRing + slot * C::TILE; };
    auto tm_dp = [&](int j) { return tmem + ((j & 1) ? C::TM_DP1 : C::TM_DP0); };
    if (cnt > 0) {
      bool ok = wwait(q_full, 0) && wwait(&full[k_slot(0)], 0);
      if (ok) {
        tc_fence_after();
        mma_scores<D, kBB, kBB, false>(tmem + C::TM_S, aQ, el_addr(k_slot(0)), idesc_s, false);
        umma_commit(s_full);
        ok = wwait(&full[v_slot(0)], 0);
      }
      if (ok) {
        tc_fence_after();
        mma_scores<D, kBB, kBB, false>(tm_dp(0), aDO, el_addr(v_slot(0)), idesc_s, false);
        umma_commit(&dp_full[0]);
        umma_commit(&empty[v_slot(0)]);
      }
      for (int idx = 0; ok && idx < cnt; ++idx) {
        const uint32_t ph = idx & 1;
        if (idx + 1 < cnt) {
          const int j = idx + 1;
          if (!wwait(s_free, ph) || !wwait(&full[k_slot(j)], k_ph(j))) break;
          tc_fence_after();
          mma_scores<D, kBB, kBB, false>(tmem + C::TM_S, aQ, el_addr(k_slot(j)), idesc_s, false);
          umma_commit(s_full);
          if (!wwait(&full[v_slot(j)], v_ph(j))) break;
          tc_fence_after();
          mma_scores<D, kBB, kBB, false>(tm_dp(j), aDO, el_addr(v_slot(j)), idesc_s, false);
          umma_commit(&dp_full[j & 1]);
          umma_commit(&empty[v_slot(j)]);
        }
        if (!wwait(&ds_full[idx & 1], (idx >> 1) & 1)) break;
        tc_fence_after();
        mma_values_split<kBB, false>(tmem + C::TM_DQ, tm_dp(idx), el_addr(k_slot(idx)), idesc_v,
                                     idx > 0);
        umma_commit(&empty[k_slot(idx)]);
        if (idx == cnt - 1) umma_commit(acc_full);
      }
    }
    umma_commit(drain);
    if (lane == 0) mbar_wait_drain(drain, 0, 1000000000ull);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // Thread (wg, sub, lane) owns query row 32 sub + lane and the key columns
    // [64 wg, 64 wg + 64) of every tile, and output columns [D/2 wg, D/2 wg + D/2).
    const int wg = warp >> 2, sub = warp & 3;
    const int row = sub * 32 + lane;
    const int t = qt * kBB + row;
    const bool valid = t < p.L;
    const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::TM_S + 64 * wg;
    const uint32_t tDQ = tmem + lane_off + C::TM_DQ + (D / 2) * wg;
    const float sl2 = p.scale_log2;
    bool ok = true;
    // D_t = dO_t . O_t - dLSE_t from this warpgroup's half of the row and the
    // other warpgroup's half (exchanged through shared memory).
    float part = 0.f;
    const size_t row_off =
        ((static_cast<size_t>(b) * p.L + (valid ? t : 0)) * p.H + h) * D + (D / 2) * wg;
    if (valid) {
      const uint4* a4 = reinterpret_cast<const uint4*>(p.dout + row_off);
      const uint4* c4 = reinterpret_cast<const uint4*>(p.o + row_off);
#pragma unroll
      for (int q = 0; q < D / 16; ++q) {
        const uint4 a = a4[q], c = c4[q];
        part += bf16lo_to_f32(a.x) * bf16lo_to_f32(c.x) + bf16hi_to_f32(a.x) * bf16hi_to_f32(c.x) +
                bf16lo_to_f32(a.y) * bf16lo_to_f32(c.y) + bf16hi_to_f32(a.y) * bf16hi_to_f32(c.y) +
                bf16lo_to_f32(a.z) * bf16lo_to_f32(c.z) + bf16hi_to_f32(a.z) * bf16hi_to_f32(c.z) +
                bf16lo_to_f32(a.w) * bf16lo_to_f32(c.w) + bf16hi_to_f32(a.w) * bf16hi_to_f32(c.w);
      }
    }
    xch[wg * kBB + row] = part;
    mbar_arrive(&xa[sub]);
    if (!warp_wait(&xa[sub], 0, abort_flag, p.status)) ok = false;
    float d_row = 0.f, lse2 = INFINITY;
    if (ok) {
      const float other = xch[(1 - wg) * kBB + row];
      if (valid) {
        const size_t li = static_cast<size_t>(bh) * p.L + t;
        // both warpgroups add the halves in the same order: identical D_t
        d_row = (wg == 0 ? part + other : other + part) - (p.dlse ? p.dlse[li] : 0.f);
        lse2 = p.lse[li] * kLog2eF;
      }
    }
    const RowRange rr = row_range(mask, t);
    for (int idx = 0; ok && idx < cnt; ++idx) {
      const uint32_t ph = idx & 1;
      const int kt = sch.tile(idx);
      const bool full_tile = sch.full(kt);
      if (!wwait(s_full, ph)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      mbar_arrive_if(s_free, lane == 0);  // S_j is in registers: S_{j+1} may be written
      if (!full_tile) {
        const int k0 = kt * kBB + 64 * wg;
        const int s1 = min(max(rr.a0 - k0, 0), 64), e1 = min(max(rr.a1 - k0, 0), 64);
        const int s2 = min(max(rr.b0 - k0, 0), 64), e2 = min(max(rr.b1 - k0, 0), 64);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const uint32_t m = bits_in(s1, e1, q) | bits_in(s2, e2, q);
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (!((m >> j) & 1u)) sr[32 * q + j] = __float_as_uint(-INFINITY);
        }
      }
      {
        const float2 sc2 = make_float2(sl2, sl2), nl2 = make_float2(-lse2, -lse2);
#pragma unroll
        for (int j = 0; j < 64; j += 2) {
          const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[j]), __uint_as_float(sr[j + 1])),
                                      sc2, nl2);
          sr[j] = __float_as_uint(ex2_approx(x.x));
          sr[j + 1] = __float_as_uint(ex2_approx(x.y));
        }
      }
      if (!wwait(&dp_full[idx & 1], (idx >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tDP = tmem + lane_off + ((idx & 1) ? C::TM_DP1 : C::TM_DP0) + 64 * wg;
      uint32_t v[32], pk[32];
      tmem_ld32(tDP, v);
      tmem_wait_ld();
      // dS = P (dP - D_t) on pairs of floats (FADD2, FMUL2)
      const float2 nd2 = make_float2(-d_row, -d_row);
      auto ds_pair = [&](int c, uint32_t v0, uint32_t v1) -> uint32_t {
        const float2 ds = __fmul2_rn(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])),
                                     __fadd2_rn(make_float2(__uint_as_float(v0), __uint_as_float(v1)), nd2));
        return pack_bf16x2(ds.x, ds.y);
      };
#pragma unroll
      for (int j = 0; j < 32; j += 2) pk[j / 2] = ds_pair(j, v[j], v[j + 1]);
      tmem_ld32(tDP + 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; j += 2) pk[16 + j / 2] = ds_pair(32 + j, v[j], v[j + 1]);
      tmem_st32(tDP, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      mbar_arrive_if(&ds_full[idx & 1], lane == 0);
    }
    // ---------------- epilogue: s dQ of this row
    if (ok) {
      const bool any = cnt > 0;
      if (any && !wwait(acc_full, 0)) ok = false;
      if (ok) {
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < D / 64; ++c) {
          uint32_t a[32];
          if (any) {
            tmem_ld32(tDQ + 32 * c, a);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) a[j] = 0u;
          }
          uint32_t pq[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            pq[j] = pack_bf16x2(__uint_as_float(a[2 * j]) * p.scale,
                                __uint_as_float(a[2 * j + 1]) * p.scale);
          if (valid) store_row_bf16(p.dq + row_off + 32 * c, pq);
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, C::TM_COLS);
}

template <int D>
cudaError_t launch_bwd_tc(const BwdTcParams& p, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(p.B) * p.H * p.Lp;
  const int64_t blocks = (rows + 7) / 8;
  bwd_prep_kernel<D><<<static_cast<unsigned>(blocks < 148 * 64 ? blocks : 148 * 64), 256, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_dkdv_tc_kernel<D><<<static_cast<unsigned>(p.B * p.H * p.n_kt), kBwdThreads,
                          DkdvCfg<D>::BYTES, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_dq_tc_kernel<D><<<static_cast<unsigned>(p.B * p.H * p.n_qt), kBwdThreads, DqCfg<D>::BYTES,
                        stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t bwd_tc_prepare() {
  cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_tc_kernel<128>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       DkdvCfg<128>::BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(bwd_dkdv_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DkdvCfg<64>::BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(bwd_dq_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DqCfg<128>::BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(bwd_dq_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DqCfg<64>::BYTES);
  return e;
}

int64_t bwd_tc_padded_len(int64_t L) { return (L + kBB - 1) / kBB * kBB; }

bool bwd_tc_supported(int64_t B, int64_t L, int64_t H, int64_t d) {
  if (d != 64 && d != 128) return false;
  // scratch (D and LSE log2 e, fp32, padded rows) must fit in the bf16 dq buffer
  if (8 * bwd_tc_padded_len(L) > 2 * d * L) return false;
  const int64_t tiles = (L + kBB - 1) / kBB;
  return B * H * tiles < (int64_t(1) << 31) - 1;
}

int bwd_tc_launch(const BwdTcArgs& a, cudaStream_t stream) {
  static thread_local BwdTcParams p;  // large (group table): not on the stack
  unsigned int* status = nullptr;
  const int rc = device_status_word(&status);
  if (rc != ATTN_JVP_OK) return rc;
  if (!encode_bf16_rows_map(&p.map_q, a.q, a.B, a.L, a.H, a.d, kBB) ||
      !encode_bf16_rows_map(&p.map_k, a.k, a.B, a.L, a.H, a.d, kBB) ||
      !encode_bf16_rows_map(&p.map_v, a.v, a.B, a.L, a.H, a.d, kBB) ||
      !encode_bf16_rows_map(&p.map_do, a.dout, a.B, a.L, a.H, a.d, kBB))
    return ATTN_JVP_ERR_CUDA;
  p.o = static_cast<const __nv_bfloat16*>(a.o);
  p.dout = static_cast<const __nv_bfloat16*>(a.dout);
  p.lse = a.lse;
  p.dlse = a.dlse;
  p.scratch = static_cast<float*>(a.dq);
  p.dq = static_cast<__nv_bfloat16*>(a.dq);
  p.dk = static_cast<__nv_bfloat16*>(a.dk);
  p.dv = static_cast<__nv_bfloat16*>(a.dv);
  p.status = status;
  p.B = static_cast<int>(a.B);
  p.H = static_cast<int>(a.H);
  p.L = static_cast<int>(a.L);
  p.Lp = static_cast<int>(bwd_tc_padded_len(a.L));
  p.n_qt = p.Lp / kBB;
  p.n_kt = p.n_qt;
  p.mask = a.mask;
  if (a.mask.mode == kModeGroups)
    for (int i = 0; i < a.mask.n_groups; ++i) p.groups[i] = a.mask.groups[i];
  p.mask.groups = nullptr;  // the kernels point it at their own parameter copy
  p.scale = a.scale;
  p.scale_log2 = a.scale * kLog2eF;
  const cudaError_t e = a.d == 128 ? launch_bwd_tc<128>(p, stream) : launch_bwd_tc<64>(p, stream);
  return e == cudaSuccess ? ATTN_JVP_OK : ATTN_JVP_ERR_CUDA;
}

}  // namespace ajvp
