// attn_jvp_tc.cu - bf16 custom-mask attention forward fused with its JVP on
// sm_100a tensor cores (tcgen05 MMA, TMEM accumulators, TMA tile loads).
//
// Causal-rCM summary page, App. B: one online-softmax pass computes the primal
// output and the tangent output with shared rescaling; masked entries get no
// tangent; the same sparse (query tile x key range) schedule drives the primal
// and tangent scores; queries and keys are tiled; outputs are O, LSE and tO.
//
// Per query tile (128 rows per CTA, one TMEM lane per row) and admissible key
// tile j (128 keys), with s the softmax scale and x = s log2(e) Q K^T:
//   MMA   S_j   = Q K_j^T                      (TMEM cols [0,128),   fp32)
//   MMA   tS'_j = tQ K_j^T + Q tK_j^T          (TMEM cols [128,256), fp32)
//   warps p = 2^(x - m), l += sum p;  u = p * s * tS', D += sum u;
//         P and U (bf16) written back over tS' (each warpgroup's 64 columns:
//         32 of P, then 32 of U), which frees the S columns for S_{j+1}
//         while the softmax of tile j is still running
//   MMA   A += P V_j                           (d = 128: TMEM cols [256,384))
//   MMA   T += U V_j + P tV_j                  (d = 128: TMEM cols [384,512))
//         (d = 64: T at [256,320) and A at [320,384), so that P tV and P V
//         are one N = 128 MMA group over the adjacent tV and V tiles)
//   end   O = A/l, mu = D/l, tO = T/l - mu O, LSE = (m + log2 l) ln 2
// which is tO = sum_j P_ij (tS_ij - mu_i) v_j + sum_j P_ij tv_j with
// tS = s (tQ K^T + Q tK^T), i.e. tP V + P tV, tP = P (tS - rowsum(P tS)).
//
// The running max m is only raised (and A, T, l, D rescaled by 2^(m_old -
// m_new)) when a tile's max exceeds it by more than kRescaleTau: every p stays
// <= 2^kRescaleTau and the final normalisation by l is exact.
//
// Head dim 128 runs on CTA pairs (clusters of two SMs, cta_group::2 MMAs over
// 256 query rows, each SM holding half of every key/value tile); head dim 64
// on single CTAs. Warp roles (320 threads, one CTA per SM, persistent):
//   warps 0-7  softmax + epilogue: two warpgroups, each owning half of the
//              key columns of a tile (and half of the output columns)
//   warp  8    TMA producer (warp-wide, one elected lane issues): Q,tQ per
//              item; (K,tK) and (tV,V) ring elements per key tile
//   warp  9    MMA issuer (warp-wide, elect.sync; the pair's leader only),
//              TMEM allocator
// Work items (batch, head, query row block) are handed out head by head so
// that units running at the same time share one head's keys in L2: from host
// work lists (each block, longest first, to the unit with the least work), or
// in snake rounds over a longest-first order when the lists do not fit.
// No TMA multicast is used anywhere: each CTA loads its own tiles (a pair's
// copies complete on the leader's barriers, the cta_group::2 form).
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx.cuh"
#include "rope_math.cuh"
#include "tiles.cuh"

namespace ajvp {

constexpr float kRescaleTau = 8.0f;
constexpr float kLn2 = 0.69314718055994530942f;

// Event clocks of CTA kTraceCta for its first kTraceTiles key tiles (trace builds only).
#ifdef AJVP_TRACE
#define AJVP_EV(tile, ev)                                                             \
  do {                                                                                \
    if (p.trace && blockIdx.x == kTraceCta && (tile) < kTraceTiles)                   \
      p.trace[(tile) * kTraceEvents + (ev)] = static_cast<long long>(clock64());      \
  } while (0)
// Clock read issued after the register holding x is available.
__device__ __forceinline__ long long clock_after(float x) {
  long long t;
  asm volatile("{\n\t.reg .pred q;\n\tsetp.eq.f32 q, %1, 0f46404C00;\n\tmov.u64 %0, %%clock64;\n\t}"
               : "=l"(t) : "f"(x));
  return t;
}
#define AJVP_EVX(tile, ev, val)                                                      \
  do {                                                                               \
    if (p.trace && blockIdx.x == kTraceCta && (tile) < kTraceTiles)                  \
      p.trace[(tile) * kTraceEvents + (ev)] = clock_after(val);                      \
  } while (0)
#else
#define AJVP_EVX(tile, ev, val) \
  do {                          \
  } while (0)
#define AJVP_EV(tile, ev) \
  do {                    \
  } while (0)
#endif

// PAIR: a cluster of two CTAs runs cta_group::2 MMAs over 256 query rows
// (128 per CTA); each CTA holds half of every K/V-type tile: 64 of the 128
// keys of K and tK, 64 of the D columns of V and tV. d = 128 runs on pairs,
// d = 64 on single CTAs; either way a tile (or half tile) is 16 KB, and the
// shared-memory ring holds NP elements of two tiles each: (K_j, tK_j) or
// (tV_j, V_j), each with one full and one empty barrier.
template <int D, bool PAIR>
struct TcCfg {
  static constexpr int BM = kTcBlockM;            // query rows per CTA
  static constexpr int BMU = PAIR ? 2 * BM : BM;  // query rows per work item
  static constexpr int BN = kTcBlockN;
  static constexpr int CH = D / 64;               // 128-byte swizzle chunks per row
  static constexpr int KROWS = PAIR ? BN / 2 : BN;  // key rows of a K-type tile held here
  static constexpr int VCH = PAIR ? CH / 2 : CH;    // 64-column chunks of a V-type tile held here
  static constexpr int TILE = KROWS * D * 2;      // bytes of one K/V-type tile (or half tile)
  static constexpr int QBYTES = BM * D * 2;       // bytes of the Q (or tQ) tile
  static constexpr int NP = 5;                    // ring elements (two tiles each)
  static constexpr int M_MMA = PAIR ? 2 * BM : BM;
  static_assert(PAIR == (D == 128), "d = 128 runs on CTA pairs, d = 64 on single CTAs");
  static_assert(KROWS * D == BN * VCH * 64, "K-type and V-type tiles fill a slot alike");
  static_assert(TILE == 16384, "16 KB tiles");
  static constexpr int DATA = 2 * QBYTES + NP * 2 * TILE;
  static constexpr int XCH = 2 * BM * 4 + 32;     // row statistics [2][BM] floats + flags [2][4]
  static constexpr int NBAR = 2 * NP + 9 + 8 + 2;  // + peer_done, stall
  static constexpr int BYTES = 1024 + DATA + XCH + NBAR * 8 + 32;
  static constexpr int ARRIVALS = PAIR ? 16 : 8;  // softmax warps arriving on s_free, p_full, u_full
  static constexpr int HALF = BN / 2;             // key columns per softmax warpgroup
  static constexpr int DH = D / 2;                // output columns per softmax warpgroup
  static constexpr uint32_t TM_S = 0;
  static constexpr uint32_t TM_TS = 128;
  static constexpr uint32_t TM_P = TM_TS;       // bf16 P over the first half of each warpgroup's tS'
  static constexpr uint32_t TM_U = TM_TS + 32;  // bf16 U over the second half
  // d = 64: T then A, adjacent, so that one N = 128 group writes [P tV | P V]
  // from the adjacent (tV, V) tiles of a ring element
  static constexpr uint32_t TM_A = PAIR ? 256 : 256 + D;
  static constexpr uint32_t TM_T = PAIR ? 256 + D : 256;
  static constexpr uint32_t TM_COLS = 512;
  static_assert(BYTES <= 232448, "shared memory budget");
  static_assert(TM_T + D <= TM_COLS && TM_A + D <= TM_COLS, "TMEM budget");
};

// Bit mask of the lowest n bits (n clamped to [0, 32]).
__device__ __forceinline__ uint32_t low_bits(int n) {
  return n <= 0 ? 0u : (n >= 32 ? 0xffffffffu : ((1u << n) - 1u));
}

struct WorkItem {
  int b, h, qt;
};

__device__ __forceinline__ int item_position(int k, int cta, int G) {
  return (k & 1) ? k * G + (G - 1 - cta) : k * G + cta;
}

// The unit's k-th work item (work lists), or its first item at snake round
// >= k (k is advanced to it).
__device__ __forceinline__ bool next_item_lane(const TcParams& p, int cta, int G, int& k, int& pos) {
  if (p.list_mode) {
    const int i = p.unit_start[cta] + k;
    if (i >= p.unit_start[cta + 1]) return false;
    pos = p.order[i];
    return true;
  }
  for (; k * G < p.n_items; ++k) {
    pos = item_position(k, cta, G);
    if (pos < p.n_items) return true;
  }
  return false;
}

// next_item for a whole (converged) warp, with warp-uniform results.
__device__ __forceinline__ bool next_item(const TcParams& p, int cta, int G, int& k, int& pos) {
  const bool has = next_item_lane(p, cta, G, k, pos);
  k = warp_uniform(k);
  pos = warp_uniform(pos);
  return warp_uniform(has ? 1 : 0) != 0;
}

__device__ __forceinline__ WorkItem decode_item(const TcParams& p, int pos) {
  const int bh = pos / p.n_qtiles;
  const int r = pos - bh * p.n_qtiles;
  WorkItem w;
  w.qt = p.list_mode ? r : (p.order_len ? static_cast<int>(p.order[r]) : (p.n_qtiles - 1 - r));
  w.b = bh / p.H;
  w.h = bh - w.b * p.H;
  return w;
}

// Rotation phase of the fused rotary embedding: the 16-byte vectors of q, k,
// tq and tk (in that order) are spread over every thread of the grid, and
// each thread has kRopeInFlight of them in flight (all loads issued before the
// first rotation), so that the phase runs at the memory's rate rather than
// its latency. The host bounds B L H d/2 below 2^32 (the vector count).
constexpr int kRopeInFlight = 8;
template <int D>
__device__ __forceinline__ void rope_phase(const TcParams& p) {
  constexpr int VPR = D / 8;  // 16-byte vectors per row of one tensor
  const unsigned per_tensor = static_cast<unsigned>(p.B) * p.L * p.H * VPR;
  const unsigned total = 4u * per_tensor;
  const unsigned stride = gridDim.x * blockDim.x;
  for (unsigned v0 = blockIdx.x * blockDim.x + threadIdx.x; v0 < total; v0 += kRopeInFlight * stride) {
    uint4 u[kRopeInFlight];
    float4 c[kRopeInFlight], sn[kRopeInFlight];
    unsigned which[kRopeInFlight], e[kRopeInFlight];
#pragma unroll
    for (int i = 0; i < kRopeInFlight; ++i) {
      const unsigned v = v0 + i * stride;
      if (v < total) {
        which[i] = v / per_tensor;
        e[i] = v - which[i] * per_tensor;  // vector within the tensor
        const unsigned r = e[i] / VPR, col = (e[i] % VPR) * 8;
        const unsigned t = (r / p.H) % p.L;  // token
        const size_t a = static_cast<size_t>(t) * (D / 2) + col / 2;
        const void* src = which[i] == 0 ? p.rope_src[0]
                          : which[i] == 1 ? p.rope_src[1]
                          : which[i] == 2 ? p.rope_src[2]
                                          : p.rope_src[3];
        c[i] = *reinterpret_cast<const float4*>(p.rope_cos + a);
        sn[i] = *reinterpret_cast<const float4*>(p.rope_sin + a);
        u[i] = reinterpret_cast<const uint4*>(src)[e[i]];
      }
    }
#pragma unroll
    for (int i = 0; i < kRopeInFlight; ++i) {
      if (v0 + i * stride < total) {
        float x[8] = {bf16lo_to_f32(u[i].x), bf16hi_to_f32(u[i].x), bf16lo_to_f32(u[i].y),
                      bf16hi_to_f32(u[i].y), bf16lo_to_f32(u[i].z), bf16hi_to_f32(u[i].z),
                      bf16lo_to_f32(u[i].w), bf16hi_to_f32(u[i].w)};
        rope_rotate_pair(x[0], x[1], c[i].x, sn[i].x);
        rope_rotate_pair(x[2], x[3], c[i].y, sn[i].y);
        rope_rotate_pair(x[4], x[5], c[i].z, sn[i].z);
        rope_rotate_pair(x[6], x[7], c[i].w, sn[i].w);
        void* dst = which[i] == 0 ? p.rope_dst[0]
                    : which[i] == 1 ? p.rope_dst[1]
                    : which[i] == 2 ? p.rope_dst[2]
                                    : p.rope_dst[3];
        reinterpret_cast<uint4*>(dst)[e[i]] =
            make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                       pack_bf16x2(x[6], x[7]));
      }
    }
  }
}

// Grid barrier on a word shared by the launches that map to it: the high 32
// bits tag the launch (epoch), the low 32 bits count its arrivals. The first
// arrival of a launch retags the word. Bounded: false if the count did not
// reach n within limit_ns. One thread per CTA calls it.
__device__ __forceinline__ bool grid_sync(unsigned long long* slot, unsigned int epoch, unsigned int n,
                                          uint64_t limit_ns) {
  __threadfence();
  const unsigned long long tag = static_cast<unsigned long long>(epoch) << 32;
  const unsigned long long hi = ~0xffffffffull;
  unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(slot);
  while (true) {
    const unsigned long long want = ((cur & hi) == tag) ? cur + 1 : (tag | 1ull);
    const unsigned long long prev = atomicCAS(slot, cur, want);
    if (prev == cur) break;
    cur = prev;
  }
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    const unsigned long long v = *reinterpret_cast<volatile unsigned long long*>(slot);
    if ((v & hi) != tag || (v & 0xffffffffull) >= n) break;  // complete (or a later launch's)
    if (globaltimer_ns() - t0 > limit_ns) return false;
    __nanosleep(256);
  }
  __threadfence();
  return true;
}

template <int D, bool PAIR>
__global__ void __launch_bounds__(kTcThreads) attn_jvp_tc_kernel(const __grid_constant__ TcParams p) {
  using C = TcCfg<D, PAIR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sTQ = smem + C::QBYTES;
  uint8_t* sRing = smem + 2 * C::QBYTES;
  float* xch = reinterpret_cast<float*>(smem + C::DATA);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::DATA + C::XCH);
  volatile uint32_t* xflags = reinterpret_cast<volatile uint32_t*>(xch + 2 * C::BM);
  uint64_t* full = bars;            // [NP] ring element landed
  uint64_t* empty = bars + C::NP;   // [NP] ring element consumed
  uint64_t* q_full = bars + 2 * C::NP + 0;
  uint64_t* q_empty = bars + 2 * C::NP + 1;
  uint64_t* s_full = bars + 2 * C::NP + 2;
  uint64_t* ts_full = bars + 2 * C::NP + 3;
  uint64_t* p_full = bars + 2 * C::NP + 4;
  uint64_t* u_full = bars + 2 * C::NP + 5;
  uint64_t* acc_full = bars + 2 * C::NP + 6;
  uint64_t* drain = bars + 2 * C::NP + 7;
  uint64_t* s_free = bars + 2 * C::NP + 8;
  uint64_t* xa = bars + 2 * C::NP + 9;   // [4] row-statistics exchange, first half
  uint64_t* xb = bars + 2 * C::NP + 13;  // [4] second half
  uint64_t* peer_done = bars + 2 * C::NP + 17;  // pair: the peer's producer has published its counts
  uint64_t* stall = bars + 2 * C::NP + 18;      // test-only wait that nothing completes
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* peer_cnt = tmem_slot + 2;  // pair, leader: the peer's ring and Q copy counts

  const int warp = warp_uniform(static_cast<int>(threadIdx.x >> 5));
  const int lane = threadIdx.x & 31;
#ifdef AJVP_TRACE
  const long long trace_c0 = clock64();
  const unsigned long long trace_t0 = globaltimer_ns();
#endif
  // Work is distributed over units: single CTAs, or CTA pairs (clusters of 2).
  const int G = PAIR ? gridDim.x / 2 : gridDim.x;
  const int cta = PAIR ? blockIdx.x / 2 : blockIdx.x;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;  // 0: issues the MMAs
  // The mask, with a group table (if any) read from this launch's parameters.
  MaskSpec mask = p.mask;
  mask.groups = p.groups;
  const bool mma_cta = rank == 0;
  // Barriers the leader waits on and other threads (of either CTA) arrive on.
  auto leader_addr = [&](uint64_t* bar) -> uint32_t {
    return PAIR ? mapa_shared(smem_u32(bar), 0) : smem_u32(bar);
  };
  auto arrive_leader = [&](uint64_t* bar) {
    if (PAIR && rank != 0)
      mbar_arrive_remote(leader_addr(bar));
    else
      mbar_arrive(bar);
  };
  // One arrival per warp (lane 0), branch-free.
  auto arrive_leader_warp = [&](uint64_t* bar) {
    if (PAIR && rank != 0)
      mbar_arrive_remote_if(leader_addr(bar), lane == 0);
    else
      mbar_arrive_if(bar, lane == 0);
  };
  auto bwait = [&](uint64_t* bar, uint32_t parity) -> bool {
    return mbar_wait(bar, parity, abort_flag, p.status, p.wait_ns);
  };
  auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
    return warp_wait(bar, parity, abort_flag, p.status, p.wait_ns);
  };

  if (p.rope) {
    // The rotated q, k, tq, tk first (every CTA a share), then all CTAs meet;
    // the attention below reads them through TMA (the async proxy). A grid
    // barrier that runs out reports a timeout; the kernel then still runs to
    // its end, and its outputs are invalid.
    rope_phase<D>(p);
    fence_proxy_async_global();
    __syncthreads();
    if (threadIdx.x == 0 && !grid_sync(p.grid_slot, p.grid_epoch, gridDim.x, p.wait_ns))
      atomicOr(p.status, kStatusTimeout);
    __syncthreads();
    fence_proxy_async_global();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NP; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(ts_full, 1);
    mbar_init(p_full, C::ARRIVALS);
    mbar_init(u_full, C::ARRIVALS);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    mbar_init(peer_done, 1);
    mbar_init(stall, 1);
    mbar_init(s_free, C::ARRIVALS);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&xa[i], 64);
      mbar_init(&xb[i], 64);
      xflags[i] = 0;
      xflags[4 + i] = 0;
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, C::TM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::TM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR)
    cluster_sync_all();  // both CTAs' barriers exist before any remote arrive
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(warp_uniform(static_cast<int>(*tmem_slot)));

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    // Ring elements in order of first use: per key tile j, (K_j, tK_j) then
    // (tV_j, V_j). In a pair both CTAs load their halves; the copies complete
    // on the leader's barriers, which only the leader's producer arms (for both).
    // The whole warp runs the loop; one elected lane issues each copy.
    {
      tma_prefetch_desc(&p.map_q);
      tma_prefetch_desc(&p.map_k);
      tma_prefetch_desc(&p.map_v);
      tma_prefetch_desc(&p.map_tq);
      tma_prefetch_desc(&p.map_tk);
      tma_prefetch_desc(&p.map_tv);
      const uint64_t keep = l2_policy_evict_last();
      [[maybe_unused]] const uint64_t once = l2_policy_evict_first();
      const CUtensorMap* maps[2][2] = {{&p.map_k, &p.map_tk}, {&p.map_tv, &p.map_v}};
      const uint32_t arm = PAIR ? 2u : 1u;  // CTAs whose copies complete on one barrier
      // One K-type (e = 0) or V-type (e = 1) tile of key tile kt into dst.
      auto load_tile = [&](uint8_t* dst, const CUtensorMap* map, int e, uint64_t* bar, int h, int kt,
                           int b, bool issue) {
        if (!issue) return;
        if constexpr (PAIR) {
          if (e == 0) {
            // keys [64 rank, 64 rank + 64) of the tile, all D columns
#pragma unroll
            for (int c = 0; c < C::CH; ++c)
              tma_load_4d_pair(dst + c * C::KROWS * 128, map, leader_addr(bar), c * 64, h,
                               kt * C::BN + static_cast<int>(rank) * C::KROWS, b, keep);
          } else {
            // all keys of the tile, columns [64 rank, 64 rank + 64)
            tma_load_4d_pair(dst, map, leader_addr(bar), static_cast<int>(rank) * 64, h, kt * C::BN,
                             b, keep);
          }
        } else {
#pragma unroll
          for (int c = 0; c < C::CH; ++c)
            tma_load_4d_hint(dst + c * C::BN * 128, map, bar, c * 64, h, kt * C::BN, b, keep);
        }
      };
      uint32_t ctr = 0, q_issued = 0, q_ph = 0;
      bool ok = true;
      int k = 0, pos = 0;
      while (ok && next_item(p, cta, G, k, pos)) {
        ++k;
        const WorkItem w = decode_item(p, pos);
        if (q_issued > 0) {
          if (!wwait(q_empty, q_ph)) { ok = false; break; }
          q_ph ^= 1;
        }
        const int q_row = w.qt * C::BMU + static_cast<int>(rank) * C::BM;
        const bool issue_q = elect_one();
        if (issue_q && mma_cta) mbar_arrive_expect_tx(q_full, arm * 2 * C::QBYTES);
#pragma unroll
        for (int c = 0; c < C::CH && issue_q; ++c) {
          if constexpr (PAIR) {
            tma_load_4d_pair(sQ + c * C::BM * 128, &p.map_q, leader_addr(q_full), c * 64, w.h, q_row,
                             w.b, once);
            tma_load_4d_pair(sTQ + c * C::BM * 128, &p.map_tq, leader_addr(q_full), c * 64, w.h,
                             q_row, w.b, once);
          } else {
            tma_load_4d(sQ + c * C::BM * 128, &p.map_q, q_full, c * 64, w.h, q_row, w.b);
            tma_load_4d(sTQ + c * C::BM * 128, &p.map_tq, q_full, c * 64, w.h, q_row, w.b);
          }
        }
        ++q_issued;
        const TileSched sch = warp_uniform(make_tile_sched(mask, w.qt, C::BMU, C::BN));
        const int cnt = sch.count();
        for (int idx = 0; ok && idx < cnt; ++idx) {
          const int kt = sch.tile(idx);
#pragma unroll 1
          for (int e = 0; e < 2; ++e) {
            const uint32_t el = ctr % C::NP;
            const uint32_t ph = (ctr / C::NP) & 1;
            if (!wwait(&empty[el], ph ^ 1)) { ok = false; break; }
            uint8_t* dst = sRing + el * 2 * C::TILE;
            const bool issue = elect_one();
            if (issue && mma_cta) mbar_arrive_expect_tx(&full[el], arm * 2 * C::TILE);
            load_tile(dst, maps[e][0], e, &full[el], w.h, kt, w.b, issue);
            load_tile(dst + C::TILE, maps[e][1], e, &full[el], w.h, kt, w.b, issue);
            ++ctr;
          }
        }
      }
      if constexpr (PAIR) {
        // Both CTAs' copies complete on the leader's barriers, which only the
        // leader arms. Before the CTAs can leave (the cluster barrier at the
        // end), the leader makes every phase that either producer started
        // complete: the peer publishes how many ring elements and Q tiles it
        // issued; where the counts differ (an abort stopped one producer
        // first) the leader takes the missing half off the pending bytes
        // (complete_tx) or arms the peer's extra copies, then waits for the
        // last phase of every slot. On a normal end every phase is complete
        // already and this costs one round trip.
        if (lane == 0) {
          const uint32_t per_el = 2 * C::TILE, per_q = 2 * C::QBYTES;  // one CTA's bytes
          if (rank != 0) {
            st_cluster_u32(mapa_shared(smem_u32(peer_cnt), 0), ctr);
            st_cluster_u32(mapa_shared(smem_u32(peer_cnt + 1), 0), q_issued);
            mbar_arrive_remote_release(mapa_shared(smem_u32(peer_done), 0));
          } else if (mbar_wait_acquire_cluster(peer_done, 0, p.wait_ns + 100000000ull)) {
            const uint32_t c_peer = peer_cnt[0], q_peer = peer_cnt[1];
            for (uint32_t e = min(ctr, c_peer); e < max(ctr, c_peer); ++e) {
              if (e < ctr)
                mbar_complete_tx(&full[e % C::NP], per_el);
              else
                mbar_arrive_expect_tx(&full[e % C::NP], per_el);
            }
            for (uint32_t i = min(q_issued, q_peer); i < max(q_issued, q_peer); ++i) {
              if (i < q_issued)
                mbar_complete_tx(q_full, per_q);
              else
                mbar_arrive_expect_tx(q_full, per_q);
            }
            const uint32_t n = max(ctr, c_peer), nq = max(q_issued, q_peer);
            for (uint32_t s = 0; s < C::NP && s < n; ++s) {
              const uint32_t last = n - 1 - ((n - 1 + C::NP - s) % C::NP);
              mbar_wait_drain(&full[s], (last / C::NP) & 1, 200000000ull);
            }
            if (nq > 0) mbar_wait_drain(q_full, (nq - 1) & 1, 200000000ull);
          }
        }
      } else if (!ok && lane == 0) {
        // Abort: let every copy already issued land before the CTA exits.
        for (uint32_t s = 0; s < C::NP && s < ctr; ++s) {
          const uint32_t last = ctr - 1 - ((ctr - 1 + C::NP - s) % C::NP);
          mbar_wait_drain(&full[s], (last / C::NP) & 1, 200000000ull);
        }
        if (q_issued > 0) mbar_wait_drain(q_full, (q_issued - 1) & 1, 200000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // Per key tile g, with ring elements KK_j = (K_j, tK_j) and VV_j = (tV_j, V_j):
    //   C: S_{g+1} = Q K_{g+1}^T        once the softmax has read S_g (s_free)
    //   A: T (+)= P_g tV_g              after P_g (p_full)
    //   B: A (+)= P_g V_g               (d = 64: A and B as one N = 128 group)
    //   D: T += U_g V_g                 after U_g (u_full)
    //   E: tS'_{g+1} = tQ K_{g+1}^T + Q tK_{g+1}^T
    // Within an item C goes first, waiting for s_free if need be: the softmax
    // releases S_g before P_g is ready, so the wait never delays A and B, and
    // S_{g+1} then runs while the softmax finishes P_g and U_g. (Issuing A and
    // B first whenever s_free was not yet there left the softmax waiting for
    // S_{g+1} behind them.) The first tile of a new item needs the new Q, so
    // its C comes after D. tcgen05.mma from one thread execute in order, so E
    // (over the columns of P_g and U_g) follows every read of them. The
    // tensor-core queue is shallow and the issuing thread waits for room, so
    // each barrier a group depends on is tested in the middle of the group
    // before it (the `rdy_*` flags): the test's latency then overlaps MMAs
    // still in flight.
    // The whole warp runs this loop with identical values in every lane (one
    // elected lane issues each MMA and commit). In a pair only the leader's
    // warp 9 issues; its commits arrive on the barriers of both CTAs.
    auto commit_all = [&](uint64_t* bar) {
      if constexpr (PAIR)
        umma_commit_pair_both(bar);
      else
        umma_commit(bar);
    };
    auto test = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __shfl_sync(0xffffffffu, mbar_test_wait(bar, parity) ? 1 : 0, 0) != 0;
    };
    if (mma_cta) {
      const uint32_t idesc_s = idesc_bf16_f32(C::M_MMA, C::BN, 0);
      const uint32_t idesc_v = idesc_bf16_f32(C::M_MMA, D, 1);
      const uint32_t idesc_v2 = idesc_bf16_f32(C::M_MMA, 2 * D, 1);
      const uint32_t aQ = smem_u32(sQ), aTQ = smem_u32(sTQ), aRing = smem_u32(sRing);
      auto el_addr = [&](uint32_t j) { return aRing + (j % C::NP) * 2 * C::TILE; };
      auto el_ph = [&](uint32_t j) { return (j / C::NP) & 1; };
      auto el_full = [&](uint32_t j) { return &full[j % C::NP]; };
      auto el_empty = [&](uint32_t j) { return &empty[j % C::NP]; };
      uint32_t q_ph = 0, p_ph = 0, u_ph = 0, sf_ph = 0;
      bool ok = true;
      int k = 0, pos = 0;
      if (next_item(p, cta, G, k, pos)) {
        ++k;
        WorkItem w = decode_item(p, pos);
        TileSched sch = warp_uniform(make_tile_sched(mask, w.qt, C::BMU, C::BN));
        int cnt = sch.count(), idx = 0;
        uint32_t g = 0;
        // prologue: scores of the first tile (ring element 0 = KK_0)
        ok = wwait(q_full, q_ph);
        q_ph ^= 1;
        if (ok) ok = wwait(el_full(0), 0);
        if (ok) {
          tc_fence_after();
          const uint32_t aK = el_addr(0), aTK = aK + C::TILE;
          mma_scores<D, C::BM, C::KROWS, PAIR>(tmem + C::TM_S, aQ, aK, idesc_s, false);
          commit_all(s_full);
          mma_scores<D, C::BM, C::KROWS, PAIR>(tmem + C::TM_TS, aTQ, aK, idesc_s, false);
          mma_scores<D, C::BM, C::KROWS, PAIR>(tmem + C::TM_TS, aQ, aTK, idesc_s, true);
          commit_all(ts_full);
          commit_all(el_empty(0));
          if (cnt == 1) commit_all(q_empty);
        }
        bool rdy_s = false;  // s_free(g) and KK_{g+1} seen complete
        while (ok) {
          // the tile after g (same item or the next one)
          bool has_next = true, new_item = false;
          WorkItem w2 = w;
          TileSched sch2 = sch;
          int cnt2 = cnt, idx2 = idx + 1;
          if (idx2 >= cnt) {
            has_next = next_item(p, cta, G, k, pos);
            if (has_next) {
              ++k;
              w2 = decode_item(p, pos);
              sch2 = warp_uniform(make_tile_sched(mask, w2.qt, C::BMU, C::BN));
              cnt2 = sch2.count();
              idx2 = 0;
              new_item = true;
            }
          }
          const uint32_t jv = 2 * g + 1, jk = 2 * g + 2;  // VV_g, KK_{g+1}
          const uint32_t aTV = el_addr(jv), aV = aTV + C::TILE;
          const uint32_t aK1 = el_addr(jk), aTK1 = aK1 + C::TILE;
          bool s_done = !has_next, rdy_p = false, rdy_v = false, rdy_u = false, rdy_k = false;
          AJVP_EV(g, 14);
          // Test-only: the first unit waits at tile stall_tile on a barrier
          // that nothing completes, so the wait runs out after wait_ns.
          if (static_cast<int>(g) == p.stall_tile && cta == 0 && !wwait(stall, 0)) break;
          auto issue_s = [&](auto hook) {
            tc_fence_after();
            AJVP_EV(g, 12);
            mma_scores<D, C::BM, C::KROWS, PAIR, D / 32>(tmem + C::TM_S, aQ, aK1, idesc_s, false, hook);
            commit_all(s_full);
            AJVP_EV(g, 0);
            sf_ph ^= 1;
            s_done = true;
            rdy_k = true;
          };
          // C, first within an item
          if (!s_done && !new_item) {
            if (!rdy_s && (!wwait(s_free, sf_ph) || !wwait(el_full(jk), el_ph(jk)))) break;
            issue_s([&] {
              rdy_v = test(el_full(jv), el_ph(jv));
              rdy_p = test(p_full, p_ph);
            });
          }
          // A, B
          if (!rdy_v && !wwait(el_full(jv), el_ph(jv))) break;
          AJVP_EV(g, 15);
          if (!rdy_p && !wwait(p_full, p_ph)) break;
          p_ph ^= 1;
          AJVP_EV(g, 1);
          tc_fence_after();
          if constexpr (PAIR) {
            mma_values_split<C::BN, PAIR>(tmem + C::TM_T, tmem + C::TM_P, aTV, idesc_v, idx > 0);
            mma_values_split<C::BN, PAIR, 3>(tmem + C::TM_A, tmem + C::TM_P, aV, idesc_v, idx > 0, [&] {
              rdy_u = test(u_full, u_ph);
            });
          } else {
            // [T | A] (+)= P [tV | V]: the two 64-column tiles as one N = 128 operand
            mma_values_split<C::BN, PAIR, 3>(tmem + C::TM_T, tmem + C::TM_P, aTV, idesc_v2, idx > 0, [&] {
              rdy_u = test(u_full, u_ph);
            });
          }
          AJVP_EV(g, 2);
          // D
          if (!rdy_u && !wwait(u_full, u_ph)) break;
          u_ph ^= 1;
          AJVP_EV(g, 3);
          tc_fence_after();
          mma_values_split<C::BN, PAIR, 3>(tmem + C::TM_T, tmem + C::TM_U, aV, idesc_v, true, [&] {
            if (has_next && !rdy_k) rdy_k = test(el_full(jk), el_ph(jk));
          });
          commit_all(el_empty(jv));
          if (idx == cnt - 1) commit_all(acc_full);
          if (!has_next) break;
          // C for a new item's first tile, which needs the new Q
          if (!s_done) {
            if (new_item) {
              if (!wwait(q_full, q_ph)) break;
              q_ph ^= 1;
            }
            if (!wwait(s_free, sf_ph)) break;
            if (!wwait(el_full(jk), el_ph(jk))) break;
            issue_s(NoHook{});
          }
          // E, over the columns of P_g and U_g (read by the MMAs above)
          if (!rdy_k && !wwait(el_full(jk), el_ph(jk))) break;
          tc_fence_after();
          const uint32_t jn = jk + 2;  // KK_{g+2}
          rdy_s = false;
          mma_scores<D, C::BM, C::KROWS, PAIR>(tmem + C::TM_TS, aTQ, aK1, idesc_s, false);
          mma_scores<D, C::BM, C::KROWS, PAIR, D / 32>(tmem + C::TM_TS, aQ, aTK1, idesc_s, true, [&] {
            rdy_s = test(s_free, sf_ph) && test(el_full(jn), el_ph(jn));
          });
          commit_all(ts_full);
          AJVP_EV(g, 4);
          commit_all(el_empty(jk));
          if (idx2 == cnt2 - 1) commit_all(q_empty);
          w = w2;
          sch = sch2;
          cnt = cnt2;
          idx = idx2;
          ++g;
        }
      }
      // Every MMA issued so far completes before TMEM is released.
      if constexpr (PAIR)
        umma_commit_pair(drain);
      else
        umma_commit(drain);
      if (lane == 0) mbar_wait_drain(drain, 0, 1000000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // Warpgroup wg (warps 4wg..4wg+3) owns key columns [64 wg, 64 wg + 64) of
    // every score tile and output columns [D/2 wg, D/2 wg + D/2); thread
    // (sub, lane) owns query row 32 sub + lane. The two warpgroups exchange
    // their row maxima through shared memory each tile.
    const int wg = warp >> 2, sub = warp & 3;
    const int row = sub * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::TM_S + 64 * wg;
    const uint32_t tTS = tmem + lane_off + C::TM_TS + 64 * wg;
    const uint32_t tA = tmem + lane_off + C::TM_A + C::DH * wg;
    const uint32_t tT = tmem + lane_off + C::TM_T + C::DH * wg;
    float* my_x = xch + wg * C::BM + row;
    const float* other_x = xch + (1 - wg) * C::BM + row;
    uint32_t xa_ph = 0, xb_ph = 0, xseq = 0;
    volatile uint32_t* my_flag = xflags + 4 * wg + sub;
    volatile uint32_t* other_flag = xflags + 4 * (1 - wg) + sub;
    // Per-tile swap of the row maxima: one flag round trip. A single buffer is
    // enough: a warpgroup writes its next tile's value only after that tile's
    // S is ready, and that S is issued only once every softmax warp has
    // arrived on s_free, which each does after reading this value. Bounded spin.
    // The swap is split: publish this warpgroup's maxima, compute P with the
    // running max meanwhile, then read the other's (normally long there).
    // Every lane takes part (same words, one request per access), so that
    // the warp does not diverge.
    auto publish_max = [&](float mine) {
      *my_x = mine;
      __syncwarp();  // every lane's value before any lane's flag
      ++xseq;
      __threadfence_block();
      *my_flag = xseq;
    };
    auto read_max = [&](float& theirs) -> bool {
      uint32_t polls = 0;
      uint64_t t0 = 0;
      while (__any_sync(0xffffffffu, static_cast<int>(*other_flag - xseq) < 0)) {
        if ((++polls & 63u) == 0) {
          if (__any_sync(0xffffffffu, *abort_flag != 0)) return false;
          const uint64_t now = globaltimer_ns();
          if (t0 == 0) t0 = now;
          if (__any_sync(0xffffffffu, now - t0 > p.wait_ns)) {
            *abort_flag = 1;
            if (lane == 0) atomicOr(p.status, kStatusTimeout);
            return false;
          }
        }
      }
      __threadfence_block();
      theirs = *other_x;
      return true;
    };
    // Swap one float per row with the other warpgroup (warps sub and sub + 4
    // share rows): write, both arrive, read, both arrive. Bounded waits.
    auto exchange = [&](float mine, float& theirs) -> bool {
      *my_x = mine;
      mbar_arrive(&xa[sub]);
      if (!warp_wait(&xa[sub], xa_ph, abort_flag, p.status, p.wait_ns)) return false;
      xa_ph ^= 1;
      theirs = *other_x;
      mbar_arrive(&xb[sub]);
      if (!warp_wait(&xb[sub], xb_ph, abort_flag, p.status, p.wait_ns)) return false;
      xb_ph ^= 1;
      return true;
    };
    const float scale_log2 = p.scale_log2;
    const float scale = p.scale;
    uint32_t s_ph = 0, ts_ph = 0, acc_ph = 0, g = 0;
    bool ok = true;
    int k = 0, pos = 0;
    while (ok && next_item(p, cta, G, k, pos)) {
      ++k;
      const WorkItem w = decode_item(p, pos);
      const int t = w.qt * C::BMU + static_cast<int>(rank) * C::BM + row;  // this thread's query row
      const RowRange rr = row_range(mask, t);
      const TileSched sch = warp_uniform(make_tile_sched(mask, w.qt, C::BMU, C::BN));
      const int cnt = sch.count();
      float m_use = -INFINITY, l = 0.f, dsum = 0.f;
      for (int idx = 0; idx < cnt; ++idx, ++g) {
        const int kt = sch.tile(idx);
        const bool full_tile = sch.full(kt);
        const int k0 = kt * C::BN + C::HALF * wg;
        if (!wwait(s_full, s_ph)) { ok = false; break; }
        s_ph ^= 1;
        if (warp == 0 && lane == 0) AJVP_EV(g, 5);
        tc_fence_after();
        uint32_t sr[C::HALF];
        tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_wait_ld();
        if (warp == 0 && lane == 0) AJVP_EVX(g, 10, __uint_as_float(sr[63]));
        if (!full_tile) {
          // admissible local columns of this row in this half tile, [s1, e1) U
          // [s2, e2), as 32-bit column masks
          const int s1 = min(max(rr.a0 - k0, 0), C::HALF);
          const int e1 = min(max(rr.a1 - k0, 0), C::HALF);
          const int s2 = min(max(rr.b0 - k0, 0), C::HALF);
          const int e2 = min(max(rr.b1 - k0, 0), C::HALF);
#pragma unroll
          for (int q = 0; q < C::HALF / 32; ++q) {
            const uint32_t m = (low_bits(e1 - 32 * q) & ~low_bits(s1 - 32 * q)) |
                               (low_bits(e2 - 32 * q) & ~low_bits(s2 - 32 * q));
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (!((m >> j) & 1u)) sr[32 * q + j] = __float_as_uint(-INFINITY);
          }
        }
        // three-input max: two new values per instruction, four chains
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int j = 0; j < C::HALF; j += 8) {
          mx0 = fmax3(mx0, __uint_as_float(sr[j]), __uint_as_float(sr[j + 1]));
          mx1 = fmax3(mx1, __uint_as_float(sr[j + 2]), __uint_as_float(sr[j + 3]));
          mx2 = fmax3(mx2, __uint_as_float(sr[j + 4]), __uint_as_float(sr[j + 5]));
          mx3 = fmax3(mx3, __uint_as_float(sr[j + 6]), __uint_as_float(sr[j + 7]));
        }
        const float my_max = fmaxf(fmax3(mx0, mx1, mx2), mx3);
        tc_fence_before();
        publish_max(my_max);
        // P of this half tile at the running max mb (bf16, packed) and its row sum.
        // The scalings and the row sums run on pairs of floats (FFMA2, FADD2).
        uint32_t pk[C::HALF / 2];
        float2 ls01 = make_float2(0.f, 0.f), ls23 = make_float2(0.f, 0.f);
        auto compute_p = [&](float mb) {
          ls01 = ls23 = make_float2(0.f, 0.f);
          const float2 sc2 = make_float2(scale_log2, scale_log2), nm2 = make_float2(-mb, -mb);
#pragma unroll
          for (int j = 0; j < C::HALF / 2; j += 2) {
            const float2 x01 = __ffma2_rn(
                make_float2(__uint_as_float(sr[2 * j]), __uint_as_float(sr[2 * j + 1])), sc2, nm2);
            const float2 x23 = __ffma2_rn(
                make_float2(__uint_as_float(sr[2 * j + 2]), __uint_as_float(sr[2 * j + 3])), sc2, nm2);
            const float2 p01 = make_float2(ex2_approx(x01.x), ex2_approx(x01.y));
            const float2 p23 = make_float2(ex2_approx(x23.x), ex2_approx(x23.y));
            ls01 = __fadd2_rn(ls01, p01);
            ls23 = __fadd2_rn(ls23, p23);
            pk[j] = pack_bf16x2(p01.x, p01.y);
            pk[j + 1] = pack_bf16x2(p23.x, p23.y);
          }
        };
        // Speculate that the running max stays (it does unless a row's max grows
        // by more than kRescaleTau): P first, the other half's maxima after.
        const bool spec = __all_sync(0xffffffffu, m_use != -INFINITY);
        if (spec) compute_p(m_use);
        if (warp == 0 && lane == 0) AJVP_EVX(g, 11, ls23.y);
        // row maximum over both halves of the tile
        float their_max;
        if (!read_max(their_max)) { ok = false; break; }
        // S_g is in registers and both warpgroups have read this tile's maxima:
        // the MMA warp may write S_{g+1} over S_g.
        __syncwarp();
        arrive_leader_warp(s_free);
        tc_fence_after();
        const float row_max = fmaxf(my_max, their_max);
        if (warp == 0 && lane == 0) AJVP_EV(g, 6);
        const float mt = row_max * scale_log2;  // log2 units; -inf if fully masked
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
        // (re)compute P when it was not speculated or the running max moved
        if (!spec || __any_sync(0xffffffffu, resc)) compute_p((m_use == -INFINITY) ? 0.f : m_use);
        // A and T to the new running max (S is no longer needed here)
        if (__any_sync(0xffffffffu, resc)) {
          // Every value MMA of earlier tiles has completed once this tile's
          // tS' has (it is issued after them and they run in issue order).
          if (!wwait(ts_full, ts_ph)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < C::DH / 32; ++c) {
            uint32_t a[32];
            tmem_ld32(tA + 32 * c, a);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) a[j] = __float_as_uint(__uint_as_float(a[j]) * alpha);
            tmem_st32(tA + 32 * c, a);
          }
#pragma unroll 1
          for (int c = 0; c < C::DH / 32; ++c) {
            uint32_t a[32];
            tmem_ld32(tT + 32 * c, a);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) a[j] = __float_as_uint(__uint_as_float(a[j]) * alpha);
            tmem_st32(tT + 32 * c, a);
          }
        }
        l += (ls01.x + ls01.y) + (ls23.x + ls23.y);
        if (warp == 0 && lane == 0) AJVP_EV(g, 7);

        if (!wwait(ts_full, ts_ph)) { ok = false; break; }
        ts_ph ^= 1;
        if (warp == 0 && lane == 0) AJVP_EV(g, 8);
        tc_fence_after();
        // tS' in two halves of 32 keys: P goes over the first half once it
        // is read, U over the second.
        uint32_t v[32];
        tmem_ld32(tTS, v);
        tmem_wait_ld();
        if (warp == 0 && lane == 0) AJVP_EVX(g, 13, __uint_as_float(v[31]));
        tmem_st32(tTS, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        arrive_leader_warp(p_full);
        uint32_t uk[C::HALF / 2];
        float2 d01 = make_float2(0.f, 0.f), d23 = make_float2(0.f, 0.f);
        const float2 sc2 = make_float2(scale, scale);
        // u = p s tS' for keys [32 h, 32 h + 32) of this warpgroup's half
        // tile, on pairs of floats (FMUL2, FADD2)
        auto u_half = [&](int h) {
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const uint32_t pa = pk[16 * h + j], pb = pk[16 * h + j + 1];
            const float2 u01 = __fmul2_rn(
                __fmul2_rn(make_float2(bf16lo_to_f32(pa), bf16hi_to_f32(pa)), sc2),
                make_float2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1])));
            const float2 u23 = __fmul2_rn(
                __fmul2_rn(make_float2(bf16lo_to_f32(pb), bf16hi_to_f32(pb)), sc2),
                make_float2(__uint_as_float(v[2 * j + 2]), __uint_as_float(v[2 * j + 3])));
            d01 = __fadd2_rn(d01, u01);
            d23 = __fadd2_rn(d23, u23);
            uk[16 * h + j] = pack_bf16x2(u01.x, u01.y);
            uk[16 * h + j + 1] = pack_bf16x2(u23.x, u23.y);
          }
        };
        u_half(0);
        tmem_ld32(tTS + 32, v);
        tmem_wait_ld();
        u_half(1);
        dsum += (d01.x + d01.y) + (d23.x + d23.y);
        tmem_st32(tTS + 32, uk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        arrive_leader_warp(u_full);
        if (warp == 0 && lane == 0) AJVP_EV(g, 9);
      }
      if (!ok) break;
      // ---------------- epilogue: O = A/l, tO = T/l - (D/l) O, LSE
      if (!wwait(acc_full, acc_ph)) { ok = false; break; }
      acc_ph ^= 1;
      tc_fence_after();
      float l_other, d_other;
      if (!exchange(l, l_other) || !exchange(dsum, d_other)) { ok = false; break; }
      const float l_tot = l + l_other;
      const float d_tot = dsum + d_other;
      const bool valid = t < p.L;
      const float inv_l = (l_tot > 0.f) ? 1.f / l_tot : 0.f;
      const float mu = d_tot * inv_l;
      const size_t row_off =
          ((static_cast<size_t>(w.b) * p.L + (valid ? t : 0)) * p.H + w.h) * D + C::DH * wg;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + row_off;
      __nv_bfloat16* torow = reinterpret_cast<__nv_bfloat16*>(p.to) + row_off;
#pragma unroll 1
      for (int c = 0; c < C::DH / 32; ++c) {
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
      if (valid && wg == 0) {
        const float mb = (m_use == -INFINITY) ? 0.f : m_use;
        p.lse[(static_cast<size_t>(w.b) * p.H + w.h) * p.L + t] = (mb + __log2f(l_tot)) * kLn2;
      }
    }
    tc_fence_before();
  }

#ifdef AJVP_TRACE
  // per CTA: SM cycles and nanoseconds from start to here (after every role)
  if (p.trace && threadIdx.x == 0) {
    p.trace[kTraceTiles * kTraceEvents + 2 * blockIdx.x] = clock64() - trace_c0;
    p.trace[kTraceTiles * kTraceEvents + 2 * blockIdx.x + 1] =
        static_cast<long long>(globaltimer_ns() - trace_t0);
  }
#endif
  if constexpr (PAIR) {
    // Neither CTA leaves (or frees its TMEM) while the leader's MMAs may still
    // read the other's shared or tensor memory.
    cluster_sync_all();
    tc_fence_after();
    if (warp == 9) tmem_dealloc_pair(tmem, C::TM_COLS);
  } else {
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, C::TM_COLS);
  }
}

size_t tc_smem_bytes(int d) {
  return d == 128 ? TcCfg<128, true>::BYTES : TcCfg<64, false>::BYTES;
}

cudaError_t tc_prepare(int d) {
  if (d == 128)
    return cudaFuncSetAttribute(attn_jvp_tc_kernel<128, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                TcCfg<128, true>::BYTES);
  return cudaFuncSetAttribute(attn_jvp_tc_kernel<64, false>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfg<64, false>::BYTES);
}

namespace {
void pair_config(cudaLaunchConfig_t* cfg, cudaLaunchAttribute* attr, int grid, cudaStream_t stream) {
  *cfg = cudaLaunchConfig_t{};
  cfg->gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg->blockDim = dim3(kTcThreads, 1, 1);
  cfg->dynamicSmemBytes = TcCfg<128, true>::BYTES;
  cfg->stream = stream;
  attr->id = cudaLaunchAttributeClusterDimension;
  attr->val.clusterDim.x = 2;
  attr->val.clusterDim.y = 1;
  attr->val.clusterDim.z = 1;
  cfg->attrs = attr;
  cfg->numAttrs = 1;
}
}  // namespace

int tc_pair_max_clusters(int sm_count) {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr;
  pair_config(&cfg, &attr, 2 * (sm_count / 2), nullptr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, attn_jvp_tc_kernel<128, true>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

cudaError_t tc_launch(int d, const TcParams& p, int grid, cudaStream_t stream) {
  // A launch with the rotation phase meets at a grid barrier: it asks for a
  // cooperative launch, which fails rather than runs if its CTAs cannot all
  // be resident at once.
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  if (d == 128) {
    pair_config(&cfg, &attr[0], grid, stream);
  } else {
    cfg = cudaLaunchConfig_t{};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = TcCfg<64, false>::BYTES;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 0;
  }
  if (p.rope) {
    attr[cfg.numAttrs].id = cudaLaunchAttributeCooperative;
    attr[cfg.numAttrs].val.cooperative = 1;
    cfg.numAttrs += 1;
  }
  if (d == 128) return cudaLaunchKernelEx(&cfg, attn_jvp_tc_kernel<128, true>, p);
  return cudaLaunchKernelEx(&cfg, attn_jvp_tc_kernel<64, false>, p);
}

}  // namespace ajvp
