// tiles.cuh - tile-level tcgen05 MMA helpers shared by the forward and
// backward tensor-core kernels (bf16 operands, fp32 TMEM accumulators).
#pragma once

#include <cstdint>

#include "mask_schedule.cuh"
#include "ptx.cuh"

namespace ajvp {

// Value of lane 0 in every lane; the whole (converged) warp calls it. The
// compiler then knows the value is the same across the warp, so a branch on
// it around warp-collective tcgen05 instructions (elect.sync, .sync.aligned)
// needs no reconvergence handling. Without it, every MMA issued after such a
// branch compiled to several times as many instructions (measured by code
// size: ~450 against ~140 bytes per tcgen05.mma).
__device__ __forceinline__ int warp_uniform(int v) { return __shfl_sync(0xffffffffu, v, 0); }

__device__ __forceinline__ TileSched warp_uniform(TileSched s) {
  s.t1_begin = warp_uniform(s.t1_begin);
  s.t1_end = warp_uniform(s.t1_end);
  s.t2_begin = warp_uniform(s.t2_begin);
  s.t2_end = warp_uniform(s.t2_end);
  s.i_a0 = warp_uniform(s.i_a0);
  s.i_a1 = warp_uniform(s.i_a1);
  s.i_b0 = warp_uniform(s.i_b0);
  s.i_b1 = warp_uniform(s.i_b1);
  return s;
}

// Operand layouts in shared memory (TMA, 128-byte swizzle): a tile of R rows
// x D columns is D/64 chunks of R rows x 128 bytes. As a K-major operand
// (Q, tQ, K, tK: contraction over d) k-step kk starts at chunk kk/4, byte
// 32 (kk%4); the stride between 8-row groups (SBO) is 1024. As an MN-major
// operand (V, tV: contraction over keys) k-step ks starts at key 16 ks; the
// 64-column blocks of d sit R*128 bytes apart (LBO), 8-key groups 1024.

// bf16 P (or U) in TMEM: warpgroup h packs keys [64 h, 64 h + 64) into the
// first 32 of its own 64 score columns, so key k sits at column
// 64 (k / 64) + (k % 64) / 2. K-step ks of the value MMAs covers keys
// [16 ks, 16 ks + 16).
__device__ __forceinline__ uint32_t tmem_a_operand(uint32_t base, int ks) {
  return base + 64 * (ks >> 2) + (ks & 3) * 8;
}

// Score MMA: D[tmem] (+)= A B^T over the head dimension, A a [rows_a x D]
// and B a [rows_b x D] K-major tile. Offsets are added to the descriptors'
// start-address field (16-byte units; tiles lie well inside its 256 KB range).
struct NoHook {
  __device__ __forceinline__ void operator()() const {}
};

// The MMA helpers call `hook` right after issuing instruction AT (if AT >= 0):
// the MMA warp tests its next barriers there, so the test's latency overlaps
// the instructions still to be issued instead of leaving the pipe idle.
template <int D, int ROWS_A, int ROWS_B, bool PAIR, int AT = -1, typename Hook = NoHook>
__device__ __forceinline__ void mma_scores(uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem,
                                           uint32_t idesc, bool accumulate, Hook hook = Hook{}) {
  const uint64_t da = smem_desc_sw128(a_smem, 16, 1024);
  const uint64_t db = smem_desc_sw128(b_smem, 16, 1024);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t oa = ((kk >> 2) * ROWS_A * 128 + (kk & 3) * 32) >> 4;
    const uint32_t ob = ((kk >> 2) * ROWS_B * 128 + (kk & 3) * 32) >> 4;
    if constexpr (PAIR)
      umma_ss_pair(d_tmem, da + oa, db + ob, idesc, (accumulate || kk > 0) ? 1u : 0u);
    else
      umma_ss(d_tmem, da + oa, db + ob, idesc, (accumulate || kk > 0) ? 1u : 0u);
    if (kk == AT) hook();
  }
}

// Value MMA: D[tmem] (+)= P[tmem] V, P a bf16 [128 x BN] tile in TMEM (in the
// two-warpgroup layout of tmem_a_operand) and V a [BN keys x D] tile read
// MN-major (for a pair, each CTA holds one 64-column chunk of it).
template <int BN, bool PAIR, int AT = -1, typename Hook = NoHook>
__device__ __forceinline__ void mma_values_split(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_smem,
                                           uint32_t idesc, bool accumulate, Hook hook = Hook{}) {
  const uint64_t db = smem_desc_sw128(b_smem, BN * 128, 1024);
#pragma unroll
  for (int ks = 0; ks < BN / 16; ++ks) {
    const uint32_t acc = (accumulate || ks > 0) ? 1u : 0u;
    if constexpr (PAIR)
      umma_ts_pair(d_tmem, tmem_a_operand(a_tmem, ks), db + ((ks * 16 * 128) >> 4), idesc, acc);
    else
      umma_ts(d_tmem, tmem_a_operand(a_tmem, ks), db + ((ks * 16 * 128) >> 4), idesc, acc);
    if (ks == AT) hook();
  }
}

}  // namespace ajvp
