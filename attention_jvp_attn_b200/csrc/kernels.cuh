// kernels.cuh - launch parameters shared by the C ABI and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "mask_schedule.cuh"

namespace ajvp {

// ---- bf16 tensor-core kernel (tcgen05 / TMEM / TMA) ----
constexpr int kTcBlockM = 128;   // query rows per tile (one TMEM lane per row)
constexpr int kTcBlockN = 128;   // keys per tile
constexpr int kTcThreads = 320;  // warps 0-7 softmax+epilogue, 8 TMA producer, 9 MMA issuer
constexpr int kMaxOrder = 4096;  // order table / work-list capacity
constexpr int kMaxUnits = 160;   // work lists: units (CTAs or CTA pairs) of the persistent grid

struct TcParams {
  CUtensorMap map_q, map_k, map_v, map_tq, map_tk, map_tv;  // [B, L, H, d] bf16, 128B swizzle
  void* o;
  void* to;
  float* lse;
  unsigned int* status;
  int B, H, L;
  int n_qtiles;  // query row blocks per (batch, head): ceil(L / 128), or ceil(L / 256) for pairs
  int n_items;   // B * H * n_qtiles
  MaskSpec mask;
  float scale_log2;  // s * log2(e)
  float scale;       // s
  int order_len;     // n_qtiles if `order` is a per-head order table, else 0 (reverse index order)
  // list_mode: unit u runs the items order[unit_start[u] .. unit_start[u+1]), each an item
  // position b*H*n_qtiles + h*n_qtiles + qt; else unit u takes rounds of a snake over
  // positions, with the query block of position r within a head given by the order table
  int list_mode;
  uint16_t unit_start[kMaxUnits + 1];
#ifdef AJVP_TRACE
  long long* trace;  // per-tile event clocks of one CTA (trace builds only)
#endif
  uint16_t order[kMaxOrder];
  GroupRange groups[kMaxGroups];  // mask.mode == kModeGroups: the row groups (mask.n_groups)
};

#ifdef AJVP_TRACE
constexpr int kTraceTiles = 512;
constexpr int kTraceEvents = 16;
constexpr int kTraceCta = 4;  // a CTA (the leader of a pair) whose first items are mostly full tiles
#endif

size_t tc_smem_bytes(int d);
cudaError_t tc_prepare(int d);  // sets the dynamic shared-memory limit (once per device)
// Clusters of two CTAs (the d = 128 kernel runs on CTA pairs) that fit on the
// device at once; 0 if unknown.
int tc_pair_max_clusters(int sm_count);
// d = 128: `grid` CTAs in clusters of two (an even number); d = 64: single CTAs.
cudaError_t tc_launch(int d, const TcParams& p, int grid, cudaStream_t stream);

// ---- fp32 CUDA-core kernel ----
constexpr int kSimtBlockQ = 32;
constexpr int kSimtBlockK = 32;
constexpr int kSimtThreads = 256;

struct SimtParams {
  const float *q, *k, *v, *tq, *tk, *tv;
  float *o, *to, *lse;
  int B, H, L;
  MaskSpec mask;
  float scale_log2, scale;
  GroupRange groups[kMaxGroups];  // mask.mode == kModeGroups: the row groups (mask.n_groups)
};

size_t simt_smem_bytes(int d);
cudaError_t simt_prepare(int d);
cudaError_t simt_launch(int d, const SimtParams& p, cudaStream_t stream);

}  // namespace ajvp
