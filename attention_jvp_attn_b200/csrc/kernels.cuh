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
  // Rotary embedding in the same launch (rope != 0): every CTA first rotates
  // a share of rope_src (q, k, tq, tk) into rope_dst, whose tensor maps the
  // attention then reads; the CTAs meet at a grid barrier in between, on the
  // word grid_slot tagged with grid_epoch.
  int rope;
  const void* rope_src[4];
  void* rope_dst[4];
  const float* rope_cos;  // [L, d/2]
  const float* rope_sin;
  unsigned long long* grid_slot;
  unsigned int grid_epoch;
  unsigned long long wait_ns;  // limit of every bounded wait (default 4 s)
  int stall_tile;              // test only: >= 0 makes unit 0's MMA issuer wait at that tile
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

// ---- bf16 backward on tensor cores (attn_jvp_bwd_tc.cu) ----
struct BwdTcArgs {
  const void *q, *k, *v, *o, *dout;  // [B, L, H, d] bf16
  const float *lse, *dlse;           // [B, H, L]; dlse may be null
  void *dq, *dk, *dv;                // [B, L, H, d] bf16; dq also serves as scratch
  int64_t B, L, H, d;
  MaskSpec mask;  // kModeGroups: mask.groups points to a host table of mask.n_groups groups
  float scale;
};
cudaError_t bwd_tc_prepare();  // sets the kernels' shared-memory limits (once per device)
// True if the tensor-core backward runs this shape (else the CUDA-core kernels do).
bool bwd_tc_supported(int64_t B, int64_t L, int64_t H, int64_t d);
int bwd_tc_launch(const BwdTcArgs& a, cudaStream_t stream);  // ATTN_JVP_* status

// ---- services of the C ABI layer for the other kernel files ----
// The current device's status word (bit 0: a bounded wait ran out), set up
// once per device; returns an ATTN_JVP_* status.
int device_status_word(unsigned int** word);
// 4-D tensor map over a dense [B, L, H, d] bf16 array: boxes of 64 columns x
// `box_rows` rows of one (batch, head), 128-byte swizzle, zero fill out of range.
bool encode_bf16_rows_map(CUtensorMap* map, const void* base, int64_t B, int64_t L, int64_t H,
                          int64_t d, int box_rows);

}  // namespace ajvp
