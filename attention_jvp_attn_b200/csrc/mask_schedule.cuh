// mask_schedule.cuh - block-sparse schedule of the custom masks (host and device).
//
// Causal-rCM summary page, App. B: masks are query groups with admissible key
// ranges ("query-key rectangles"); one sparse schedule drives both the primal
// and the tangent scores, so fully masked key tiles are never visited.
//
// Masks (same page, section 3 "Continuous-time consistency" for the packed
// teacher-forcing sequence; section 2 "Autoregressive video diffusion" for
// block-causal attention):
//   teacher forcing: L = 2 n c, tokens [0, nc) are clean chunks, [nc, 2nc) noisy.
//     clean query in chunk j:  keys [0, (j+1) c)
//     noisy query in chunk i:  keys [0, i c)  U  [nc + i c, nc + (i+1) c)
//   block causal: L = n c, query in chunk j: keys [0, (j+1) c)
// Every row's admissible set is [0, a1) U [b0, b1) (second part possibly
// empty). All first parts lie in [0, nc), all second parts in [nc, 2nc), so a
// group of rows has union [0, max a1) U [min b0, max b1) and intersection
// [0, min a1) U (common b-range if all rows share one noisy chunk).
#pragma once

#include <cstdint>

#if defined(__CUDACC__)
#define AJVP_HD __host__ __device__ __forceinline__
#else
#define AJVP_HD inline
#endif

namespace ajvp {

enum : int { kModeTeacherForcing = 0, kModeBlockCausal = 1 };

struct MaskSpec {
  int mode;
  int c;  // chunk tokens
  int n;  // chunks
  int L;  // sequence length
};

// Admissible keys of one query row: [0, a1) U [b0, b1).
struct RowRange {
  int a1, b0, b1;
};

AJVP_HD RowRange row_range(const MaskSpec& m, int t) {
  RowRange r;
  if (m.mode == kModeBlockCausal) {
    r.a1 = (t / m.c + 1) * m.c;
    r.b0 = r.b1 = 0;
    return r;
  }
  const int nc = m.n * m.c;
  if (t < nc) {
    r.a1 = (t / m.c + 1) * m.c;
    r.b0 = r.b1 = 0;
  } else {
    const int i = (t - nc) / m.c;
    r.a1 = i * m.c;
    r.b0 = nc + i * m.c;
    r.b1 = r.b0 + m.c;
  }
  return r;
}

AJVP_HD bool row_allows(const RowRange& r, int k) { return k < r.a1 || (k >= r.b0 && k < r.b1); }

// First row after t whose admissible set may differ from row t's.
AJVP_HD int next_group_start(const MaskSpec& m, int t) {
  if (m.mode == kModeTeacherForcing) {
    const int nc = m.n * m.c;
    if (t >= nc) return nc + ((t - nc) / m.c + 1) * m.c;
  }
  return (t / m.c + 1) * m.c;
}

// Key-tile schedule of one query tile: the tiles [0, n1) and then
// [t2_begin, t2_end); a tile is "full" when every pair in it is admissible
// for every valid row of the query tile.
struct TileSched {
  int n1;
  int t2_begin, t2_end;
  int i_a1;        // intersection, first part [0, i_a1)
  int i_b0, i_b1;  // intersection, second part [i_b0, i_b1) (may be empty)
  int bn;

  AJVP_HD int count() const { return n1 + (t2_end - t2_begin); }
  AJVP_HD int tile(int idx) const { return idx < n1 ? idx : t2_begin + (idx - n1); }
  AJVP_HD bool full(int kt) const {
    const int k0 = kt * bn, k1 = k0 + bn;
    return k1 <= i_a1 || (k0 >= i_b0 && k1 <= i_b1);
  }
};

AJVP_HD int cdiv(int a, int b) { return (a + b - 1) / b; }

// Schedule for query rows [q_tile * bm, min(L, (q_tile+1) * bm)) and key tiles of bn.
AJVP_HD TileSched make_tile_sched(const MaskSpec& m, int q_tile, int bm, int bn) {
  const int r0 = q_tile * bm;
  const int r1 = (r0 + bm < m.L) ? r0 + bm : m.L;
  int u_a1 = 0, u_b0 = 0x7fffffff, u_b1 = 0;  // union
  int x_a1 = 0x7fffffff, x_b0 = 0, x_b1 = 0;  // intersection
  bool all_b = true, b_set = false, b_same = true;
  for (int t = r0; t < r1;) {
    const RowRange r = row_range(m, t);
    if (r.a1 > u_a1) u_a1 = r.a1;
    if (r.a1 < x_a1) x_a1 = r.a1;
    if (r.b1 > r.b0) {
      if (r.b0 < u_b0) u_b0 = r.b0;
      if (r.b1 > u_b1) u_b1 = r.b1;
      if (!b_set) {
        x_b0 = r.b0;
        x_b1 = r.b1;
        b_set = true;
      } else if (r.b0 != x_b0) {
        b_same = false;
      }
    } else {
      all_b = false;
    }
    t = next_group_start(m, t);
  }
  const bool any_b = b_set;
  TileSched s;
  s.bn = bn;
  s.i_a1 = (x_a1 == 0x7fffffff) ? 0 : x_a1;
  if (all_b && b_set && b_same) {
    s.i_b0 = x_b0;
    s.i_b1 = x_b1;
  } else {
    s.i_b0 = s.i_b1 = 0;
  }
  if (!any_b) {
    s.n1 = cdiv(u_a1, bn);
    s.t2_begin = s.t2_end = 0;
    return s;
  }
  if (u_b0 <= u_a1) {  // the two parts touch: one contiguous range
    const int hi = u_b1 > u_a1 ? u_b1 : u_a1;
    s.n1 = cdiv(hi, bn);
    s.t2_begin = s.t2_end = 0;
    return s;
  }
  s.n1 = cdiv(u_a1, bn);
  int b_begin = u_b0 / bn;
  if (b_begin < s.n1) b_begin = s.n1;  // a tile shared by both parts is listed once
  s.t2_begin = b_begin;
  s.t2_end = cdiv(u_b1, bn);
  if (s.t2_end < s.t2_begin) s.t2_end = s.t2_begin;
  return s;
}

}  // namespace ajvp
