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
//   groups (the general form of the same page's App. B: query groups with
//     admissible key ranges): a table of row groups in order; group g holds
//     rows [row_end of g-1, row_end of g) and admits keys [a0, a1) U [b0, b1).
// Every row's admissible set is [a0, a1) U [b0, b1) (either part possibly
// empty; a1 <= b0). A block of rows is scheduled over the union
// [min a0, max a1) U [min b0, max b1) (a gap inside either part is visited
// and masked); a key tile is "full" inside the intersection
// [max a0, min a1) U (the b-range, if every row has the same one).
#pragma once

#include <cstdint>

#if defined(__CUDACC__)
#define AJVP_HD __host__ __device__ __forceinline__
#else
#define AJVP_HD inline
#endif

namespace ajvp {

enum : int { kModeTeacherForcing = 0, kModeBlockCausal = 1, kModeGroups = 2 };

// One row group of a general mask: rows up to row_end (exclusive) since the
// previous group, keys [a0, a1) U [b0, b1).
struct GroupRange {
  int row_end, a0, a1, b0, b1;
};
constexpr int kMaxGroups = 512;

struct MaskSpec {
  int mode;
  int c;  // chunk tokens
  int n;  // chunks
  int L;  // sequence length
  int n_groups;               // kModeGroups: table length
  const GroupRange* groups;   // kModeGroups: the table (host or device address)
};

// Admissible keys of one query row: [a0, a1) U [b0, b1).
struct RowRange {
  int a0, a1, b0, b1;
};

// Index of the group holding row t: the first with row_end > t.
AJVP_HD int group_of(const MaskSpec& m, int t) {
  int lo = 0, hi = m.n_groups - 1;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (m.groups[mid].row_end > t)
      hi = mid;
    else
      lo = mid + 1;
  }
  return lo;
}

AJVP_HD RowRange row_range(const MaskSpec& m, int t) {
  RowRange r;
  r.a0 = 0;
  if (m.mode == kModeGroups) {
    const GroupRange g = m.groups[group_of(m, t)];
    r.a0 = g.a0;
    r.a1 = g.a1;
    r.b0 = g.b0;
    r.b1 = g.b1;
    return r;
  }
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

AJVP_HD bool row_allows(const RowRange& r, int k) {
  return (k >= r.a0 && k < r.a1) || (k >= r.b0 && k < r.b1);
}

// First row after t whose admissible set may differ from row t's.
AJVP_HD int next_group_start(const MaskSpec& m, int t) {
  if (m.mode == kModeGroups) return m.groups[group_of(m, t)].row_end;
  if (m.mode == kModeTeacherForcing) {
    const int nc = m.n * m.c;
    if (t >= nc) return nc + ((t - nc) / m.c + 1) * m.c;
  }
  return (t / m.c + 1) * m.c;
}

// Key-tile schedule of one query tile: the tiles [t1_begin, t1_end) and then
// [t2_begin, t2_end); a tile is "full" when every pair in it is admissible
// for every valid row of the query tile.
struct TileSched {
  int t1_begin, t1_end;
  int t2_begin, t2_end;
  int i_a0, i_a1;  // intersection, first part [i_a0, i_a1) (may be empty)
  int i_b0, i_b1;  // intersection, second part [i_b0, i_b1) (may be empty)
  int bn;

  AJVP_HD int count() const { return (t1_end - t1_begin) + (t2_end - t2_begin); }
  AJVP_HD int tile(int idx) const {
    const int n1 = t1_end - t1_begin;
    return idx < n1 ? t1_begin + idx : t2_begin + (idx - n1);
  }
  AJVP_HD bool full(int kt) const {
    const int k0 = kt * bn, k1 = k0 + bn;
    return (k0 >= i_a0 && k1 <= i_a1) || (k0 >= i_b0 && k1 <= i_b1);
  }
};

AJVP_HD int cdiv(int a, int b) { return (a + b - 1) / b; }

// Schedule for query rows [q_tile * bm, min(L, (q_tile+1) * bm)) and key tiles of bn.
AJVP_HD TileSched make_tile_sched(const MaskSpec& m, int q_tile, int bm, int bn) {
  const int r0 = q_tile * bm;
  const int r1 = (r0 + bm < m.L) ? r0 + bm : m.L;
  int u_a0 = 0x7fffffff, u_a1 = 0, u_b0 = 0x7fffffff, u_b1 = 0;  // union (non-empty parts)
  int x_a0 = 0, x_a1 = 0x7fffffff;                                 // intersection, first part
  int x_b0 = 0, x_b1 = 0;
  bool all_b = true, b_set = false, b_same = true;
  for (int t = r0; t < r1;) {
    const RowRange r = row_range(m, t);
    if (r.a1 > r.a0) {
      if (r.a0 < u_a0) u_a0 = r.a0;
      if (r.a1 > u_a1) u_a1 = r.a1;
    }
    if (r.a0 > x_a0) x_a0 = r.a0;
    if (r.a1 < x_a1) x_a1 = r.a1;
    if (r.b1 > r.b0) {
      if (r.b0 < u_b0) u_b0 = r.b0;
      if (r.b1 > u_b1) u_b1 = r.b1;
      if (!b_set) {
        x_b0 = r.b0;
        x_b1 = r.b1;
        b_set = true;
      } else if (r.b0 != x_b0 || r.b1 != x_b1) {
        b_same = false;
      }
    } else {
      all_b = false;
    }
    t = next_group_start(m, t);
  }
  TileSched s;
  s.bn = bn;
  s.i_a0 = x_a0;
  s.i_a1 = (x_a1 == 0x7fffffff || x_a1 < x_a0) ? x_a0 : x_a1;
  if (all_b && b_set && b_same) {
    s.i_b0 = x_b0;
    s.i_b1 = x_b1;
  } else {
    s.i_b0 = s.i_b1 = 0;
  }
  const bool any_a = u_a1 > 0 && u_a0 != 0x7fffffff;
  const bool any_b = b_set;
  s.t1_begin = s.t1_end = s.t2_begin = s.t2_end = 0;
  if (!any_a && !any_b) return s;
  if (!any_b) {
    s.t1_begin = u_a0 / bn;
    s.t1_end = cdiv(u_a1, bn);
    return s;
  }
  if (!any_a) {
    s.t1_begin = u_b0 / bn;
    s.t1_end = cdiv(u_b1, bn);
    return s;
  }
  const int lo = u_a0 < u_b0 ? u_a0 : u_b0;
  if (u_b0 <= u_a1) {  // the two parts touch: one contiguous range
    const int hi = u_b1 > u_a1 ? u_b1 : u_a1;
    s.t1_begin = lo / bn;
    s.t1_end = cdiv(hi, bn);
    return s;
  }
  s.t1_begin = u_a0 / bn;
  s.t1_end = cdiv(u_a1, bn);
  int b_begin = u_b0 / bn;
  if (b_begin < s.t1_end) b_begin = s.t1_end;  // a tile shared by both parts is listed once
  s.t2_begin = b_begin;
  s.t2_end = cdiv(u_b1, bn);
  if (s.t2_end < s.t2_begin) s.t2_end = s.t2_begin;
  return s;
}

// Query tiles [lo, hi] (tiles of bq rows, n_qt of them) outside which no row
// can see key tile kt (tiles of bk keys): exact for the closed-form masks
// (teacher forcing: clean keys are seen from their chunk's clean rows on,
// noisy keys only by their own chunk's noisy rows; block causal: from the
// key's chunk on), every tile for a group table or a tile past L.
AJVP_HD void key_tile_query_bounds(const MaskSpec& m, int kt, int bk, int n_qt, int bq, int& lo,
                                   int& hi) {
  lo = 0;
  hi = n_qt - 1;
  const int k0 = kt * bk;
  if (m.mode == kModeGroups || k0 >= m.L) return;
  const int c = m.c;
  const int nc = m.n * c;
  if (m.mode == kModeTeacherForcing && k0 >= nc) {
    const int k1 = (k0 + bk < m.L ? k0 + bk : m.L) - 1;  // last key of the tile
    const int i0 = (k0 - nc) / c, i1 = (k1 - nc) / c;
    lo = (nc + i0 * c) / bq;
    const int h = (nc + i1 * c + c - 1) / bq;
    hi = h < n_qt - 1 ? h : n_qt - 1;
    return;
  }
  lo = ((k0 / c) * c) / bq;
}

}  // namespace ajvp
