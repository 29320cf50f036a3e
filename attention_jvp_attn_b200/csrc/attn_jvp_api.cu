// attn_jvp_api.cu - the C ABI declared in include/attn_jvp.h: argument
// validation, TMA descriptor encoding, work ordering, launches, status words.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstddef>
#include <cstring>
#include <functional>
#include <mutex>
#include <utility>

#include "attn_jvp.h"
#include "kernels.cuh"

namespace {

using ajvp::MaskSpec;

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxSeq = int64_t(1) << 30;
constexpr int kGridSlots = 1024;  // launches with a grid barrier in flight at once, at most
constexpr size_t kStateBytes = 256 + kGridSlots * sizeof(unsigned long long);

struct DeviceState {
  bool ready = false;
  int status_code = ATTN_JVP_OK;  // why the device is unusable, if it is
  int sm_count = 0;
  int pair_clusters = 0;           // CTA pairs resident at once (0: pair kernel unavailable)
  unsigned int* status = nullptr;  // device status word (bit 0: a bounded wait ran out)
  // Grid-barrier words of the fused rotary-embedding launches (kGridSlots of
  // them after the status word, in the same allocation), and the launch count
  // that tags them.
  unsigned long long* grid_slots = nullptr;
  unsigned int grid_epoch = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
#ifdef AJVP_TRACE
long long* g_trace = nullptr;
#endif

// Per-device set-up, done once under the lock: checks the device is sm_100,
// allocates the 4-byte status word and raises the kernels' shared-memory limit.
int device_state(DeviceState** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return ATTN_JVP_ERR_NO_DEVICE;
  }
  if (dev >= kMaxDevices) return ATTN_JVP_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& st = g_dev[dev];
  if (!st.ready) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&st.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_JVP_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return ATTN_JVP_ERR_NO_DEVICE;  // built for sm_100a only
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn) {
        cudaGetLastError();
        return ATTN_JVP_ERR_CUDA;
      }
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    if (cudaMalloc(&st.status, kStateBytes) != cudaSuccess) {
      cudaGetLastError();
      st.status = nullptr;
      return ATTN_JVP_ERR_CUDA;
    }
    st.grid_slots = reinterpret_cast<unsigned long long*>(reinterpret_cast<char*>(st.status) + 256);
    if (cudaMemset(st.status, 0, kStateBytes) != cudaSuccess ||
        ajvp::tc_prepare(128) != cudaSuccess || ajvp::tc_prepare(64) != cudaSuccess ||
        ajvp::simt_prepare(128) != cudaSuccess || ajvp::simt_prepare(64) != cudaSuccess) {
      cudaGetLastError();
      cudaFree(st.status);
      st.status = nullptr;
      return ATTN_JVP_ERR_CUDA;
    }
    st.pair_clusters = ajvp::tc_pair_max_clusters(st.sm_count);
    st.ready = true;
  }
  *out = &st;
  return ATTN_JVP_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int validate_mask(const attn_jvp_mask& m, int64_t* L_expected) {
  if (m.mode != ATTN_JVP_MASK_TEACHER_FORCING && m.mode != ATTN_JVP_MASK_BLOCK_CAUSAL)
    return ATTN_JVP_ERR_INVALID_ARGUMENT;
  if (m.chunk_tokens < 1 || m.n_chunks < 1) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  const int64_t per = (m.mode == ATTN_JVP_MASK_TEACHER_FORCING) ? 2 : 1;
  const int64_t L = per * int64_t(m.n_chunks) * int64_t(m.chunk_tokens);
  if (L > kMaxSeq) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  *L_expected = L;
  return ATTN_JVP_OK;
}

// Shape checks common to both mask forms (L is checked against the mask by the caller).
int validate_shape(const attn_jvp_shape* s) {
  if (!s) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  if (s->B < 1 || s->H < 1 || s->L < 1) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  if (s->dtype != ATTN_JVP_BF16 && s->dtype != ATTN_JVP_F32) return ATTN_JVP_ERR_UNSUPPORTED;
  if (s->d != 64 && s->d != 128) return ATTN_JVP_ERR_UNSUPPORTED;
  if (!(s->scale <= 0.f || std::isfinite(s->scale))) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  if (s->L > kMaxSeq) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  if (s->B > 65535 || s->H > 65535) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  if (s->B * s->H * ((s->L + ajvp::kTcBlockM - 1) / ajvp::kTcBlockM) > int64_t(1) << 31)
    return ATTN_JVP_ERR_INVALID_ARGUMENT;
  return ATTN_JVP_OK;
}

// A group table: 1..ATTN_JVP_MAX_GROUPS groups whose row_end increase to L,
// each with 0 <= k0_begin <= k0_end <= k1_begin <= k1_end <= L and at least
// one admissible key.
int validate_groups(const attn_jvp_shape* s, const attn_jvp_group* g, int32_t n) {
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
  if (prev != s->L) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  return ATTN_JVP_OK;
}

int validate(const attn_jvp_shape* s, attn_jvp_mask mask) {
  if (!s) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  if (s->B < 1 || s->H < 1 || s->L < 1) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  if (s->dtype != ATTN_JVP_BF16 && s->dtype != ATTN_JVP_F32) return ATTN_JVP_ERR_UNSUPPORTED;
  if (s->d != 64 && s->d != 128) return ATTN_JVP_ERR_UNSUPPORTED;
  if (!(s->scale <= 0.f || std::isfinite(s->scale))) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  int64_t L = 0;
  const int rc = validate_mask(mask, &L);
  if (rc != ATTN_JVP_OK) return rc;
  if (s->L != L) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  if (s->B > 65535 || s->H > 65535) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  // element counts must fit the kernels' 32-bit tile coordinates and 64-bit offsets
  if (s->B * s->H * ((s->L + ajvp::kTcBlockM - 1) / ajvp::kTcBlockM) > int64_t(1) << 31)
    return ATTN_JVP_ERR_INVALID_ARGUMENT;
  return ATTN_JVP_OK;
}

float softmax_scale(const attn_jvp_shape* s) {
  return s->scale > 0.f ? s->scale : 1.0f / std::sqrt(static_cast<float>(s->d));
}

bool encode_bf16_map(CUtensorMap* map, const void* base, const attn_jvp_shape* s, int box_rows) {
  return ajvp::encode_bf16_rows_map(map, base, s->B, s->L, s->H, s->d, box_rows);
}

MaskSpec mask_spec(attn_jvp_mask m, int64_t L) {
  MaskSpec ms;
  ms.mode = m.mode;
  ms.c = m.chunk_tokens;
  ms.n = m.n_chunks;
  ms.L = static_cast<int>(L);
  ms.n_groups = 0;
  ms.groups = nullptr;
  return ms;
}

// A validated group table in the kernels' form (host copy, for the launch).
struct GroupTable {
  ajvp::GroupRange g[ajvp::kMaxGroups];
  int n = 0;
};

MaskSpec groups_spec(const attn_jvp_group* groups, int32_t n, int64_t L, GroupTable* t) {
  for (int32_t i = 0; i < n; ++i)
    t->g[i] = ajvp::GroupRange{groups[i].row_end, groups[i].k0_begin, groups[i].k0_end,
                               groups[i].k1_begin, groups[i].k1_end};
  t->n = n;
  MaskSpec ms;
  ms.mode = ajvp::kModeGroups;
  ms.c = ms.n = 0;
  ms.L = static_cast<int>(L);
  ms.n_groups = n;
  ms.groups = t->g;
  return ms;
}

// The mask as the kernels' parameters carry it: a table (if any) is copied in.
void set_mask(MaskSpec* dst, ajvp::GroupRange* dst_groups, const MaskSpec& ms) {
  *dst = ms;
  if (ms.mode == ajvp::kModeGroups)
    std::memcpy(dst_groups, ms.groups, sizeof(ajvp::GroupRange) * ms.n_groups);
  dst->groups = nullptr;  // the kernels point it at their own parameter copy
}

// Query row blocks (of `bm` rows) of one head, most key tiles first (ties:
// lower block first, the order a stable sort gives). Host scratch is fixed
// thread-local arrays: building the order allocates nothing.
int fill_order(const MaskSpec& ms, int n_qtiles, int bm, uint16_t* order) {
  if (n_qtiles > ajvp::kMaxOrder) return 0;
  static thread_local int cost[ajvp::kMaxOrder];
  static thread_local int idx[ajvp::kMaxOrder];
  for (int t = 0; t < n_qtiles; ++t) {
    cost[t] = ajvp::make_tile_sched(ms, t, bm, ajvp::kTcBlockN).count();
    idx[t] = t;
  }
  std::sort(idx, idx + n_qtiles,
            [&](int a, int b) { return cost[a] != cost[b] ? cost[a] > cost[b] : a < b; });
  for (int r = 0; r < n_qtiles; ++r) order[r] = static_cast<uint16_t>(idx[r]);
  return n_qtiles;
}

// Work lists for `units` units of the persistent grid: head by head (so that
// running units share a head's keys in L2), each query block of the head goes,
// longest first, to the unit with the least work so far (ties: lowest unit).
// Work is the block's key-tile count. Returns false if the lists do not fit.
// The min-heap of unit loads and the per-item assignment live in fixed
// thread-local arrays: no host allocation per call.
bool fill_work_lists(const MaskSpec& ms, int bh_count, int n_qtiles, int bm, int units,
                     const uint16_t* head_order, uint16_t* lists, uint16_t* unit_start) {
  const int n_items = bh_count * n_qtiles;
  if (n_items > ajvp::kMaxOrder || units < 1 || units > ajvp::kMaxUnits) return false;
  static thread_local int cost[ajvp::kMaxOrder];
  static thread_local uint16_t item_pos[ajvp::kMaxOrder];  // assignment order: item position
  static thread_local uint16_t item_unit[ajvp::kMaxOrder];  // and its unit
  static thread_local std::pair<int64_t, int> heap[ajvp::kMaxUnits];  // (work so far, unit)
  for (int t = 0; t < n_qtiles; ++t)
    cost[t] = ajvp::make_tile_sched(ms, t, bm, ajvp::kTcBlockN).count();
  // min-heap on (work, unit): the comparator is "greater"
  const auto cmp = std::greater<std::pair<int64_t, int>>();
  for (int u = 0; u < units; ++u) heap[u] = {0, u};
  std::make_heap(heap, heap + units, cmp);
  int a = 0;
  for (int bh = 0; bh < bh_count; ++bh) {
    for (int r = 0; r < n_qtiles; ++r) {
      const int qt = head_order ? head_order[r] : n_qtiles - 1 - r;
      std::pop_heap(heap, heap + units, cmp);
      std::pair<int64_t, int>& x = heap[units - 1];
      item_pos[a] = static_cast<uint16_t>(bh * n_qtiles + qt);
      item_unit[a] = static_cast<uint16_t>(x.second);
      ++a;
      x.first += cost[qt];
      std::push_heap(heap, heap + units, cmp);
    }
  }
  // Lists in unit order, each unit's items in assignment order.
  for (int u = 0; u <= units; ++u) unit_start[u] = 0;
  for (int i = 0; i < n_items; ++i) ++unit_start[item_unit[i] + 1];
  for (int u = 0; u < units; ++u) unit_start[u + 1] += unit_start[u];
  static thread_local uint16_t fill[ajvp::kMaxUnits];
  for (int u = 0; u < units; ++u) fill[u] = unit_start[u];
  for (int i = 0; i < n_items; ++i) lists[fill[item_unit[i]]++] = item_pos[i];
  return true;
}

// Test-only settings of the bf16 forward launches of this host thread (see
// attn_jvp_debug_wait): the bounded-wait limit and a tile at which unit 0's
// MMA issuer waits on a barrier that nothing completes.
thread_local uint64_t t_wait_ns = 4000000000ull;
thread_local int t_stall_tile = -1;

// Rotary embedding in the same launch: q, k, tq, tk are rotated into the
// four `out` buffers (which the attention then reads) by the cos/sin tables.
struct RopeArgs {
  const float* cos;
  const float* sin;
  void* out[4];
};

int launch_bf16(DeviceState* st, const attn_jvp_shape* s, const void* q, const void* k,
                const void* v, const void* tq, const void* tk, const void* tv, const MaskSpec& ms,
                void* o, void* to, float* lse, cudaStream_t stream,
                const RopeArgs* rope = nullptr) {
  static thread_local ajvp::TcParams p;  // large (order table): not on the stack
  std::memset(&p, 0, offsetof(ajvp::TcParams, order));
  if (rope) {
    const void* src[4] = {q, k, tq, tk};
    for (int i = 0; i < 4; ++i) {
      p.rope_src[i] = src[i];
      p.rope_dst[i] = rope->out[i];
    }
    p.rope = 1;
    p.rope_cos = rope->cos;
    p.rope_sin = rope->sin;
    {
      std::lock_guard<std::mutex> lock(g_mu);
      p.grid_epoch = st->grid_epoch++;
    }
    p.grid_slot = st->grid_slots + (p.grid_epoch % kGridSlots);
    q = rope->out[0];
    k = rope->out[1];
    tq = rope->out[2];
    tk = rope->out[3];
  }
  // d = 128 runs on CTA pairs: each CTA loads 64 of the 128 keys of a K or tK tile.
  const bool pair = s->d == 128;
  if (pair && st->pair_clusters <= 0) return ATTN_JVP_ERR_CUDA;
  const int k_rows = pair ? ajvp::kTcBlockN / 2 : ajvp::kTcBlockN;
  const int bmu = pair ? 2 * ajvp::kTcBlockM : ajvp::kTcBlockM;
  if (!encode_bf16_map(&p.map_q, q, s, ajvp::kTcBlockM) ||
      !encode_bf16_map(&p.map_k, k, s, k_rows) ||
      !encode_bf16_map(&p.map_v, v, s, ajvp::kTcBlockN) ||
      !encode_bf16_map(&p.map_tq, tq, s, ajvp::kTcBlockM) ||
      !encode_bf16_map(&p.map_tk, tk, s, k_rows) ||
      !encode_bf16_map(&p.map_tv, tv, s, ajvp::kTcBlockN))
    return ATTN_JVP_ERR_CUDA;
  p.o = o;
  p.to = to;
  p.lse = lse;
  p.status = st->status;
  p.B = static_cast<int>(s->B);
  p.H = static_cast<int>(s->H);
  p.L = static_cast<int>(s->L);
  p.n_qtiles = static_cast<int>((s->L + bmu - 1) / bmu);
  p.n_items = p.B * p.H * p.n_qtiles;
  set_mask(&p.mask, p.groups, ms);
  const float sc = softmax_scale(s);
  p.scale = sc;
  p.scale_log2 = sc * 1.4426950408889634f;
  p.wait_ns = t_wait_ns;
  p.stall_tile = t_stall_tile;
  p.order_len = fill_order(ms, p.n_qtiles, bmu, p.order);
#ifdef AJVP_TRACE
  p.trace = g_trace;
#endif
  const int grid = pair ? 2 * std::min(st->pair_clusters, p.n_items)
                        : std::min(st->sm_count, p.n_items);
  {
    static thread_local uint16_t head_order[ajvp::kMaxOrder];
    const bool have_order = p.order_len > 0;
    if (have_order) std::memcpy(head_order, p.order, sizeof(uint16_t) * p.n_qtiles);
    p.list_mode = fill_work_lists(ms, p.B * p.H, p.n_qtiles, bmu, pair ? grid / 2 : grid,
                                  have_order ? head_order : nullptr, p.order, p.unit_start)
                      ? 1
                      : 0;
    if (!p.list_mode && have_order) std::memcpy(p.order, head_order, sizeof(uint16_t) * p.n_qtiles);
  }
  if (ajvp::tc_launch(static_cast<int>(s->d), p, grid, stream) != cudaSuccess)
    return ATTN_JVP_ERR_CUDA;
  return ATTN_JVP_OK;
}

int launch_f32(const attn_jvp_shape* s, const void* q, const void* k, const void* v,
               const void* tq, const void* tk, const void* tv, const MaskSpec& ms, void* o,
               void* to, float* lse, cudaStream_t stream) {
  static thread_local ajvp::SimtParams p;  // large (group table): not on the stack
  p.q = static_cast<const float*>(q);
  p.k = static_cast<const float*>(k);
  p.v = static_cast<const float*>(v);
  p.tq = static_cast<const float*>(tq);
  p.tk = static_cast<const float*>(tk);
  p.tv = static_cast<const float*>(tv);
  p.o = static_cast<float*>(o);
  p.to = static_cast<float*>(to);
  p.lse = lse;
  p.B = static_cast<int>(s->B);
  p.H = static_cast<int>(s->H);
  p.L = static_cast<int>(s->L);
  set_mask(&p.mask, p.groups, ms);
  const float sc = softmax_scale(s);
  p.scale = sc;
  p.scale_log2 = sc * 1.4426950408889634f;
  if (ajvp::simt_launch(static_cast<int>(s->d), p, stream) != cudaSuccess) return ATTN_JVP_ERR_CUDA;
  return ATTN_JVP_OK;
}

int64_t round256(int64_t x) { return (x + 255) & ~int64_t(255); }

// attn_jvp_fwd_host: heads in up to kHostChunks chunks (one head per chunk
// when H <= kHostChunks), two staging slots. Small chunks keep the part that
// cannot overlap (the first chunk's copy in, the last chunk's kernel and copy
// out) short: the copies in are the bulk of the call.
constexpr int64_t kHostChunks = 16;

// Copy streams and events of attn_jvp_fwd_host, created once per device and
// kept (like the status word): a call creates nothing.
struct HostPipe {
  std::mutex mu;  // one host-path call at a time per device (the call is synchronous)
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t inp[2] = {nullptr, nullptr}, comp[2] = {nullptr, nullptr},
              outp[2] = {nullptr, nullptr};
};
HostPipe g_pipe[kMaxDevices];

int host_pipe(HostPipe** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return ATTN_JVP_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  HostPipe& pp = g_pipe[dev];
  if (!pp.ready) {
    const unsigned ef = cudaEventDisableTiming;
    bool ok = cudaStreamCreateWithFlags(&pp.in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&pp.out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&pp.start, ef) == cudaSuccess &&
              cudaEventCreateWithFlags(&pp.done, ef) == cudaSuccess;
    for (int i = 0; ok && i < 2; ++i)
      ok = cudaEventCreateWithFlags(&pp.inp[i], ef) == cudaSuccess &&
           cudaEventCreateWithFlags(&pp.comp[i], ef) == cudaSuccess &&
           cudaEventCreateWithFlags(&pp.outp[i], ef) == cudaSuccess;
    if (!ok) {
      cudaGetLastError();
      return ATTN_JVP_ERR_CUDA;
    }
    pp.ready = true;
  }
  *out = &pp;
  return ATTN_JVP_OK;
}

// Pointer checks and the launch for either dtype (shape and mask validated).
int run_checked(const attn_jvp_shape* shape, const void* q, const void* k, const void* v,
                const void* tq, const void* tk, const void* tv, const MaskSpec& ms, void* o,
                void* to, float* lse, void* stream) {
  const void* ptrs[9] = {q, k, v, tq, tk, tv, o, to, lse};
  for (const void* ptr : ptrs)
    if (!ptr) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return ATTN_JVP_ERR_MISALIGNED;
  DeviceState* st = nullptr;
  const int rc = device_state(&st);
  if (rc != ATTN_JVP_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (shape->dtype == ATTN_JVP_BF16) return launch_bf16(st, shape, q, k, v, tq, tk, tv, ms, o, to, lse, s);
  return launch_f32(shape, q, k, v, tq, tk, tv, ms, o, to, lse, s);
}

// ---- allocation-free variant ---------------------------------------------
// Scratch of attn_jvp_fwd_noalloc: a file-scope device array (one per device
// that loads the library). Word 0 is the kernel's status word; the rest is
// reserved. Host code must not pass `g_noalloc_scratch` itself to a kernel (on
// the host it is only a stand-in symbol): its device address comes from
// cudaGetSymbolAddress, looked up once per device below.
constexpr int kNoAllocScratchWords = ATTN_JVP_NOALLOC_SCRATCH_BYTES / 4;
constexpr int kNoAllocWordsNeeded = 1;
static __device__ __align__(256) unsigned int g_noalloc_scratch[kNoAllocScratchWords];

struct NoAllocState {
  bool ready = false;
  int sm_count = 0;
  int pair_clusters = 0;
  unsigned int* scratch = nullptr;  // device address of g_noalloc_scratch on this device
};
NoAllocState g_noalloc[kMaxDevices];

// Per-device set-up without any allocation: device check, tensor-map encoder,
// kernel attributes and the scratch array's device address.
int noalloc_state(NoAllocState** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return ATTN_JVP_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  NoAllocState& st = g_noalloc[dev];
  if (!st.ready) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&st.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_JVP_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return ATTN_JVP_ERR_NO_DEVICE;
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn) {
        cudaGetLastError();
        return ATTN_JVP_ERR_CUDA;
      }
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || addr == nullptr) {
      cudaGetLastError();
      return ATTN_JVP_ERR_CUDA;
    }
    if (ajvp::tc_prepare(128) != cudaSuccess || ajvp::tc_prepare(64) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_JVP_ERR_CUDA;
    }
    st.scratch = static_cast<unsigned int*>(addr);
    st.pair_clusters = ajvp::tc_pair_max_clusters(st.sm_count);
    st.ready = true;
  }
  *out = &st;
  return ATTN_JVP_OK;
}


}  // namespace

namespace ajvp {

int device_status_word(unsigned int** word) {
  DeviceState* st = nullptr;
  const int rc = device_state(&st);
  if (rc != ATTN_JVP_OK) return rc;
  *word = st->status;
  return ATTN_JVP_OK;
}

bool encode_bf16_rows_map(CUtensorMap* map, const void* base, int64_t B, int64_t L, int64_t H,
                          int64_t d, int box_rows) {
  if (!g_encode) return false;
  const cuuint64_t dims[4] = {cuuint64_t(d), cuuint64_t(H), cuuint64_t(L), cuuint64_t(B)};
  const cuuint64_t strides[3] = {cuuint64_t(d) * 2, cuuint64_t(H * d) * 2,
                                 cuuint64_t(L * H * d) * 2};
  const cuuint32_t box[4] = {64, 1, cuuint32_t(box_rows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace ajvp

extern "C" {

int attn_jvp_fwd(const attn_jvp_shape* shape, const void* q, const void* k, const void* v,
                 const void* tq, const void* tk, const void* tv, attn_jvp_mask mask, void* o,
                 void* to, float* lse, void* stream) {
  const int rc = validate(shape, mask);
  if (rc != ATTN_JVP_OK) return rc;
  return run_checked(shape, q, k, v, tq, tk, tv, mask_spec(mask, shape->L), o, to, lse, stream);
}

int attn_jvp_fwd_rope(const attn_jvp_shape* shape, const void* q, const void* k, const void* v,
                      const void* tq, const void* tk, const void* tv, const float* cos,
                      const float* sin, attn_jvp_mask mask, void* q_rot, void* k_rot,
                      void* tq_rot, void* tk_rot, void* o, void* to, float* lse, void* stream) {
  const int rc = validate(shape, mask);
  if (rc != ATTN_JVP_OK) return rc;
  const void* ptrs[15] = {q, k, v, tq, tk, tv, cos, sin, q_rot, k_rot, tq_rot, tk_rot, o, to, lse};
  for (const void* ptr : ptrs)
    if (!ptr) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return ATTN_JVP_ERR_MISALIGNED;
  // the fused rotation counts 16-byte vectors of the four tensors in 32 bits
  if (shape->B * shape->L * shape->H * (shape->d / 2) >= (int64_t(1) << 32)) return ATTN_JVP_ERR_UNSUPPORTED;
  if (shape->dtype == ATTN_JVP_F32) {
    // fp32: the stand-alone rotation pass, then the CUDA-core attention kernel
    const int r = attn_jvp_rope(shape, q, k, tq, tk, cos, sin, q_rot, k_rot, tq_rot, tk_rot, stream);
    if (r != ATTN_JVP_OK) return r;
    return run_checked(shape, q_rot, k_rot, v, tq_rot, tk_rot, tv, mask_spec(mask, shape->L), o, to,
                       lse, stream);
  }
  DeviceState* st = nullptr;
  const int r = device_state(&st);
  if (r != ATTN_JVP_OK) return r;
  RopeArgs rope{cos, sin, {q_rot, k_rot, tq_rot, tk_rot}};
  return launch_bf16(st, shape, q, k, v, tq, tk, tv, mask_spec(mask, shape->L), o, to, lse,
                     static_cast<cudaStream_t>(stream), &rope);
}

int attn_jvp_fwd_groups(const attn_jvp_shape* shape, const void* q, const void* k, const void* v,
                        const void* tq, const void* tk, const void* tv,
                        const attn_jvp_group* groups, int32_t n_groups, void* o, void* to,
                        float* lse, void* stream) {
  int rc = validate_shape(shape);
  if (rc != ATTN_JVP_OK) return rc;
  rc = validate_groups(shape, groups, n_groups);
  if (rc != ATTN_JVP_OK) return rc;
  static thread_local GroupTable table;
  const MaskSpec ms = groups_spec(groups, n_groups, shape->L, &table);
  return run_checked(shape, q, k, v, tq, tk, tv, ms, o, to, lse, stream);
}

int64_t attn_jvp_host_staging_bytes(const attn_jvp_shape* shape) {
  if (!shape || shape->B < 1 || shape->L < 1 || shape->H < 1 || shape->d < 1) return 0;
  if (shape->dtype != ATTN_JVP_BF16 && shape->dtype != ATTN_JVP_F32) return 0;
  const int64_t esz = shape->dtype == ATTN_JVP_BF16 ? 2 : 4;
  const int64_t n_chunks = shape->H >= kHostChunks ? kHostChunks : shape->H;
  const int64_t hc = (shape->H + n_chunks - 1) / n_chunks;
  const int64_t slot = 8 * round256(shape->B * shape->L * hc * shape->d * esz) +
                       round256(shape->B * hc * shape->L * 4);
  return (n_chunks > 1 ? 2 : 1) * slot;
}

int attn_jvp_fwd_host(const attn_jvp_shape* shape, const void* h_q, const void* h_k,
                      const void* h_v, const void* h_tq, const void* h_tk, const void* h_tv,
                      attn_jvp_mask mask, void* h_o, void* h_to, float* h_lse, void* d_buf,
                      void* stream) {
  int rc = validate(shape, mask);
  if (rc != ATTN_JVP_OK) return rc;
  const void* hp[9] = {h_q, h_k, h_v, h_tq, h_tk, h_tv, h_o, h_to, h_lse};
  for (const void* ptr : hp)
    if (!ptr) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  if (!d_buf) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  if (reinterpret_cast<uintptr_t>(d_buf) & 255u) return ATTN_JVP_ERR_MISALIGNED;
  HostPipe* hpp = nullptr;
  rc = host_pipe(&hpp);
  if (rc != ATTN_JVP_OK) return rc;
  HostPipe& pp = *hpp;
  std::lock_guard<std::mutex> call_lock(pp.mu);
  const int64_t B = shape->B, L = shape->L, H = shape->H, d = shape->d;
  const int64_t esz = shape->dtype == ATTN_JVP_BF16 ? 2 : 4;
  // Heads go in chunks of hc: H2D of chunk c+1 (copy stream) overlaps the
  // kernel of chunk c (caller's stream) and the D2H of chunk c-1 (second copy
  // stream), through two staging slots.
  const int64_t n_chunks = H >= kHostChunks ? kHostChunks : H;
  const int64_t hc_max = (H + n_chunks - 1) / n_chunks;
  const int64_t t_slot = round256(B * L * hc_max * d * esz);  // one tensor of a chunk
  const int64_t l_slot = round256(B * hc_max * L * 4);
  const int64_t slot_bytes = 8 * t_slot + l_slot;
  const int n_slots = n_chunks > 1 ? 2 : 1;
  char* base = static_cast<char*>(d_buf);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const void* hin[6] = {h_q, h_k, h_v, h_tq, h_tk, h_tv};
  void* hout[2] = {h_o, h_to};
  const size_t row = static_cast<size_t>(H * d * esz);  // host row pitch (one token, all heads)
  bool ok = true;
  // The copy streams start after work already queued on the caller's stream.
  ok = ok && cudaEventRecord(pp.start, s) == cudaSuccess;
  ok = ok && cudaStreamWaitEvent(pp.in, pp.start, 0) == cudaSuccess;
  ok = ok && cudaStreamWaitEvent(pp.out, pp.start, 0) == cudaSuccess;
  for (int64_t c = 0; ok && c < n_chunks; ++c) {
    const int64_t h0 = c * hc_max;
    const int64_t hc = std::min(hc_max, H - h0);
    if (hc <= 0) break;
    const int sl = static_cast<int>(c % n_slots);
    char* slot = base + sl * slot_bytes;
    void* dt[8];
    for (int i = 0; i < 8; ++i) dt[i] = slot + i * t_slot;
    float* d_lse = reinterpret_cast<float*>(slot + 8 * t_slot);
    const size_t width = static_cast<size_t>(hc * d * esz);
    // inputs of chunk c into slot sl, once the kernel of chunk c - 2 has read them
    if (c >= n_slots) ok = ok && cudaStreamWaitEvent(pp.in, pp.comp[sl], 0) == cudaSuccess;
    for (int i = 0; ok && i < 6; ++i)
      ok = cudaMemcpy2DAsync(dt[i], width, static_cast<const char*>(hin[i]) + h0 * d * esz, row,
                             width, static_cast<size_t>(B * L), cudaMemcpyHostToDevice,
                             pp.in) == cudaSuccess;
    ok = ok && cudaEventRecord(pp.inp[sl], pp.in) == cudaSuccess;
    // the kernel of chunk c, once its inputs are in and chunk c - 2's outputs are out
    ok = ok && cudaStreamWaitEvent(s, pp.inp[sl], 0) == cudaSuccess;
    if (c >= n_slots) ok = ok && cudaStreamWaitEvent(s, pp.outp[sl], 0) == cudaSuccess;
    if (!ok) break;
    attn_jvp_shape cs = *shape;
    cs.H = hc;
    rc = attn_jvp_fwd(&cs, dt[0], dt[1], dt[2], dt[3], dt[4], dt[5], mask, dt[6], dt[7], d_lse,
                      stream);
    if (rc != ATTN_JVP_OK) return rc;
    ok = cudaEventRecord(pp.comp[sl], s) == cudaSuccess;
    // outputs of chunk c to the host
    ok = ok && cudaStreamWaitEvent(pp.out, pp.comp[sl], 0) == cudaSuccess;
    for (int i = 0; ok && i < 2; ++i)
      ok = cudaMemcpy2DAsync(static_cast<char*>(hout[i]) + h0 * d * esz, row, dt[6 + i], width,
                             width, static_cast<size_t>(B * L), cudaMemcpyDeviceToHost,
                             pp.out) == cudaSuccess;
    // LSE: [B, hc, L] of the chunk into rows (b, h0 .. h0 + hc) of [B, H, L]
    ok = ok && cudaMemcpy2DAsync(h_lse + h0 * L, static_cast<size_t>(H * L * 4), d_lse,
                                 static_cast<size_t>(hc * L * 4), static_cast<size_t>(hc * L * 4),
                                 static_cast<size_t>(B), cudaMemcpyDeviceToHost,
                                 pp.out) == cudaSuccess;
    ok = ok && cudaEventRecord(pp.outp[sl], pp.out) == cudaSuccess;
  }
  // The caller's stream ends after the last copy out.
  ok = ok && cudaEventRecord(pp.done, pp.out) == cudaSuccess;
  ok = ok && cudaStreamWaitEvent(s, pp.done, 0) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    return ATTN_JVP_ERR_CUDA;
  }
  return attn_jvp_sync_status(stream);
}

int attn_jvp_sync_status(void* stream) {
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != ATTN_JVP_OK) return rc;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_JVP_ERR_CUDA;
  }
  unsigned int word = 0;
  if (cudaMemcpy(&word, st->status, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_JVP_ERR_CUDA;
  }
  if (word != 0) {
    cudaMemset(st->status, 0, sizeof(unsigned int));
    return ATTN_JVP_ERR_DEVICE_TIMEOUT;
  }
  return ATTN_JVP_OK;
}

const char* attn_jvp_status_string(int status) {
  switch (status) {
    case ATTN_JVP_OK: return "ok";
    case ATTN_JVP_ERR_INVALID_ARGUMENT: return "invalid argument";
    case ATTN_JVP_ERR_UNSUPPORTED: return "unsupported dtype or head dim";
    case ATTN_JVP_ERR_MISALIGNED: return "pointer not aligned";
    case ATTN_JVP_ERR_CUDA: return "CUDA error";
    case ATTN_JVP_ERR_DEVICE_TIMEOUT: return "device wait timed out; outputs invalid";
    case ATTN_JVP_ERR_NO_DEVICE: return "no usable sm_100 device";
    default: return "unknown status";
  }
}

int64_t attn_jvp_unmasked_pairs(attn_jvp_mask mask) {
  int64_t L = 0;
  if (validate_mask(mask, &L) != ATTN_JVP_OK) return -1;
  const int64_t c = mask.chunk_tokens, n = mask.n_chunks;
  const int64_t tf = c * c * n * (n + 1);
  return mask.mode == ATTN_JVP_MASK_TEACHER_FORCING ? tf : tf / 2;
}

int32_t attn_jvp_schedule_tiles_groups(const attn_jvp_group* groups, int32_t n_groups, int64_t L,
                                       int32_t block_m, int32_t block_n, int32_t q_tile,
                                       int32_t* tiles, uint8_t* full, int32_t cap) {
  attn_jvp_shape shape{1, L, 1, 64, ATTN_JVP_BF16, 0.f};
  if (L < 1 || L > kMaxSeq || validate_groups(&shape, groups, n_groups) != ATTN_JVP_OK) return -1;
  if (block_m < 1 || block_n < 1 || q_tile < 0 || cap < 0) return -1;
  if (int64_t(q_tile) * block_m >= L) return -1;
  if ((tiles == nullptr || full == nullptr) && cap > 0) return -1;
  static thread_local GroupTable table;
  const MaskSpec ms = groups_spec(groups, n_groups, L, &table);
  const ajvp::TileSched s = ajvp::make_tile_sched(ms, q_tile, block_m, block_n);
  const int n = s.count();
  for (int i = 0; i < n && i < cap; ++i) {
    tiles[i] = s.tile(i);
    full[i] = s.full(s.tile(i)) ? 1 : 0;
  }
  return n;
}

int32_t attn_jvp_schedule_tiles(attn_jvp_mask mask, int64_t L, int32_t block_m, int32_t block_n,
                                int32_t q_tile, int32_t* tiles, uint8_t* full, int32_t cap) {
  int64_t Lx = 0;
  if (validate_mask(mask, &Lx) != ATTN_JVP_OK || Lx != L) return -1;
  if (block_m < 1 || block_n < 1 || q_tile < 0 || cap < 0) return -1;
  if (int64_t(q_tile) * block_m >= L) return -1;
  if ((tiles == nullptr || full == nullptr) && cap > 0) return -1;
  const MaskSpec ms = mask_spec(mask, L);
  const ajvp::TileSched s = ajvp::make_tile_sched(ms, q_tile, block_m, block_n);
  const int n = s.count();
  for (int i = 0; i < n && i < cap; ++i) {
    tiles[i] = s.tile(i);
    full[i] = s.full(s.tile(i)) ? 1 : 0;
  }
  return n;
}

int32_t attn_jvp_key_tile_query_bounds(attn_jvp_mask mask, int64_t L, int32_t block_m,
                                       int32_t block_n, int32_t k_tile, int32_t* lo, int32_t* hi) {
  int64_t Lx = 0;
  if (validate_mask(mask, &Lx) != ATTN_JVP_OK || Lx != L) return -1;
  if (block_m < 1 || block_n < 1 || k_tile < 0 || !lo || !hi) return -1;
  if (int64_t(k_tile) * block_n >= L) return -1;
  const int n_qt = static_cast<int>((L + block_m - 1) / block_m);
  int a = 0, b = 0;
  ajvp::key_tile_query_bounds(mask_spec(mask, L), k_tile, block_n, n_qt, block_m, a, b);
  *lo = a;
  *hi = b;
  return 0;
}

int32_t attn_jvp_version(void) { return 100; }

int attn_jvp_debug_wait(int64_t limit_ns, int32_t stall_tile) {
  if (limit_ns < 0 || limit_ns > int64_t(60) * 1000000000) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  if (stall_tile < -1) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  t_wait_ns = limit_ns == 0 ? 4000000000ull : static_cast<uint64_t>(limit_ns);
  t_stall_tile = stall_tile;
  return ATTN_JVP_OK;
}

int attn_jvp_fwd_noalloc(const attn_jvp_shape* shape, const void* q, const void* k,
                         const void* v, const void* tq, const void* tk, const void* tv,
                         attn_jvp_mask mask, void* o, void* to, float* lse, void* stream) {
  int rc = validate(shape, mask);
  if (rc != ATTN_JVP_OK) return rc;
  if (shape->dtype != ATTN_JVP_BF16) return ATTN_JVP_ERR_UNSUPPORTED;
  if (kNoAllocWordsNeeded > kNoAllocScratchWords) return ATTN_JVP_ERR_UNSUPPORTED;
  const void* ptrs[9] = {q, k, v, tq, tk, tv, o, to, lse};
  for (const void* ptr : ptrs)
    if (!ptr) return ATTN_JVP_ERR_INVALID_ARGUMENT;
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return ATTN_JVP_ERR_MISALIGNED;
  NoAllocState* st = nullptr;
  rc = noalloc_state(&st);
  if (rc != ATTN_JVP_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The shared word keeps the previous call's value: clear it first.
  if (cudaMemsetAsync(st->scratch, 0, kNoAllocWordsNeeded * sizeof(unsigned int), s) !=
      cudaSuccess) {
    cudaGetLastError();
    return ATTN_JVP_ERR_CUDA;
  }
  DeviceState launch_state;
  launch_state.ready = true;
  launch_state.sm_count = st->sm_count;
  launch_state.pair_clusters = st->pair_clusters;
  launch_state.status = st->scratch;
  rc = launch_bf16(&launch_state, shape, q, k, v, tq, tk, tv, mask_spec(mask, shape->L), o, to, lse,
                   s);
  if (rc != ATTN_JVP_OK) return rc;
  // The word is read back on the same stream (not the legacy default stream),
  // then one wait for the stream covers the kernel and the copy.
  unsigned int word = 0;
  if (cudaMemcpyAsync(&word, st->scratch, sizeof(word), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_JVP_ERR_CUDA;
  }
  return word != 0 ? ATTN_JVP_ERR_DEVICE_TIMEOUT : ATTN_JVP_OK;
}


#ifdef AJVP_TRACE
// Trace builds only: device buffer of kTraceTiles x kTraceEvents int64 clocks
// that the next bf16 launches fill for CTA 0 (NULL disables).
void attn_jvp_set_trace(void* dev_buf) { g_trace = static_cast<long long*>(dev_buf); }
#endif

}  // extern "C"
