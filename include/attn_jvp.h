/*
 * attn_jvp.h - C ABI of the B200 (sm_100a) custom-mask attention + JVP library.
 *
 * The operation (Causal-rCM summary page, App. B "FlashAttention-2 JVP Kernel
 * with Custom Masks"): for queries Q, keys K, values V and tangents tQ, tK,
 * tV, with softmax scale s and an additive mask M (0 where a query may attend
 * to a key, -inf elsewhere),
 *
 *     S  = s Q K^T + M,        P  = softmax(S) (row-wise),    O = P V
 *     tS = s (tQ K^T + Q tK^T)
 *     tP = P * (tS - rowsum(P * tS))                (elementwise *)
 *     tO = tP V + P tV
 *     LSE_i = log sum_j exp(S_ij)                   (natural log)
 *
 * Masked entries receive no tangent, because the discrete mask has none
 * (App. B); the tangent uses exactly the primal masked operator and the same
 * sparse schedule (App. B). The library returns the primal output, the
 * log-sum-exp values and the tangent output (App. B, last item).
 *
 * Masks are given as {mode, chunk_tokens c, n_chunks n}:
 *   ATTN_JVP_MASK_TEACHER_FORCING: the packed sequence [clean chunks | noisy
 *     chunks], L = 2 n c (Causal-rCM page, section 3 "Continuous-time
 *     consistency", TF-masked packed forward; Causal Forcing summary page,
 *     section 2, clean and noisy videos concatenated under a causal mask).
 *     A clean query in chunk j attends to clean chunks <= j. A noisy query in
 *     chunk i attends to clean chunks < i and to its own noisy chunk.
 *   ATTN_JVP_MASK_BLOCK_CAUSAL: L = n c; a query in chunk j attends to
 *     chunks <= j (Causal-rCM page, section 2 "Autoregressive video
 *     diffusion": causal across temporal blocks, full attention inside one).
 * Attention inside one chunk is full in both modes.
 *
 * Layout: q, k, v, tq, tk, tv, o, to are dense row-major [B, L, H, d] arrays
 * (d innermost) of the element type `dtype`; lse is a dense [B, H, L] float
 * array. All of them are DEVICE pointers of the current CUDA device unless a
 * function says otherwise.
 *
 * Ownership: the caller owns every buffer; the library never frees or keeps
 * a caller pointer after the call returns (work is stream-ordered: buffers
 * must stay valid until the stream reaches the launched work). The library
 * keeps, per device, a small status word and cached tensor-map descriptors;
 * it allocates nothing else. Outputs must not overlap inputs or each other.
 *
 * Errors: every function returns an int status (ATTN_JVP_OK = 0 on success)
 * and never throws. Argument errors are detected on the host before anything
 * is launched. attn_jvp_fwd does not synchronize; device-side faults of the
 * launched work (a bounded wait that ran out) are reported later by
 * attn_jvp_sync_status.
 *
 * Threading: functions may be called from several host threads; the cached
 * descriptors are protected by a lock.
 */
#ifndef ATTN_JVP_H_
#define ATTN_JVP_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------- */
enum {
  ATTN_JVP_OK = 0,
  ATTN_JVP_ERR_INVALID_ARGUMENT = 1, /* null pointer, bad size, L inconsistent with the mask */
  ATTN_JVP_ERR_UNSUPPORTED = 2,      /* dtype or head_dim the kernels do not implement */
  ATTN_JVP_ERR_MISALIGNED = 3,       /* a pointer is not 16-byte aligned */
  ATTN_JVP_ERR_CUDA = 4,             /* a CUDA runtime or driver call failed */
  ATTN_JVP_ERR_DEVICE_TIMEOUT = 5,   /* a kernel's bounded wait ran out; the outputs are invalid */
  ATTN_JVP_ERR_NO_DEVICE = 6         /* no usable sm_100 device */
};

/* ---- mask ------------------------------------------------------------ */
typedef enum {
  ATTN_JVP_MASK_TEACHER_FORCING = 0,
  ATTN_JVP_MASK_BLOCK_CAUSAL = 1
} attn_jvp_mask_mode;

typedef struct {
  int32_t mode;         /* attn_jvp_mask_mode */
  int32_t chunk_tokens; /* c >= 1: tokens per chunk (one latent frame = 1560 in Wan2.1) */
  int32_t n_chunks;     /* n >= 1 */
} attn_jvp_mask;

/*
 * General masks (Causal-rCM summary page, App. B: the kernel takes masks as
 * query groups with admissible key ranges). Group g covers the query rows
 * [row_end of group g-1 (0 for g = 0), row_end of group g); each of those rows
 * may attend to keys [k0_begin, k0_end) and [k1_begin, k1_end). A table lists
 * 1 to ATTN_JVP_MAX_GROUPS groups in row order, the last ending at L, with
 * 0 <= k0_begin <= k0_end <= k1_begin <= k1_end <= L and at least one key per
 * group (either range may be empty). The teacher-forcing mask is such a table
 * with one group per chunk of rows (clean chunks, then noisy chunks).
 */
#define ATTN_JVP_MAX_GROUPS 512
typedef struct {
  int32_t row_end;
  int32_t k0_begin, k0_end;
  int32_t k1_begin, k1_end;
} attn_jvp_group;

/* ---- problem --------------------------------------------------------- */
typedef enum {
  ATTN_JVP_BF16 = 0, /* bf16 inputs/outputs, fp32 accumulation, tensor cores */
  ATTN_JVP_F32 = 1   /* fp32 inputs/outputs, fp32 arithmetic on CUDA cores */
} attn_jvp_dtype;

typedef struct {
  int64_t B;     /* batch >= 1 */
  int64_t L;     /* sequence length: 2 n c (teacher forcing) or n c (block causal) */
  int64_t H;     /* heads >= 1 */
  int64_t d;     /* head dim: 64 or 128 */
  int32_t dtype; /* attn_jvp_dtype */
  float scale;   /* softmax scale s; <= 0 selects 1/sqrt(d) */
} attn_jvp_shape;

/*
 * attn_jvp_fwd - O, tO and LSE of masked softmax attention and its JVP in one
 * fused pass (App. B: same online-softmax pass and shared rescaling for the
 * primal and tangent accumulators; fully masked key tiles are skipped).
 *
 *   shape   problem sizes and element type (host pointer, read during the call)
 *   q..tv   device inputs, [B, L, H, d] of `shape->dtype`, 16-byte aligned
 *   mask    mask mode and chunking; L must equal 2 n c or n c
 *   o, to   device outputs, [B, L, H, d] of `shape->dtype`, 16-byte aligned
 *   lse     device output, [B, H, L] float (natural-log log-sum-exp of the
 *           scaled, masked scores)
 *   stream  cudaStream_t to launch on (NULL = legacy default stream)
 *
 * Returns ATTN_JVP_OK after enqueueing the work, or an error code with
 * nothing launched. The call does not synchronize with the device.
 */
int attn_jvp_fwd(const attn_jvp_shape* shape,
                 const void* q, const void* k, const void* v,
                 const void* tq, const void* tk, const void* tv,
                 attn_jvp_mask mask,
                 void* o, void* to, float* lse,
                 void* stream);

/*
 * attn_jvp_fwd_groups - attn_jvp_fwd with a general mask given as a table of
 * row groups (see attn_jvp_group) instead of {mode, c, n}: same operation,
 * layouts, outputs and asynchronous behaviour.
 *
 *   groups    host array of n_groups groups; read during the call only (it is
 *             copied into the launch), the caller keeps ownership
 *   n_groups  1 .. ATTN_JVP_MAX_GROUPS
 *
 * Returns ATTN_JVP_ERR_INVALID_ARGUMENT for a table that breaks the rules
 * above (rows not increasing to L, ranges out of order or outside [0, L), a
 * group with no key) and ATTN_JVP_ERR_UNSUPPORTED for more than
 * ATTN_JVP_MAX_GROUPS groups; nothing is launched then. Each query block is
 * scheduled over the union of its rows' ranges, so key tiles in a gap of that
 * union are visited (and fully masked); tables whose neighbouring groups have
 * similar ranges waste little.
 */
int attn_jvp_fwd_groups(const attn_jvp_shape* shape,
                        const void* q, const void* k, const void* v,
                        const void* tq, const void* tk, const void* tv,
                        const attn_jvp_group* groups, int32_t n_groups,
                        void* o, void* to, float* lse,
                        void* stream);

/*
 * attn_jvp_fwd_host - the same operation on HOST buffers: copies the six
 * inputs host->device, runs attn_jvp_fwd, copies O, tO and LSE device->host
 * and waits for the stream. Host buffers should be pinned (page-locked) for
 * the copies to run at full speed (and to overlap with the kernel); pageable
 * memory also works.
 *
 * The heads go in up to 16 chunks (one head per chunk when H <= 16) through
 * two staging slots: the copies in
 * of chunk c+1 and the copies out of chunk c-1 run on two copy streams while
 * the kernel of chunk c runs on `stream`, ordered by events. The copy
 * streams and events are created on the first call on a device and kept
 * (like the status word); calls on one device are serialised by a lock.
 * Results are the same bits as attn_jvp_fwd on the same inputs.
 *
 *   h_q..h_tv  host inputs, [B, L, H, d]
 *   h_o, h_to  host outputs, [B, L, H, d];  h_lse host output [B, H, L]
 *   d_buf      caller-owned device staging buffer of at least
 *              attn_jvp_host_staging_bytes(shape) bytes, 256-byte aligned
 *   stream     stream for the copies and the kernel
 *
 * Returns the status of the whole sequence, including any device fault
 * (the call synchronizes on `stream`).
 */
int attn_jvp_fwd_host(const attn_jvp_shape* shape,
                      const void* h_q, const void* h_k, const void* h_v,
                      const void* h_tq, const void* h_tk, const void* h_tv,
                      attn_jvp_mask mask,
                      void* h_o, void* h_to, float* h_lse,
                      void* d_buf, void* stream);

/* Bytes of device staging attn_jvp_fwd_host needs for `shape` (0 on a bad shape):
 * two slots of one chunk of heads (8 tensors and the LSE of ceil(H / 16) heads,
 * each piece rounded up to 256 bytes), or one slot of the whole problem when H = 1. */
int64_t attn_jvp_host_staging_bytes(const attn_jvp_shape* shape);

/*
 * attn_jvp_sync_status - synchronizes `stream`, then reports and clears the
 * device status word of the current device: ATTN_JVP_ERR_DEVICE_TIMEOUT if a
 * kernel gave up on a bounded wait since the last call, ATTN_JVP_ERR_CUDA if
 * the stream reported an error, else ATTN_JVP_OK.
 */
int attn_jvp_sync_status(void* stream);

/* Static, NUL-terminated description of a status code. */
const char* attn_jvp_status_string(int status);

/*
 * attn_jvp_fwd_noalloc - attn_jvp_fwd for callers that cannot allocate device
 * memory (an allocator-free runtime, a plugin host that owns every device
 * buffer, code running where cudaMalloc is forbidden or would break a memory
 * budget). It allocates no device memory: not on the first call, not later.
 * (Its host-side work lists are built in fixed thread-local arrays, not on
 * the heap.) There is no counterpart in the pages; it is an addition of this
 * library.
 *
 * The bf16 kernel needs one word of scratch device memory besides its inputs
 * and outputs: the status word that a bounded wait sets when it runs out.
 * attn_jvp_fwd keeps that word in memory the library allocates once per
 * device. This entry point instead uses a fixed file-scope device array of
 * ATTN_JVP_NOALLOC_SCRATCH_BYTES bytes (ATTN_JVP_NOALLOC_SCRATCH_BYTES / 4
 * words, of which this version uses 1), which every GPU that loads the
 * library holds until the process exits. The scratch does not grow with the
 * problem; the entry point rejects any layout that would need more words than
 * the array holds with ATTN_JVP_ERR_UNSUPPORTED, and rejects problems the
 * kernels cannot run exactly as attn_jvp_fwd does.
 *
 * Only bf16 is accepted (the fp32 kernel needs no scratch; use attn_jvp_fwd).
 * Arguments, layout and outputs are those of attn_jvp_fwd. Unlike it, this
 * call is synchronous: it clears the scratch word on `stream`, launches,
 * copies the word back on `stream`, waits for `stream` and returns the
 * status of the launched work, so a bounded-wait timeout is reported here as
 * ATTN_JVP_ERR_DEVICE_TIMEOUT.
 *
 * The first call on a device (with that device current) looks up the array's
 * device address and the kernels' launch attributes; make that first call
 * before any stream capture. All calls share the one array: calls that
 * overlap on the GPU (other threads or streams) race on it.
 */
#define ATTN_JVP_NOALLOC_SCRATCH_BYTES 256
int attn_jvp_fwd_noalloc(const attn_jvp_shape* shape,
                         const void* q, const void* k, const void* v,
                         const void* tq, const void* tk, const void* tv,
                         attn_jvp_mask mask,
                         void* o, void* to, float* lse,
                         void* stream);

/* ---- backward of the primal attention --------------------------------- */

/*
 * attn_jvp_bwd - gradients dQ, dK, dV of the masked primal attention
 * O = softmax(s Q K^T + M) V, for training the network whose forward
 * attn_jvp_fwd computes. The fused forward returns LSE so that a backward
 * pass can rebuild P without a second softmax pass (Causal-rCM summary page,
 * App. B, last item); the pages say nothing more about the backward, and
 * this is the plain gradient under the same mask:
 *
 *     P_ij  = exp(s q_i . k_j - LSE_i) on admissible pairs, 0 elsewhere
 *     D_i   = dO_i . O_i - dLSE_i
 *     dS_ij = P_ij ((dO_i . v_j) - D_i)
 *     dV = P^T dO,    dK = s dS^T Q,    dQ = s dS K
 *
 * (dLSE is an optional cotangent of LSE; with it the result is the gradient
 * of a loss that also depends on LSE.)
 *
 *   shape      as for attn_jvp_fwd (same dtype, d and scale rules)
 *   q, k, v    device inputs of the forward, [B, L, H, d] of shape->dtype
 *   o          the forward's output O, [B, L, H, d] of shape->dtype
 *   dout       the cotangent dO of O, [B, L, H, d] of shape->dtype
 *   lse        the forward's LSE, [B, H, L] float (natural log)
 *   dlse       cotangent of LSE, [B, H, L] float, or NULL for none
 *   mask       the forward's mask
 *   dq, dk, dv device outputs, [B, L, H, d] of shape->dtype
 *   stream     cudaStream_t to launch on
 *
 * All pointers 16-byte aligned; outputs must not overlap inputs or each
 * other. Each output element has one writer, so results are the same bits
 * on every run. Keys that no row may attend to get zero gradients. lse must
 * be the forward's (finite) LSE of these inputs.
 *
 * bf16 (when 8 * 128 ceil(L/128) <= 2 d L, i.e. L >= 8 for d = 64 and
 * L >= 4 for d = 128): tensor cores, fp32 accumulation, P and dS rounded to
 * bf16 before the dV, dK and dQ products, outputs rounded to nearest even.
 * Three launches: per-row D_i = dO_i . O_i - dLSE_i and LSE_i log2(e) (fp32,
 * written into the dq buffer, which serves as scratch until the last launch
 * overwrites it with dQ), then dK and dV per block of 128 keys, then dQ per
 * block of 128 query rows. Its waits are bounded: a wait that runs out is
 * reported by attn_jvp_sync_status as ATTN_JVP_ERR_DEVICE_TIMEOUT.
 * fp32 (and bf16 below those lengths): fp32 arithmetic on CUDA cores, two
 * launches (dQ per block of 32 query rows, dK and dV per block of 32 keys).
 *
 * Returns ATTN_JVP_OK after enqueueing, or an error code with nothing
 * launched (argument errors are found on the host before any device call).
 * Does not synchronize.
 */
int attn_jvp_bwd(const attn_jvp_shape* shape,
                 const void* q, const void* k, const void* v,
                 const void* o, const void* dout,
                 const float* lse, const float* dlse,
                 attn_jvp_mask mask,
                 void* dq, void* dk, void* dv,
                 void* stream);

/* attn_jvp_bwd with a group-table mask (validated as for attn_jvp_fwd_groups). */
int attn_jvp_bwd_groups(const attn_jvp_shape* shape,
                        const void* q, const void* k, const void* v,
                        const void* o, const void* dout,
                        const float* lse, const float* dlse,
                        const attn_jvp_group* groups, int32_t n_groups,
                        void* dq, void* dk, void* dv,
                        void* stream);

/* ---- rotary position embedding ahead of the attention ------------------ */

/*
 * attn_jvp_rope - rotary position embedding of q, k and their tangents tq, tk
 * (Causal-rCM summary page, section 3, "KV Cache": RoPE is the positional
 * treatment of queries and keys, one of the attention's neighbours in the
 * layer-level JVP). The pages give no formula; this is the standard rotary
 * embedding on adjacent pairs, with per-token angles phi supplied as tables:
 *
 *     x'_2i   = x_2i cos(phi_ti) - x_2i+1 sin(phi_ti)
 *     x'_2i+1 = x_2i sin(phi_ti) + x_2i+1 cos(phi_ti)
 *
 * for every batch and head of token t. The rotation does not depend on its
 * input, so the tangents of the rotated queries and keys are the rotated
 * tangents; attn_jvp_fwd on the four outputs (with v and tv unchanged) is the
 * attention JVP with RoPE in front.
 *
 *   shape              as for attn_jvp_fwd (dtype, d; scale unused)
 *   q, k, tq, tk       device inputs, [B, L, H, d] of shape->dtype
 *   cos, sin           device tables, [L, d/2] float (token t, pair i)
 *   q_out .. tk_out    device outputs, [B, L, H, d] of shape->dtype; each may be
 *                      its own input (in place), and must not overlap any other
 *   stream             cudaStream_t to launch on
 *
 * All pointers 16-byte aligned. Arithmetic is fp32; bf16 outputs are rounded
 * to nearest even. One launch, one pass over HBM. Returns ATTN_JVP_OK after
 * enqueueing, or an error code with nothing launched; does not synchronize.
 */
int attn_jvp_rope(const attn_jvp_shape* shape,
                  const void* q, const void* k, const void* tq, const void* tk,
                  const float* cos, const float* sin,
                  void* q_out, void* k_out, void* tq_out, void* tk_out,
                  void* stream);

/*
 * attn_jvp_fwd_rope - attn_jvp_fwd with the rotary position embedding of
 * attn_jvp_rope applied to q, k and their tangents tq, tk first, in the same
 * launch for bf16 (Causal-rCM summary page, section 3, "KV Cache": RoPE on
 * queries and keys, the attention's neighbour in the layer-level JVP). The
 * operation is attn_jvp_fwd(R q, R k, v, R tq, R tk, tv) with R the rotation
 * by the cos/sin tables; the rotated tensors R q, R k, R tq, R tk are also
 * returned (the backward of the attention and a post-RoPE key cache need them).
 *
 *   q..tv       device inputs, [B, L, H, d] of shape->dtype
 *   cos, sin    device tables, [L, d/2] float (token t, pair i), as for attn_jvp_rope
 *   mask        as for attn_jvp_fwd
 *   q_rot..tk_rot  device outputs, [B, L, H, d]: the rotated q, k, tq, tk; each
 *               may be its own input (in place) and must not overlap any other
 *   o, to, lse  device outputs, as for attn_jvp_fwd
 *   stream      cudaStream_t to launch on
 *
 * bf16: one kernel launch. Its CTAs first rotate a share of q, k, tq, tk
 * each (one pass over HBM), meet at a bounded grid barrier and then run the
 * attention on the rotated tensors. The launch is cooperative (all its CTAs
 * resident at once, or it fails with ATTN_JVP_ERR_CUDA). The barrier uses
 * one of 1024 per-device words, tagged by a per-device launch count, so up
 * to 1024 such calls may be in flight on a device at once. fp32: the
 * rotation pass and then the CUDA-core kernel (two launches).
 *
 * All pointers 16-byte aligned; B * L * H * head_dim / 2 < 2^32 (else
 * ATTN_JVP_ERR_UNSUPPORTED).
 * Returns ATTN_JVP_OK after enqueueing, or an error code with nothing
 * launched. Does not synchronize; a bounded wait that runs out (the grid
 * barrier included) is reported by attn_jvp_sync_status.
 */
int attn_jvp_fwd_rope(const attn_jvp_shape* shape,
                      const void* q, const void* k, const void* v,
                      const void* tq, const void* tk, const void* tv,
                      const float* cos, const float* sin,
                      attn_jvp_mask mask,
                      void* q_rot, void* k_rot, void* tq_rot, void* tk_rot,
                      void* o, void* to, float* lse,
                      void* stream);

/* ---- host-side helpers (need no GPU) ---------------------------------- */

/* Number of admissible (query, key) pairs per (batch, head):
 * c^2 n (n+1) for teacher forcing, c^2 n (n+1) / 2 for block causal; -1 on a
 * bad mask. Effective FLOPs of one call are 12 d B H times this. */
int64_t attn_jvp_unmasked_pairs(attn_jvp_mask mask);

/*
 * attn_jvp_schedule_tiles - the key-tile schedule the bf16 kernel runs for one
 * query tile (App. B: masks as query groups with admissible key ranges; the
 * same sparse schedule drives primal and tangent scores).
 *
 *   mask, L       mask and sequence length (validated as for attn_jvp_fwd)
 *   block_m/_n    query / key tile sizes (rows / columns)
 *   q_tile        query tile index, 0 <= q_tile < ceil(L / block_m)
 *   tiles, full   caller arrays of `cap` entries: key tile indices in visit
 *                 order, and 1 where every (query, key) pair of the tile is
 *                 admissible (no element mask needed), 0 where it is partial
 *   cap           capacity of both arrays
 *
 * Returns the number of key tiles (>= 0; entries beyond `cap` are not
 * written) or -1 on a bad argument. Key tiles not listed are fully masked.
 */
int32_t attn_jvp_schedule_tiles(attn_jvp_mask mask, int64_t L, int32_t block_m,
                                int32_t block_n, int32_t q_tile,
                                int32_t* tiles, uint8_t* full, int32_t cap);

/*
 * attn_jvp_schedule_tiles_groups - the same for a group-table mask (the table
 * validated as for attn_jvp_fwd_groups, L = its last row_end). Returns the
 * number of key tiles or -1 on a bad argument.
 */
int32_t attn_jvp_schedule_tiles_groups(const attn_jvp_group* groups, int32_t n_groups, int64_t L,
                                       int32_t block_m, int32_t block_n, int32_t q_tile,
                                       int32_t* tiles, uint8_t* full, int32_t cap);

/*
 * attn_jvp_key_tile_query_bounds - the range of query tiles [*lo, *hi] that
 * the backward's dK/dV kernel scans for key tile k_tile (the transpose of
 * the schedule above: the query tiles whose schedule lists the key tile all
 * lie in the range). Exact for the closed-form masks (teacher forcing: clean
 * keys are seen from their chunk's clean rows on, noisy keys only by their
 * own chunk's noisy rows; block causal: from the key's chunk on).
 *
 *   mask, L       mask and sequence length (validated as for attn_jvp_fwd)
 *   block_m/_n    query / key tile sizes
 *   k_tile        key tile index, 0 <= k_tile < ceil(L / block_n)
 *
 * Returns 0, or -1 on a bad argument (nothing written).
 */
int32_t attn_jvp_key_tile_query_bounds(attn_jvp_mask mask, int64_t L, int32_t block_m,
                                       int32_t block_n, int32_t k_tile, int32_t* lo, int32_t* hi);

/*
 * attn_jvp_debug_wait - TEST ONLY: drives the bf16 forward kernels' bounded
 * waits to run out without a device fault (a wait on a barrier that nothing
 * completes), so that the timeout path can be tested. Not part of the
 * operation (the pages have no counterpart); it exists for failure-detection
 * tests.
 *
 *   limit_ns    limit of every bounded wait of the bf16 forward kernels
 *               launched later from the calling host thread; 0 restores
 *               the default of 4 s (at most 60 s)
 *   stall_tile  -1: no stall. >= 0: in those launches the first work unit's
 *               MMA issuer, at its stall_tile-th key tile, waits on a barrier
 *               that nothing completes. The wait runs out after limit_ns, the
 *               kernel drains the copies and MMAs in flight, frees its tensor
 *               memory and returns; attn_jvp_sync_status (or
 *               attn_jvp_fwd_noalloc itself) reports
 *               ATTN_JVP_ERR_DEVICE_TIMEOUT and the outputs are invalid.
 *
 * The settings are per host thread and stay until changed; call
 * attn_jvp_debug_wait(0, -1) to restore normal operation. Returns
 * ATTN_JVP_ERR_INVALID_ARGUMENT for values out of range.
 */
int attn_jvp_debug_wait(int64_t limit_ns, int32_t stall_tile);

/* Library version, major * 10000 + minor * 100 + patch. */
int32_t attn_jvp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_JVP_H_ */
