/*
 * sta.h -- C ABI of the B200 (sm_100a) Sliding Tile Attention library, libsta.so.
 *
 * Sliding Tile Attention ("Fast Video Generation with Sliding Tile Attention",
 * Abstract; summary page, Methodology and Novelty): the T x H x W tokens of a
 * video latent are grouped into non-overlapping tiles of tile_t x tile_h x
 * tile_w tokens.  Every query tile attends densely to all key tiles inside a
 * window of (w_t, w_h, w_w) tiles around it (window sizes may differ per head,
 * summary page, Methodology), so no attention block is ever partly masked
 * (summary page, Novelty: "eliminating mixed blocks").  The pages do not state
 * the border rule; this library centres the window on the query tile and
 * shifts it inward at the borders so it stays inside the tile grid:
 *     start_d = clamp(qtile_d - floor(w_d / 2), 0, G_d - w_d),
 * with w_d first clamped to the grid size G_d.
 *
 * Conventions shared by every call:
 *   - Tensors are bf16, [batch][heads][N][head_dim] row-major, N = T*H*W, in
 *     raster token order n = (t*H + h)*W + w -- unless the plan was created with
 *     STA_PROBLEM_TILED, in which case token rows are tile-major: all tokens of
 *     tile 0 (tiles ordered t outer, w inner), in-tile order t outer, w inner,
 *     then tile 1, and so on.
 *   - LSE is fp32 [batch][heads][N] (same token order), natural log, the
 *     softmax scale included.
 *   - Device pointers must be 16-byte aligned, otherwise STA_ERR_ALIGNMENT.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Compute calls
 *     only enqueue work and return; they never synchronize unless
 *     STA_CALL_CHECK is passed.
 *   - The caller owns every tensor and the workspace.  A plan owns its device
 *     tables and frees them in sta_plan_destroy.
 *   - A plan's tables live on the device that was current when it was created,
 *     and compute calls (sta_permute, sta_forward, sta_forward_host,
 *     sta_backward, sta_backward_noalloc) enqueue on the calling thread's
 *     current device: a call made while another device is current fails with
 *     STA_ERR_INVALID_ARG and enqueues nothing.
 *   - A plan is immutable after creation and may be used from several streams
 *     at once as long as each concurrent call has its own workspace.
 *   - All argument checking happens on the host before any launch; a failing
 *     call launches nothing.
 */
#ifndef STA_H_
#define STA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  STA_OK = 0,
  STA_ERR_INVALID_ARG = 1, /* null pointer, bad window (< 1), bad flag */
  STA_ERR_SHAPE = 2,       /* tile does not divide T, H or W; sizes < 1; too large */
  STA_ERR_UNSUPPORTED = 3, /* head_dim not 64/128, tile volume not a multiple of 8 */
  STA_ERR_ALIGNMENT = 4,   /* a device pointer is not 16-byte aligned */
  STA_ERR_WORKSPACE = 5,   /* workspace missing or smaller than required */
  STA_ERR_OOM = 6,         /* host or device allocation failed */
  STA_ERR_CUDA = 7,        /* a CUDA runtime call failed */
  STA_ERR_TIMEOUT = 8      /* (STA_CALL_CHECK only) a kernel wait ran out; the
                              kernel stopped early and its outputs are invalid */
} sta_status;

/* sta_problem.flags */
#define STA_PROBLEM_BACKWARD 0x1u /* also build the tables sta_backward needs */
#define STA_PROBLEM_TILED 0x2u    /* tensors use tile-major token order */
#define STA_PROBLEM_HOST_ONLY 0x4u /* build the host tables only (no device, no
                                      upload); compute calls on such a plan fail
                                      with STA_ERR_INVALID_ARG.  For tooling and
                                      for inspecting lists on machines without
                                      a GPU. */
#define STA_PROBLEM_DEVICE_CHECK_TEST 0x10u /* testing only: the plan is built
                                      and uploaded as usual but records a
                                      device number that is never current, so
                                      every compute call on it fails the
                                      device check (STA_ERR_INVALID_ARG) before
                                      anything is enqueued.  Lets a machine
                                      with one GPU test that check. */

/* flags of sta_forward / sta_backward */
#define STA_CALL_CHECK 0x1u /* synchronize `stream` after the launch and report
                               kernel timeouts / CUDA errors in the status */

typedef struct {
  int32_t batch, heads, head_dim;  /* head_dim in {64, 128} */
  int32_t T, H, W;                 /* latent size in tokens */
  int32_t tile_t, tile_h, tile_w;  /* must divide T, H, W exactly; the tile
                                      volume must be a multiple of 8 tokens */
  const int32_t *window;           /* host, heads*3 ints: (w_t, w_h, w_w) per head,
                                      in tiles, each >= 1; larger than the grid
                                      clamps to the grid (= full attention on
                                      that axis).  Copied at plan creation. */
  float scale;                     /* softmax scale; <= 0 means 1/sqrt(head_dim) */
  uint32_t flags;                  /* STA_PROBLEM_* */
} sta_problem;

typedef struct sta_plan_s *sta_plan_t;

/* Build the plan for one problem (the "planner"): validates the problem,
 * computes every head's window start per query tile, the KV-tile list of every
 * (head, query tile) -- the whole key tiles attended, in ascending tile index --
 * and, with STA_PROBLEM_BACKWARD, the inverse lists (for every key tile, the
 * query tiles whose window holds it).  Uploads them to the current device
 * (synchronous cudaMalloc + cudaMemcpy).  *out receives the plan on success and
 * is left untouched on failure.  Size limits (STA_ERR_SHAPE beyond them, before
 * any table is built): batch * heads * T*H*W rows below 2^31 - 1024, and
 * heads * tiles * (largest per-head window in tiles) list entries below
 * 2^31 - 1, since rows and list positions are 32-bit on the device. */
sta_status sta_plan_create(const sta_problem *problem, sta_plan_t *out);

/* Free the plan and its device tables (NULL is accepted).  The caller must
 * ensure no launch that uses the plan is still running. */
sta_status sta_plan_destroy(sta_plan_t plan);

/* Workspace bytes needed by sta_forward and sta_backward (either pointer may
 * be NULL). */
sta_status sta_plan_workspace_size(sta_plan_t plan, size_t *fwd_bytes, size_t *bwd_bytes);

/* Host copy of the KV-tile list of every query tile of one head, for tests and
 * tooling: out[q * per_tile + i] is the i-th key tile (ascending tile-major
 * index t outer, w inner) of query tile q; per_tile = product of the clamped
 * window sizes.  *n receives n_tiles * per_tile; fails with
 * STA_ERR_INVALID_ARG if cap < *n. */
sta_status sta_plan_kv_tiles(sta_plan_t plan, int32_t head, int32_t *out, size_t cap, size_t *n);

/* Host copy of the inverse lists of one head (plan built with
 * STA_PROBLEM_BACKWARD): CSR with offsets[n_tiles + 1] and indices[offsets[n_tiles]];
 * indices[offsets[k] .. offsets[k+1]) are the query tiles (ascending) whose
 * window contains key tile k.  Either output may be NULL to query sizes:
 * *n_indices receives offsets[n_tiles]. */
sta_status sta_plan_q_tiles(sta_plan_t plan, int32_t head, int32_t *offsets, int32_t *indices,
                            size_t cap_indices, size_t *n_indices);

/* Number of tiles of the plan's grid and tokens per tile. */
sta_status sta_plan_geometry(sta_plan_t plan, int32_t *n_tiles, int32_t *tile_volume);

/* Host copy of one of the plan's work lists, for tests and tooling.  Rows of a
 * tile are cut into blocks of 128 (the last one partial): block b of tile t of
 * a (batch, head) slice s = batch * heads + head is numbered t * nb + b, with
 * nb = ceil(tile_volume / 128).
 *   which = STA_WORK_FORWARD (0): the forward's items, 4 int32 each:
 *       (slice, block A, block B or -1, 0).  A and B attend to the same key
 *       tiles; items with B = -1 (lone blocks) come last, *n_lone of them.
 *   which = STA_WORK_FORWARD_HOST (1): the same items in sta_forward_host's
 *       order (slice groups one after another), 4 int32 each.
 *   which = STA_WORK_DKDV (2) / STA_WORK_DQ (3): the backward's items, 2 int32
 *       each: (slice, key block) / (slice, query block); empty for a plan
 *       built without STA_PROBLEM_BACKWARD.
 * *n_items receives the item count (out may be NULL to query it; otherwise
 * cap_items must be >= *n_items, else STA_ERR_INVALID_ARG).  n_lone may be
 * NULL.  This call has no counterpart in the method's description
 * ("Fast Video Generation with Sliding Tile Attention"). */
#define STA_WORK_FORWARD 0
#define STA_WORK_FORWARD_HOST 1
#define STA_WORK_DKDV 2
#define STA_WORK_DQ 3
sta_status sta_plan_work_items(sta_plan_t plan, int32_t which, int32_t *out, size_t cap_items, size_t *n_items,
                               int32_t *n_lone);

/* Number of kernels one sta_forward / sta_backward call of this plan enqueues
 * on its stream (the status-word memset of STA_CALL_CHECK is not counted;
 * `backward` is 0 for a plan built without STA_PROBLEM_BACKWARD).  For sizing
 * CUDA-graph captures and for launch accounting.  Either pointer may be NULL;
 * host-only plans report what a device plan of the same problem launches.
 * This call has no counterpart in the method's description
 * ("Fast Video Generation with Sliding Tile Attention"). */
sta_status sta_plan_launches(sta_plan_t plan, int32_t *forward, int32_t *backward);

/* Token permutation between raster and tile-major order for a bf16 tensor
 * [batch][heads][N][head_dim] of the plan's shape:
 *   inverse == 0: dst[tile-major position of token n] = src[n]   (raster -> tiles)
 *   inverse != 0: dst[n] = src[tile-major position of token n]   (tiles -> raster)
 * src and dst must not overlap.  Enqueued on `stream`. */
sta_status sta_permute(sta_plan_t plan, const void *src, void *dst, int32_t inverse, void *stream);

/* Forward pass: o = softmax(q k^T * scale restricted to each query's window) v,
 * and lse = log-sum-exp of the same scores (nullable).  q, k, v, o are bf16
 * [batch][heads][N][head_dim]; lse is fp32 [batch][heads][N].  The softmax is
 * computed in fp32 with bf16 tensor-core products accumulated in fp32; o is
 * rounded to bf16 (nearest even).  `workspace` must hold at least fwd_bytes of
 * sta_plan_workspace_size (missing or smaller: STA_ERR_WORKSPACE); its first
 * bytes carry the kernel status word that STA_CALL_CHECK reads. */
sta_status sta_forward(sta_plan_t plan, const void *q, const void *k, const void *v, void *o,
                       float *lse, void *workspace, size_t workspace_bytes, void *stream,
                       uint32_t flags);

/* Device workspace that sta_forward_host needs: device copies of q, k, v, o
 * and lse, then sta_forward's own workspace.  This call has no counterpart in
 * the method's description ("Fast Video Generation with Sliding Tile
 * Attention"). */
sta_status sta_plan_host_workspace_size(sta_plan_t plan, size_t *bytes);

/* Forward pass on HOST tensors (same computation and layouts as sta_forward):
 * q, k, v are read from host memory and o (and lse, nullable) written to host
 * memory; `workspace` is device memory of at least
 * sta_plan_host_workspace_size bytes, 16-byte aligned.  The (batch, head)
 * slices are processed in up to 24 groups: the inputs of one group are copied
 * to the device while the previous group is computed, and each group's
 * outputs are copied back while later groups run, on two internal streams
 * ordered against `stream` with events (one cudaMemcpyAsync per tensor and
 * group).  The call returns after enqueueing; when `stream` reaches the end of
 * the call, o and lse are in host memory.  Copies overlap only for page-locked
 * host memory.  With tiles that are not TMA boxes of the raster tensor, the
 * whole tensors are copied in, computed and copied out in order.  Host buffers must stay valid and unchanged until
 * `stream` has passed the call.  This call has no counterpart in the
 * method's description ("Fast Video Generation with Sliding Tile
 * Attention"). */
sta_status sta_forward_host(sta_plan_t plan, const void *q, const void *k, const void *v, void *o, float *lse,
                            void *workspace, size_t workspace_bytes, void *stream, uint32_t flags);

/* Backward pass for the fine-tuning case ("Fast Video Generation with Sliding
 * Tile Attention", Abstract: fine-tuning with STA).  With P = softmax of the
 * windowed scores and D_i = sum_c dO_ic O_ic:
 *   dV = P^T dO;  dS = P o (dO V^T - D);  dQ = scale dS K;  dK = scale dS^T Q,
 * all sums running only over (query, key) pairs inside the window.  Inputs
 * q, k, v, o, dout bf16 and lse fp32 exactly as sta_forward produced them;
 * outputs dq, dk, dv bf16 of the same shape as q.  The plan must have been
 * created with STA_PROBLEM_BACKWARD (else STA_ERR_INVALID_ARG); the workspace
 * must hold bwd_bytes (missing or smaller: STA_ERR_WORKSPACE). */
sta_status sta_backward(sta_plan_t plan, const void *q, const void *k, const void *v,
                        const void *o, const float *lse, const void *dout, void *dq, void *dk,
                        void *dv, void *workspace, size_t workspace_bytes, void *stream,
                        uint32_t flags);

/* sta_backward without a caller workspace.  (No counterpart in the method's
 * description: this is a calling convention of this library.)  Meant for
 * callers that cannot allocate device memory where they run the backward
 * pass -- for example when a framework's caching allocator already owns the
 * whole device, or on a path
 * where the memory footprint must not change once set up -- and so cannot hand
 * over a workspace.  The temporaries go to a file-scope device array of 32 MiB
 * inside libsta.so instead; every GPU that loads the library holds that array
 * until the process exits.  Same arguments, results, flags and argument
 * checks as sta_backward, minus the workspace.
 *   - Fails with STA_ERR_WORKSPACE when the plan's backward workspace
 *     (sta_plan_workspace_size, bwd_bytes) exceeds 32 MiB; the other argument
 *     errors are those of sta_backward.  A failing call enqueues nothing.
 *   - Uses the array of the plan's device, which must be the current one (as
 *     for every compute call).  The first call on a device looks up the
 *     array's device address (cudaGetSymbolAddress, with that device
 *     current); make that first call before any stream capture.
 *   - Allocates nothing: no cudaMalloc / cudaFree, no allocating library call.
 *     Enqueues exactly what sta_backward enqueues (with STA_CALL_CHECK, that
 *     includes its status-word memset).
 *   - All calls share the one array, which keeps the previous call's contents;
 *     everything a call reads from it is written earlier in the same call (the
 *     status word is cleared by STA_CALL_CHECK, which alone reads it).  Calls
 *     that overlap on the GPU (other streams, other host threads on the same
 *     device) race on it: order them. */
sta_status sta_backward_noalloc(sta_plan_t plan, const void *q, const void *k, const void *v,
                                const void *o, const float *lse, const void *dout, void *dq,
                                void *dk, void *dv, void *stream, uint32_t flags);

/* Process-wide limit, in nanoseconds, on every barrier wait inside the
 * kernels launched after this call (default 2 s).  When a wait runs out the
 * kernel stops early, records the error in the workspace status word and
 * returns; a call made with STA_CALL_CHECK then reports STA_ERR_TIMEOUT.  This
 * is the hook the failure-detection tests use; ordinary callers never need it. */
void sta_set_wait_limit_ns(uint64_t ns);

/* Static description of a status code. */
const char *sta_status_string(sta_status status);

#ifdef __cplusplus
}
#endif

#endif /* STA_H_ */
