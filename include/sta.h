/*
 * sta.h -- C ABI of the Sliding Tile Attention (STA) library (libsta): forward
 * and backward passes.
 *
 * The method: "Fast Video Generation with Sliding Tile Attention".  A video
 * latent of L_t x L_h x L_w tokens is cut into tiles, contiguous cubes of
 * T_t x T_h x T_w tokens whose size equals one attention block (podcast
 * transcript at hotaipapers.com, segment on tiles and FlashAttention blocks).
 * Each query tile attends, with exact softmax, only to the key/value tiles
 * inside a 3D window of tiles centred on it; the window slides tile by tile, so
 * all queries of a tile share one key set and every computed block is dense
 * (same transcript, segment on dense / empty / mixed blocks; dianyo.github.io
 * ICML-2025 post, STA section "Observation & Proposed Method").  The window is
 * chosen per head (transcript, segment on head specialisation).
 *
 * Readings fixed by this library where the pages are silent:
 *   - window extent in tiles e_d = min(W_d / T_d, n_d), n_d = ceil(L_d / T_d);
 *   - a latent axis that is not a multiple of the tile is padded at its high
 *     end to whole tiles; padding tokens are neither keys nor queries (the
 *     pages describe divisible latents only);
 *   - window start s_d = clamp(q_d - floor(e_d / 2), 0, n_d - e_d): the window
 *     is shifted to stay inside the volume (this is the reading that gives the
 *     91% sparsity the atlas.scime.ai summary reports for w = (18,24,24));
 *   - tile-major token order: tiles in raster order over the tile grid, tokens
 *     inside a tile in raster order over (t, h, w) offsets, w fastest;
 *   - LSE = m + ln(sum exp(s - m)) in natural-log, scaled-score units.
 *
 * Conventions for every call:
 *   - All tensors are row-major [B, heads, N, d], owned by the caller,
 *     device-resident, contiguous, 16-byte aligned (fp32 LSE rows: 4-byte).
 *     Raster-order tensors hold the latent's N = L_t * L_h * L_w tokens;
 *     tile-major tensors hold whole tiles, N_tiles = n_t n_h n_w * tile volume
 *     rows (equal to N when every axis is a multiple of the tile).  Tile-major
 *     inputs have zero padding rows, as sta_tile_reorder writes them; in
 *     tile-major outputs (o, lse, dq, dk, dv) the padding rows are unspecified:
 *     a 128-row block of padding rows only is not computed at all.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Device work
 *     is enqueued asynchronously on it; nothing here synchronises except
 *     sta_plan, sta_plan_destroy and sta_last_device_status.
 *   - Calls return a status and never throw, abort or print.  Argument errors
 *     are detected before any launch.  Faults and device-side timeouts of
 *     launched work are reported by sta_last_device_status.
 *   - Empty problems: a plan may have batch 0, and the permutations take
 *     outer 0 and sta_window_stats slices 0.  Such calls check their other
 *     arguments, launch nothing and return STA_OK; their tensor pointers are
 *     not read and may be NULL (an empty PyTorch tensor has a null data
 *     pointer).
 */
#ifndef STA_H_
#define STA_H_

#include <stdint.h>

#if defined(__GNUC__)
#define STA_API __attribute__((visibility("default")))
#else
#define STA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    STA_OK = 0,
    STA_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer, geometry mismatch */
    STA_ERR_UNSUPPORTED = 2, /* valid request this build does not implement (e.g. head_dim) */
    STA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
    STA_ERR_TIMEOUT = 4,     /* a device-side wait ran past its time limit */
    STA_ERR_OOM = 5,         /* device or host allocation failed */
    STA_ERR_BOUNDS = 6       /* a plan index failed a device-side check (debug build, libsta_debug.so) */
} sta_status;

/* Latent and tile extents in tokens, (t, h, w) order. */
typedef struct {
    int32_t lat_t, lat_h, lat_w;
    int32_t tile_t, tile_h, tile_w;
} sta_geom;

/* Opaque plan: the per-head key-tile lists and the work list of one
 * (geometry, batch, heads, windows) problem.  Library-owned. */
typedef struct sta_plan_s* sta_plan_t;

/* Build a plan and upload it to the current CUDA device.
 *   g          : geometry; L_d >= 1 and T_d >= 1 (an axis that is not a
 *                multiple of its tile is padded to whole tiles).
 *   batch      : B >= 0 (0: an empty plan, see the conventions);  heads: H >= 1
 *   window_thw : host array [heads][3], window per head in tokens; every entry
 *                a positive multiple of the tile extent on its axis (windows
 *                wider than the volume are clamped to it)
 *   stream     : stream for the upload (the call waits for it to finish)
 *   out        : receives the plan handle
 * The plan holds, per distinct window, the ascending list of key-tile ids of
 * every query tile (CSR) and its transpose, the forward work list of
 * (b, h, query row block) items in descending order of list length, the
 * backward's one-block work lists (ordered for a persistent grid of one CTA
 * per SM), the raster origin of every tile, and for padded latents the real-key
 * mask of every 128-key chunk.  The work lists hold only row blocks with at
 * least one real token.  Allocates device memory; free it with
 * sta_plan_destroy.  Errors: INVALID_ARG, UNSUPPORTED (tile volume not a
 * multiple of 128 tokens, or more than 2^31 - 1 tile-major rows), OOM, CUDA.
 *
 * Sharing a plan: the forward and backward kernels hand out work items at run
 * time through a counter, which each launch takes from a pool of 256 in the
 * plan (in turn) and zeroes on its own stream first.  Calls on one stream may
 * share a plan without limit; calls running at the same time on different
 * streams may share it while at most 256 of them are in flight at once.  A
 * CUDA graph records the counter it was captured with: one captured graph
 * must not be replayed on two streams at the same time (capture it once per
 * stream, or use one plan per stream). */
STA_API sta_status sta_plan(const sta_geom* g, int32_t batch, int32_t heads,
                    const int32_t* window_thw, void* stream, sta_plan_t* out);

/* Same plan, host side only (no device memory, no CUDA call): for inspection
 * with sta_plan_query / sta_plan_stats on machines without a GPU.  A host-only
 * plan is rejected by sta_forward with INVALID_ARG. */
STA_API sta_status sta_plan_host(const sta_geom* g, int32_t batch, int32_t heads,
                         const int32_t* window_thw, sta_plan_t* out);

/* Release a plan and its device memory (synchronises the device first).
 * NULL is accepted.  The handle must not be in use by queued work. */
STA_API sta_status sta_plan_destroy(sta_plan_t p);

/* Key-tile list of query tile `q_tile` (raster tile id) for head `head`:
 * writes min(count, cap) ascending tile ids to kv_ids (host) and the full
 * length to *count.  INVALID_ARG on a bad head / tile / pointer. */
STA_API sta_status sta_plan_query(sta_plan_t p, int32_t head, int32_t q_tile,
                          int32_t* kv_ids, int32_t cap, int32_t* count);

/* Transposed list of key tile `k_tile` for head `head`: the query tiles whose
 * window holds it, ascending.  Writes min(count, cap) ids to q_ids (host) and
 * the full length to *count.  The backward's dK / dV kernel walks these lists.
 * INVALID_ARG on a bad head / tile / pointer. */
STA_API sta_status sta_plan_key_query(sta_plan_t p, int32_t head, int32_t k_tile,
                                      int32_t* q_ids, int32_t cap, int32_t* count);

/* Plan totals: computed (query tile, key tile) pairs over all batches and
 * heads, and number of work items.  Either pointer may be NULL. */
STA_API sta_status sta_plan_stats(sta_plan_t p, int64_t* computed_tile_pairs, int64_t* work_items);

/* Copy the forward's work list to host memory, four int32 per item:
 * (b * heads + h, 128-row query block, -1, window id), in the order the
 * kernel hands the items out (longest key lists first).  Row block r covers
 * tile-major rows [128 r, 128 r + 128) of its head; every block holding a real
 * token appears once, blocks of padding rows only never.  Writes min(count,
 * cap) items and the full count to *count.  For tests/inspection.  Each
 * block's 128-key chunks are split between two softmax warpgroups. */
STA_API sta_status sta_plan_work_items(sta_plan_t p, int32_t* items4, int64_t cap, int64_t* count);

/* Copy one of the backward's work lists to host memory, four int32 per item:
 * (b * heads + h, 128-row block, -1, window id); which = 0: the dQ kernel's
 * query blocks, 1: the dK / dV kernel's key blocks.  Each lists every block
 * of every (b, h) that holds a real token once, ordered for a persistent grid
 * of one CTA per SM.
 * Writes min(count, cap) items and the full count.  For tests/inspection. */
STA_API sta_status sta_plan_backward_items(sta_plan_t p, int32_t which, int32_t* items4, int64_t cap,
                                           int64_t* count);

/* Raster -> tile-major token permutation.
 *   src       : device, [outer, N, row_bytes] bytes (raster)
 *   dst       : device, [outer, N_tiles, row_bytes] bytes (tile-major; padding
 *               rows written as zeros), not overlapping src
 *   outer     : B * heads (any count >= 0)
 *   row_bytes : bytes of one token row (d * element size; 4 for a fp32 LSE
 *               row); rows move intact, bit-exact
 * dst[o, tile_major(i)] = src[o, i] for every raster token i. */
STA_API sta_status sta_tile_reorder(const void* src, void* dst, int64_t outer,
                            int32_t row_bytes, const sta_geom* g, void* stream);

/* Inverse permutation: dst[o, i] = src[o, tile_major(i)]; src is tile-major
 * [outer, N_tiles, row_bytes] (its padding rows are not read), dst raster
 * [outer, N, row_bytes]. */
STA_API sta_status sta_tile_unreorder(const void* src, void* dst, int64_t outer,
                              int32_t row_bytes, const sta_geom* g, void* stream);

/* STA forward on tile-major tensors.
 *   q, k, v : device bf16 [B, heads, N_tiles, d], tile-major token order
 *   o       : device bf16 [B, heads, N_tiles, d], tile-major (written)
 *   lse     : device fp32 [B, heads, N_tiles], tile-major (written): natural-log
 *             log-sum-exp of the scaled scores of each query row
 *   head_dim: d, 64 or 128 (else UNSUPPORTED)
 *   softmax_scale: multiplies q . k before the softmax (e.g. 1/sqrt(d));
 *             finite and > 0, else INVALID_ARG
 * For every (b, h) and query tile q, over the key tiles of the plan's list:
 * S = scale * Q_q K^T, exact online softmax with running max and sum in fp32,
 * O = softmax(S) V rounded to bf16.  Allocates nothing; enqueues a 4-byte
 * memset (the plan's work counter, see sta_plan) and one kernel on `stream`.
 * The plan must come from sta_plan on the current device. */
STA_API sta_status sta_forward(sta_plan_t p, const void* q, const void* k, const void* v,
                       void* o, float* lse, int32_t head_dim, float softmax_scale,
                       void* stream);

/* STA forward on raster-order tensors, the token permutation fused into the
 * kernel's loads and stores (no reorder / unreorder passes).
 *   q, k, v : device bf16 [B, heads, N, d] in raster token order (t, h, w)
 *   o       : device bf16 [B, heads, N, d], raster order (written)
 *   lse     : device fp32 [B, heads, N], raster order (written)
 * Same arithmetic and results as sta_tile_reorder -> sta_forward ->
 * sta_tile_unreorder, bit for bit.  Each 128-row block of a tile must be a box
 * of whole (h, w) slices (tile_h * tile_w divides 128) or a run of whole w rows
 * of one slice (128 divides tile_h * tile_w and tile_w divides 128), else
 * UNSUPPORTED; 6x8x8 tiles are two slices per block.  Other rules as sta_forward. */
STA_API sta_status sta_forward_raster(sta_plan_t p, const void* q, const void* k, const void* v,
                                      void* o, float* lse, int32_t head_dim, float softmax_scale,
                                      void* stream);

/* STA backward on tile-major tensors: gradients of the forward's output with
 * respect to q, k and v.  The pages use STA in fine-tuning ("Fast Video
 * Generation with Sliding Tile Attention": podcast transcript at
 * hotaipapers.com, fine-tuning segment; dianyo.github.io ICML-2025 post, STA
 * section, last paragraph), which needs these gradients; they give no backward
 * kernel.  This call computes the exact gradient of the forward's function with
 * the tile window held fixed (the mask has no gradient):
 *   P_ij = exp(scale q_i . k_j - lse_i) over the plan's key tiles of i's tile,
 *   D_i = dout_i . o_i,  dS_ij = P_ij (dout_i . v_j - D_i),
 *   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,
 *   dv_j = sum_i P_ij dout_i.
 *   q, k, v, o : device bf16 [B, heads, N_tiles, d], tile-major; o and lse as
 *                written by sta_forward for the same q, k, v and plan
 *   dout       : device bf16 [B, heads, N_tiles, d], tile-major: gradient w.r.t. o
 *   lse        : device fp32 [B, heads, N_tiles], tile-major
 *   dq, dk, dv : device bf16 [B, heads, N_tiles, d], tile-major (written; distinct
 *                from every input)
 *   workspace  : device fp32, 2 * B * heads * N floats, 16-byte aligned,
 *                caller-owned; on return plane 0 holds -D_i and plane 1
 *                -lse_i * log2(e), tile-major (N = tiles x tile volume, the
 *                tile-major row count)
 *   head_dim, softmax_scale: as sta_forward
 * P and dS enter the tensor-core products as bf16 with fp32 accumulation;
 * dq, dk, dv are rounded to bf16.  No atomics: results are deterministic.
 * Allocates nothing; enqueues three kernels (and two 4-byte memsets of work
 * counters) on `stream`.  Errors: INVALID_ARG
 * (null or misaligned pointer, bad scale, plan not on the current device),
 * UNSUPPORTED (head_dim), CUDA. */
STA_API sta_status sta_backward(sta_plan_t p, const void* q, const void* k, const void* v,
                                const void* o, const void* dout, const float* lse, void* dq,
                                void* dk, void* dv, float* workspace, int32_t head_dim,
                                float softmax_scale, void* stream);

/* STA backward on raster-order tensors, the token permutation fused into the
 * kernels' loads and stores: q, k, v, o, dout, dq, dk, dv are [B, heads, N, d]
 * and lse [B, heads, N] in raster order (N = L_t * L_h * L_w), as written by
 * sta_forward_raster; the workspace is as for sta_backward (tile-major, whole
 * tiles: 2 * B * heads * tiles * tile volume floats).  Same arithmetic and
 * results as permuting to tile-major, sta_backward, and permuting back, bit for
 * bit.  Tile shapes as sta_forward_raster (else UNSUPPORTED). */
STA_API sta_status sta_backward_raster(sta_plan_t p, const void* q, const void* k, const void* v,
                                       const void* o, const void* dout, const float* lse, void* dq,
                                       void* dk, void* dv, float* workspace, int32_t head_dim,
                                       float softmax_scale, void* stream);

/* Per-(b, h) statistics of a candidate window against the full window, for
 * choosing a window per head by profiling ("Fast Video Generation with Sliding
 * Tile Attention": podcast transcript at hotaipapers.com, segments on the 3D
 * locality pattern and on head specialisation; dianyo.github.io ICML-2025
 * post, STA section, "Observation & Proposed Method").
 *   lse_w, lse_full : device fp32 [slices, tokens]: the forward's LSE with the
 *                     candidate window and with a window covering the volume
 *   o_w, o_full     : device bf16 [slices, tokens, head_dim], the matching
 *                     outputs, 16-byte aligned; any token order, the same in
 *                     all four tensors
 *   recall          : device fp64 [slices] (written): mean over rows of
 *                     exp(lse_w - lse_full), the attention recall, i.e. the
 *                     share of each row's full-attention softmax mass that the
 *                     window keeps
 *   mse             : device fp64 [slices] (written): mean of (o_w - o_full)^2
 *                     over rows and channels (the mask-search loss, read here
 *                     as the output's mean squared error against full attention)
 * 0 <= slices (B * heads) <= 2^28, tokens >= 1, head_dim a positive multiple
 * of 8, else INVALID_ARG.  One kernel (a cluster of 8 CTAs per slice),
 * deterministic; allocates nothing. */
STA_API sta_status sta_window_stats(const float* lse_w, const float* lse_full, const void* o_w,
                                    const void* o_full, int64_t slices, int64_t tokens, int32_t head_dim,
                                    double* recall, double* mse, void* stream);

/* Pick a window per head from profiled candidates (host only, no CUDA call).
 * The pages profile a predefined list of windows per head and keep, per head,
 * one that preserves quality ("Fast Video Generation with Sliding Tile
 * Attention": podcast transcript at hotaipapers.com, segment on head
 * specialisation; dianyo.github.io ICML-2025 post, STA section); they give no
 * selection rule.  This library's reading: each head takes the candidate with
 * the fewest attended tiles (ties: the one listed first) whose recall and
 * output error meet every given bound; the window covering the volume when
 * none does.
 *   g         : geometry (tile counts per candidate: prod_d min(W_d / T_d, n_d))
 *   heads     : H >= 1;  n_cand >= 0 candidates
 *   cand_thw  : host int32 [n_cand][3], windows in tokens (positive multiples
 *               of the tile, as for sta_plan)
 *   recall    : host fp64 [n_cand][heads], e.g. sta_window_stats' recall
 *               averaged over the batch
 *   mse       : host fp64 [n_cand][heads], the same for the output error
 *   max_mse   : upper bound on mse, or a negative value for none
 *   min_recall: lower bound on recall, or a negative value for none
 *   out_thw   : host int32 [heads][3] (written), window per head in tokens
 * INVALID_ARG on a bad geometry, count, candidate or null pointer. */
STA_API sta_status sta_window_pick(const sta_geom* g, int32_t heads, int32_t n_cand, const int32_t* cand_thw,
                                   const double* recall, const double* mse, double max_mse, double min_recall,
                                   int32_t* out_thw);

/* Forward pipeline from host memory (no counterpart on the pages: a runtime
 * piece for callers whose Q, K, V live in host memory).  At the pages' 720p
 * size the PCIe copies of one call take longer than its attention, so the
 * pipeline overlaps them across calls: a ring of `depth` device buffer sets
 * and three streams, the copy-in of call i+1, the forward (sta_forward_raster)
 * of call i and the copy-out of call i-1 running at once.
 *
 * sta_pipe_create: plan from sta_plan on the current device (its tile shape
 *   must suit sta_forward_raster, else UNSUPPORTED; batch 0 is INVALID_ARG:
 *   nothing to pipeline); head_dim 64 or 128;
 *   softmax_scale finite and > 0; 1 <= depth <= 8.  Allocates depth x (four
 *   [B, heads, N, d] bf16 tensors + one fp32 LSE) of device memory and three
 *   streams; OOM / CUDA on failure.  The plan must outlive the pipeline.
 * sta_pipe_submit: enqueue one call on raster-order host tensors: q, k, v
 *   read and o, lse written, shapes as sta_forward_raster.  Returns at once.
 *   The host buffers should be pinned (cudaHostAlloc, or pin_memory in
 *   PyTorch) or the copies do not overlap; q, k, v must stay unchanged and
 *   o, lse unread until sta_pipe_wait.  INVALID_ARG on null pointers or a
 *   different current device.
 * sta_pipe_wait: block until all submitted calls are done; returns the first
 *   CUDA error or the plan's device status (as sta_last_device_status).
 * sta_pipe_destroy: wait, then free everything (NULL accepted).
 * A pipeline holds no lock: calls on one pipeline must come from one host
 * thread at a time (separate pipelines may be driven from separate threads). */
typedef struct sta_pipe_s* sta_pipe_t;
STA_API sta_status sta_pipe_create(sta_plan_t p, int32_t head_dim, float softmax_scale, int32_t depth,
                                   sta_pipe_t* out);
STA_API sta_status sta_pipe_submit(sta_pipe_t pipe, const void* q_host, const void* k_host,
                                   const void* v_host, void* o_host, float* lse_host);
STA_API sta_status sta_pipe_wait(sta_pipe_t pipe);
STA_API sta_status sta_pipe_destroy(sta_pipe_t pipe);

/* STA forward that allocates nothing (this call has no counterpart in the
 * paper; it exists for deployment).
 *
 * sta_plan puts the plan in device memory it allocates with cudaMalloc.  Some
 * callers cannot do that: a process whose device memory belongs to another
 * allocator or pool that forbids outside cudaMalloc calls; a service that
 * reserves all its memory at start-up and allows no allocation, and none of
 * the device synchronisation cudaMalloc may cause, while it serves; a plugin
 * host that only hands a library the buffers it is meant to touch.  This call
 * takes the geometry, batch, heads and per-head windows of sta_plan and the
 * tensors of sta_forward (same layouts and rules: tile-major q, k, v, o, lse),
 * and keeps the plan in a fixed scratch array compiled into the library: 4 MiB
 * of device memory on every GPU that loads the library, held until the process
 * exits.  It computes the same results as sta_plan + sta_forward.
 *
 * Limits: every latent axis a multiple of its tile (padded latents need
 * sta_plan + sta_forward), heads <= 1024, and the plan must fit the scratch:
 *   256 + 16 * B * heads * tiles * (tile volume / 128)
 *       + 4 * (n_windows * (tiles + 1) + sum over distinct windows of
 *              tiles * window_tiles) <= 4 MiB
 * (the 720p and 42x64x112 workloads of this library use 0.36 and 2.1 MiB).
 * Larger problems, heads > 1024 or a padded latent return STA_ERR_UNSUPPORTED
 * before any work.  batch 0 returns STA_OK at once (pointers unread).
 *
 * Behaviour: the first call on a device looks up the scratch's device address
 * (cudaGetSymbolAddress) and caches it.  Each call enqueues two kernels on
 * `stream`: one writes the plan
 * into the scratch (from the windows, which it receives as kernel arguments;
 * nothing is copied from host memory) and clears the status word and work
 * counter kept there, the second is the forward.  Every call shares the one
 * scratch array: calls whose work overlaps on the GPU (different streams, or
 * threads enqueueing concurrently) race and must be serialised by the caller,
 * e.g. by using one stream.  A device-side timeout ends the kernel cleanly but
 * is not reported by this call (use sta_forward with a plan and
 * sta_last_device_status to observe it).  Errors: as sta_plan and
 * sta_forward, UNSUPPORTED beyond the limits, CUDA on a failed launch. */
STA_API sta_status sta_forward_noalloc(const sta_geom* g, int32_t batch, int32_t heads,
                                       const int32_t* window_thw, const void* q, const void* k,
                                       const void* v, void* o, float* lse, int32_t head_dim,
                                       float softmax_scale, void* stream);

/* Synchronise `stream`, then report (and clear) the first asynchronous error
 * of work enqueued with this plan: CUDA for a launch or execution fault,
 * BOUNDS when a kernel of the debug build found a plan index out of range
 * (it then stops without using it), TIMEOUT when a device-side wait gave up. */
STA_API sta_status sta_last_device_status(sta_plan_t p, void* stream);

/* Check every index of a plan's host copy against the plan's extents: CSR
 * offsets non-decreasing and inside the id arrays, key and query tile ids
 * inside the tile grid, work items inside (b, h), row block and window
 * ranges, each transposed list the transpose of the forward lists, tile
 * origins inside the padded latent.  sta_plan and sta_plan_host run it on
 * every plan they build.  Returns INVALID_ARG (text in
 * sta_last_error_detail) for the first violation, OK otherwise. */
STA_API sta_status sta_plan_validate(sta_plan_t p);

/* Debug only: overwrite one plan entry, on the host copy and, for a plan on
 * a device, in its device array (synchronous copy), to test sta_plan_validate
 * and the device-side checks of the debug build.  which = 0: forward key-tile
 * id csr_ids[index]; 1: field index % 4 of forward work item index / 4 (bh,
 * block, unused, window); 2: forward CSR offset csr_off[index]; 3: transposed
 * query-tile id tcsr_ids[index].  INVALID_ARG for an index outside the array.
 * A plan changed this way must only run on the debug build. */
STA_API sta_status sta_debug_plan_poke(sta_plan_t p, int32_t which, int64_t index, int32_t value);

/* Name and text of the last CUDA error met by a libsta call in the calling
 * thread (e.g. "cudaErrorLaunchOutOfResources: ..."), or "no error".  The
 * string stays valid until the thread's next failing call. */
STA_API const char* sta_last_error_detail(void);

/* Static string naming a status code. */
STA_API const char* sta_status_string(sta_status s);

/* Debug only: makes a device-side wait of the next forward calls
 * (sta_forward, sta_forward_raster) run out on a barrier nothing arrives at,
 * so the timeout path can be tested without a fault.  Every wait of those
 * calls then has the time limit `limit_ms` (1..10000).
 *   mode 0: off (the default).
 *   mode 1: the load warp's first wait runs out: the kernel issues no copy or
 *           MMA and exits.
 *   mode 2: in every CTA that takes a second work item, the S-issuing
 *           thread's wait at the start of that item runs out after the first
 *           item has been computed and the second item's query block and K/V
 *           chunks have been issued; the kernel waits (bounded) for those
 *           copies and its MMAs, frees TMEM and exits.
 * In both cases the outputs are left partly written and
 * sta_last_device_status returns TIMEOUT.  Any other mode: INVALID_ARG. */
STA_API sta_status sta_debug_inject_timeout(int32_t mode, int32_t limit_ms);

#ifdef __cplusplus
}
#endif

#endif /* STA_H_ */
