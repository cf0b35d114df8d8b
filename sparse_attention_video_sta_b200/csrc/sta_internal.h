// sta_internal.h -- internal types shared by the libsta translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <vector>

#include "sta.h"

namespace sta {

// Work counters per plan (see sta_plan_s::d_counters).
constexpr int kCounterPool = 256;

// Query rows per MMA slot (tcgen05 M for cta_group::1) and keys per K/V chunk.
constexpr int kSubRows = 128;
constexpr int kChunkKeys = 128;

// Device status bits written by kernels (OR-ed).
constexpr uint32_t kDevTimeout = 1u;
constexpr uint32_t kDevBounds = 2u;  // a plan index failed its check (debug build)

// Extents a plan's device arrays must respect (checked by the debug build).
struct PlanBounds {
    int32_t n_bh;          // batch * heads
    int32_t tiles;         // tiles per head
    int32_t sub_per_tile;  // 128-row blocks per tile
    int32_t tile_tokens;
    int32_t n_win;         // distinct windows
    int32_t n_ids;         // entries of the CSR id array walked
};

// One work item of the forward and backward kernels: one 128-row block of
// one (b, h) (a query block, or a key block for the dK / dV kernel).
struct WorkItem {
    int32_t bh;   // b * heads + h
    int32_t qa;   // row block within the head: tile * sub_per_tile + sub
    int32_t qb;   // unused, -1
    int32_t win;  // distinct-window id of head h
};
static_assert(sizeof(WorkItem) == 16, "WorkItem is loaded as one int4");

struct PlanHost {
    sta_geom g;
    int32_t batch = 0, heads = 0;
    int32_t n_tiles[3] = {0, 0, 0};
    int32_t tiles_per_head = 0;
    int32_t tile_tokens = 0;
    int32_t sub_per_tile = 0;                // tile_tokens / kSubRows
    std::vector<int32_t> head_win;           // [heads] distinct-window id
    std::vector<int32_t> win_ext;            // [n_win][3] clamped extents in tiles
    std::vector<int32_t> csr_off;            // [n_win][tiles_per_head + 1], global offsets
    std::vector<int32_t> csr_ids;            // key-tile ids, ascending per list
    std::vector<WorkItem> f1_items;          // forward work list of one-block items, longest lists first
    // Backward: for each key tile the query tiles whose window holds it
    // (the forward lists transposed), and one-block work lists for the dQ
    // kernel (qa = query block) and the dK/dV kernel (qa = key block).
    std::vector<int32_t> tcsr_off;           // [n_win][tiles_per_head + 1], global offsets
    std::vector<int32_t> tcsr_ids;           // query-tile ids, ascending per list
    std::vector<WorkItem> bq_items;
    std::vector<WorkItem> bkv_items;
    std::vector<int32_t> tile_origin;        // [tiles_per_head][4]: raster (w, h, t) origin of each tile, 0
    bool padded = false;                     // some axis is not a multiple of the tile
    std::vector<uint32_t> key_mask;          // padded only: [tiles][sub_per_tile][4] real-key bits per chunk
    int64_t computed_pairs = 0;              // B * sum_h sum_q |list|
};

}  // namespace sta

struct sta_plan_s {
    sta::PlanHost h;
    bool on_device = false;
    int device = -1;
    int32_t* d_off = nullptr;
    int32_t* d_ids = nullptr;
    sta::WorkItem* d_f1_items = nullptr;
    uint32_t* d_status = nullptr;
    int32_t* d_origin = nullptr;  // device copy of tile_origin (16-byte rows)
    uint32_t* d_kmask = nullptr;  // device copy of key_mask (padded latents only)
    // Work counters of the forward's run-time item hand-out: each launch takes
    // the next of a pool (zeroed on its stream first), so calls that share the
    // plan on different streams use different counters (up to the pool size
    // in flight at once).
    int32_t* d_counters = nullptr;
    mutable std::atomic<uint32_t> launch_seq{0};
    int32_t* d_toff = nullptr;
    int32_t* d_tids = nullptr;
    sta::WorkItem* d_bq_items = nullptr;
    sta::WorkItem* d_bkv_items = nullptr;
};

namespace sta {

// Shape of one 128-row block of a tile as a box of whole (t, h) slices, for
// loading Q, K, V straight from raster layout: box_t slices of tile_h rows, or
// box_h rows of one slice (blocks_per_slice blocks per slice).  ok = false when
// a block is not such a box.
struct RasterBox {
    int32_t box_t, box_h, blocks_per_slice;
    bool ok;
};
RasterBox raster_box(const sta_geom& g);

// Forward kernel launch (sta_forward.cu): tile-major tensors, or raster tensors
// with the permutation done by the kernel's loads and stores (`raster`).
// Returns a CUDA error code.
cudaError_t launch_forward(const sta_plan_s* p, const void* q, const void* k, const void* v,
                           void* o, float* lse, int head_dim, float softmax_scale,
                           cudaStream_t stream, int inject_timeout, uint64_t timeout_ns, bool raster);

// Device-side view of a plan whose arrays live in memory the caller provides
// (used by the no-allocation entry point, sta_noalloc.cu).
struct RawPlanView {
    int32_t batch, heads, tiles_per_head, tile_tokens, sub_per_tile;
    const WorkItem* items;  // one-block items
    int32_t n_items;
    int32_t* item_counter;  // zero before the launch (the run-time item hand-out)
    const int32_t* off;
    const int32_t* ids;
    uint32_t* status;
    uint64_t timeout_ns;
    int32_t n_win, n_ids;  // CSR extents (checked by the debug build)
};

// Forward launch from a RawPlanView (sta_forward.cu).  Returns a CUDA error code.
cudaError_t launch_forward_raw(const RawPlanView& pv, const void* q, const void* k, const void* v,
                               void* o, float* lse, int head_dim, float softmax_scale,
                               cudaStream_t stream);

// Backward launches (sta_backward.cu): the D / log2-LSE pass, then the dQ and
// dK / dV kernels, on tile-major tensors or (`raster`) on raster tensors with
// the permutation fused.  Returns a CUDA error code.
cudaError_t launch_backward(const sta_plan_s* p, const void* q, const void* k, const void* v,
                            const void* o, const void* dout, const float* lse, void* dq, void* dk,
                            void* dv, float* workspace, int head_dim, float softmax_scale,
                            cudaStream_t stream, uint64_t timeout_ns, bool raster);

// Per-slice recall / loss reduction for the window search (sta_search.cu).
cudaError_t launch_window_stats(const float* lse_w, const float* lse_full, const void* o_w, const void* o_full,
                                int64_t slices, int64_t tokens, int head_dim, double* recall, double* mse,
                                cudaStream_t stream);

// Permutation launch (sta_permute.cu).  inverse = false: raster -> tile-major.
cudaError_t launch_permute(const void* src, void* dst, int64_t outer, int32_t row_bytes,
                           const sta_geom& g, bool inverse, cudaStream_t stream);

}  // namespace sta
