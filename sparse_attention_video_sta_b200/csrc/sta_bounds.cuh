// sta_bounds.cuh -- device-side checks of plan indices in the debug build.
//
// Built with STA_DEBUG_BOUNDS defined (libsta_debug.so), the forward and
// backward kernels check every work item they take and the key-tile list it
// names before any load or product uses them: the item index, its (b, h),
// row block and window id, the list's CSR offsets and every tile id in it.
// The TMA row coordinates derived from a checked item are inside the tensors
// by construction, and are checked too.  A failed check sets kDevBounds in
// the status word, raises the CTA's abort flag and hands the other roles no
// more items, so the kernel exits cleanly; sta_last_device_status then
// returns STA_ERR_BOUNDS.  The regular build compiles the checks out.
#pragma once

#include <stdint.h>

#include "sta_internal.h"

namespace sta {

#ifdef STA_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
#else
constexpr bool kDebugBounds = false;
#endif

// Checks work item u (of n_items) and its key-tile list (CSR off / ids) against
// the plan's extents; records kDevBounds and returns false on any violation.
__device__ __forceinline__ bool item_in_bounds(const WorkItem* items, int32_t n_items, int32_t u, const int32_t* off,
                                               const int32_t* ids, const PlanBounds& b, uint32_t* status) {
    bool ok = u >= 0 && u < n_items;
    if (ok) {
        const WorkItem w = items[u];
        ok = w.bh >= 0 && w.bh < b.n_bh && w.qa >= 0 && w.qa < b.tiles * b.sub_per_tile && w.win >= 0 &&
             w.win < b.n_win;
        if (ok) {
            const int32_t tile = w.qa / b.sub_per_tile;
            const int32_t* o = off + int64_t(w.win) * (b.tiles + 1);
            const int32_t lo = o[tile], hi = o[tile + 1];
            ok = lo >= 0 && lo <= hi && hi <= b.n_ids;
            for (int32_t i = lo; ok && i < hi; ++i) {
                const int32_t t = ids[i];
                ok = t >= 0 && t < b.tiles;
            }
            // TMA rows of the item's own block and of the last row of any tile
            const int64_t rows = int64_t(b.n_bh) * b.tiles * b.tile_tokens;
            ok = ok && int64_t(w.bh) * b.tiles * b.tile_tokens + int64_t(b.tiles) * b.tile_tokens <= rows;
        }
    }
    if (!ok) atomicOr(status, kDevBounds);
    return ok;
}

}  // namespace sta
