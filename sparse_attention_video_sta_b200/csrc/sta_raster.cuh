// sta_raster.cuh -- reading and writing raster-order tensors straight from the
// STA kernels (the tile permutation fused into their loads and stores).
//
// A tile is a contiguous spatio-temporal cube of tokens (podcast transcript at
// hotaipapers.com, segment on tiles); the kernels work on 128-row blocks of a
// tile in tile-major row order (tile's own (t, h, w) offsets in raster order).
// When a block is a box of whole (h, w) slices of its tile, or whole w rows of
// one slice, a 5D TMA box (64 elements of d, T_w, box_h, box_t, 1) over the
// raster tensor [B*H, L_t, L_h, L_w, d] lands in shared memory in exactly that
// row order, with the 128-byte swizzle the tcgen05 descriptors expect.  Boxes
// at a padded edge read past the latent and get zeros.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "sta_internal.h"
#include "sta_ptx.cuh"

namespace sta {

struct RasterGeom {
    int32_t lat_t, lat_h, lat_w;
    int32_t tile_t, tile_h, tile_w;
    int32_t n_h, n_w;                        // tiles along h and w
    int32_t box_t, box_h, blocks_per_slice;  // one 128-row block as a TMA box
    int32_t sub_per_tile;
    int32_t tokens_raster;    // raster rows per (b, h): the latent's tokens
    const int4* tile_origin;  // [tiles]: raster (w, h, t) origin of each tile
};

// Raster geometry of a device plan (its tile origin table included).
inline RasterGeom raster_geom(const sta_plan_s* pl) {
    const PlanHost& P = pl->h;
    const RasterBox rb = raster_box(P.g);
    RasterGeom g;
    g.lat_t = P.g.lat_t;
    g.lat_h = P.g.lat_h;
    g.lat_w = P.g.lat_w;
    g.tile_t = P.g.tile_t;
    g.tile_h = P.g.tile_h;
    g.tile_w = P.g.tile_w;
    g.n_h = P.n_tiles[1];
    g.n_w = P.n_tiles[2];
    g.box_t = rb.box_t;
    g.box_h = rb.box_h;
    g.blocks_per_slice = rb.blocks_per_slice;
    g.sub_per_tile = P.sub_per_tile;
    g.tokens_raster = P.g.lat_t * P.g.lat_h * P.g.lat_w;
    g.tile_origin = reinterpret_cast<const int4*>(pl->d_origin);
    return g;
}

// 5D map over a raster [BH, L_t, L_h, L_w, d] bf16 tensor whose box is one
// 128-row block of a tile: 64 elements x tile_w x box_h x box_t x 1, 128-byte
// swizzle.
inline cudaError_t make_raster_map(PFN_cuTensorMapEncodeTiled_v12000 fn, CUtensorMap* m, const void* ptr,
                                   const sta_geom& g, int64_t bh, int d, int box_t, int box_h) {
    const cuuint64_t row = cuuint64_t(d) * 2;
    cuuint64_t dims[5] = {cuuint64_t(d), cuuint64_t(g.lat_w), cuuint64_t(g.lat_h), cuuint64_t(g.lat_t),
                          cuuint64_t(bh)};
    cuuint64_t strides[4] = {row, row * g.lat_w, row * g.lat_w * g.lat_h, row * g.lat_w * g.lat_h * g.lat_t};
    cuuint32_t box[5] = {64, cuuint32_t(g.tile_w), cuuint32_t(box_h), cuuint32_t(box_t), 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Load 128-row block `sub` of the tile whose raster (w, h, t) origin is `org`
// (from the plan's table) of head bh from a raster tensor: the origin of the
// block's box inside the tile, `col_blocks` boxes of 64 columns, `box_bytes`
// apart.
__device__ __forceinline__ void raster_load_at(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                               const RasterGeom& g, int32_t bh, int4 org, int32_t sub,
                                               int col_blocks, int box_bytes) {
    int32_t t0 = org.z, h0 = org.y;
    if (g.blocks_per_slice == 1) {
        t0 += sub * g.box_t;
    } else {
        t0 += sub / g.blocks_per_slice;
        h0 += (sub % g.blocks_per_slice) * g.box_h;
    }
    for (int cb = 0; cb < col_blocks; ++cb) ptx::tma_load_5d(dst + cb * box_bytes, m, bar, cb * 64, org.x, h0, t0, bh);
}

// The same for block `sub` of tile `tile` (origin looked up here).
__device__ __forceinline__ void raster_load(uint32_t dst, const CUtensorMap* m, uint32_t bar, const RasterGeom& g,
                                            int32_t bh, int32_t tile, int32_t sub, int col_blocks, int box_bytes) {
    raster_load_at(dst, m, bar, g, bh, __ldg(g.tile_origin + tile), sub, col_blocks, box_bytes);
}

// Raster row of row `r` of 128-row block `blk` of head bh; -1 for a padding
// row (a token past the latent; only when kPadded).
template <bool kPadded>
__device__ __forceinline__ int64_t raster_row(const RasterGeom& g, int32_t bh, int32_t blk, int32_t r) {
    const int32_t tile = blk / g.sub_per_tile, sub = blk - tile * g.sub_per_tile;
    const int32_t it = tile / (g.n_h * g.n_w), ih = (tile / g.n_w) % g.n_h, iw = tile % g.n_w;
    const int32_t l = sub * kSubRows + r;  // tile-local row, raster over the tile's (t, h, w)
    const int32_t lw = l % g.tile_w, lh = (l / g.tile_w) % g.tile_h, lt = l / (g.tile_w * g.tile_h);
    const int32_t t = it * g.tile_t + lt, h = ih * g.tile_h + lh, w = iw * g.tile_w + lw;
    if (kPadded && (t >= g.lat_t || h >= g.lat_h || w >= g.lat_w)) return -1;
    const int64_t token = (int64_t(t) * g.lat_h + h) * g.lat_w + w;
    return int64_t(bh) * g.tokens_raster + token;
}

}  // namespace sta
