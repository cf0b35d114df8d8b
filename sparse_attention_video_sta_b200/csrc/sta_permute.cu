// sta_permute.cu -- raster <-> tile-major token permutation.
//
// A tile is a contiguous spatio-temporal cube of tokens (podcast transcript at
// hotaipapers.com, segment on tiles): tile-major order lists tiles in raster
// order over the tile grid and the tokens of a tile in raster order over their
// (t, h, w) offsets.  Token rows move intact, so the permutation is bit-exact.
//
// One CTA moves one (outer slice, tile).  Inside a tile, the T_w tokens of one
// (t, h) offset are consecutive both in raster order and in tile-major order,
// so consecutive threads read and write consecutive addresses on both sides.
// The per-tile map from local token index to raster offset is built once per
// CTA in shared memory.  HBM-bound: 2 x tensor bytes per pass.
//
// A latent axis that is not a multiple of the tile is padded at its high end
// to whole tiles: the tile-major layout holds every tile whole, and its
// padding rows (tokens past the latent) are written as zeros by the reorder
// and skipped by the inverse.  Only tiles at the padded edge test rows.
#include <cuda_runtime.h>
#include <stdint.h>

#include "sta_internal.h"

namespace sta {
namespace {

constexpr int kPermThreads = 256;
constexpr int kMaxTableTokens = 12288;  // 48 KB of int32 in shared memory

struct PermGeom {
    int32_t lat_t, lat_h, lat_w;
    int32_t tile_t, tile_h, tile_w;
    int32_t n_h, n_w;       // tiles along h and w
    int32_t tiles;          // tiles per head
    int32_t tile_tokens;
    int64_t tokens;         // raster tokens per head
    int64_t tm_tokens;      // tile-major rows per head (tiles * tile_tokens)
};

__device__ __forceinline__ int64_t local_to_raster(const PermGeom& g, int32_t l) {
    const int32_t x = l % g.tile_w;
    const int32_t r = l / g.tile_w;
    const int32_t y = r % g.tile_h;
    const int32_t t = r / g.tile_h;
    return (int64_t(t) * g.lat_h + y) * g.lat_w + x;
}

// V = element type moved per thread; vpr = elements per token row.
// kInverse = false: raster -> tile-major.
template <typename V, bool kTable, bool kInverse>
__global__ void __launch_bounds__(kPermThreads)
permute_kernel(const V* __restrict__ src, V* __restrict__ dst, PermGeom g, int32_t vpr,
               int32_t vpr_shift, int64_t blocks) {
    extern __shared__ int32_t table[];
    if (kTable) {
        for (int32_t l = threadIdx.x; l < g.tile_tokens; l += blockDim.x)
            table[l] = int32_t(local_to_raster(g, l));
        __syncthreads();
    }
    const int64_t per_tile = int64_t(g.tile_tokens) * vpr;
    for (int64_t blk = blockIdx.x; blk < blocks; blk += gridDim.x) {
        const int64_t outer = blk / g.tiles;
        const int32_t tile = int32_t(blk - outer * g.tiles);
        const int32_t it = tile / (g.n_h * g.n_w);
        const int32_t ih = (tile / g.n_w) % g.n_h;
        const int32_t iw = tile % g.n_w;
        const int64_t origin = (int64_t(it) * g.tile_t * g.lat_h + int64_t(ih) * g.tile_h) * g.lat_w +
                               int64_t(iw) * g.tile_w;
        const int64_t r_slice = outer * g.tokens, t_slice = outer * g.tm_tokens;
        const int64_t tm_base = int64_t(tile) * g.tile_tokens;
        // valid extents of this tile (smaller than the tile only at a padded edge)
        const int32_t vt = min(g.tile_t, g.lat_t - it * g.tile_t);
        const int32_t vh = min(g.tile_h, g.lat_h - ih * g.tile_h);
        const int32_t vw = min(g.tile_w, g.lat_w - iw * g.tile_w);
        const bool edge = vt < g.tile_t || vh < g.tile_h || vw < g.tile_w;
        auto split = [&](int64_t e, int32_t& l, int32_t& c) {
            if (vpr_shift >= 0) {
                l = int32_t(e >> vpr_shift);
                c = int32_t(e & (vpr - 1));
            } else {
                l = int32_t(e / vpr);
                c = int32_t(e - int64_t(l) * vpr);
            }
        };
        if (!edge) {  // a whole tile: no per-row test
#pragma unroll 4
            for (int64_t e = threadIdx.x; e < per_tile; e += blockDim.x) {
                int32_t l, c;
                split(e, l, c);
                const int64_t tmaj = t_slice + tm_base + l;
                const int64_t raster = r_slice + origin + (kTable ? int64_t(table[l]) : local_to_raster(g, l));
                if (kInverse)
                    dst[raster * vpr + c] = src[tmaj * vpr + c];
                else
                    dst[tmaj * vpr + c] = src[raster * vpr + c];
            }
        } else {  // a tile at the padded edge
            for (int64_t e = threadIdx.x; e < per_tile; e += blockDim.x) {
                int32_t l, c;
                split(e, l, c);
                const int64_t tmaj = t_slice + tm_base + l;
                const int32_t x = l % g.tile_w, y = (l / g.tile_w) % g.tile_h, t = l / (g.tile_w * g.tile_h);
                if (t >= vt || y >= vh || x >= vw) {  // padding row: zero in tile-major, absent in raster
                    if (!kInverse) dst[tmaj * vpr + c] = V{};
                    continue;
                }
                const int64_t raster = r_slice + origin + (kTable ? int64_t(table[l]) : local_to_raster(g, l));
                if (kInverse)
                    dst[raster * vpr + c] = src[tmaj * vpr + c];
                else
                    dst[tmaj * vpr + c] = src[raster * vpr + c];
            }
        }
    }
}

template <typename V>
cudaError_t launch_typed(const void* src, void* dst, int64_t outer, int32_t row_bytes,
                         const PermGeom& g, bool inverse, cudaStream_t stream) {
    const int32_t vpr = row_bytes / int32_t(sizeof(V));
    int32_t shift = -1;
    if ((vpr & (vpr - 1)) == 0) {
        shift = 0;
        while ((1 << shift) < vpr) ++shift;
    }
    const int64_t blocks = outer * g.tiles;
    int dev = 0, sms = 0;
    if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return e;
    if (cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev); e != cudaSuccess) return e;
    const int64_t cap = int64_t(sms) * 16;
    const unsigned grid = unsigned(blocks < cap ? blocks : cap);
    if (g.tile_tokens <= kMaxTableTokens) {
        const size_t smem = size_t(g.tile_tokens) * sizeof(int32_t);
        auto kern = inverse ? permute_kernel<V, true, true> : permute_kernel<V, true, false>;
        if (smem > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
            if (e != cudaSuccess) return e;
        }
        kern<<<grid, kPermThreads, smem, stream>>>(static_cast<const V*>(src), static_cast<V*>(dst), g, vpr, shift,
                                                   blocks);
    } else {
        auto kern = inverse ? permute_kernel<V, false, true> : permute_kernel<V, false, false>;
        kern<<<grid, kPermThreads, 0, stream>>>(static_cast<const V*>(src), static_cast<V*>(dst), g, vpr, shift,
                                                blocks);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_permute(const void* src, void* dst, int64_t outer, int32_t row_bytes,
                           const sta_geom& sg, bool inverse, cudaStream_t stream) {
    PermGeom g;
    g.lat_t = sg.lat_t;
    g.lat_h = sg.lat_h;
    g.lat_w = sg.lat_w;
    g.tile_t = sg.tile_t;
    g.tile_h = sg.tile_h;
    g.tile_w = sg.tile_w;
    g.n_h = (sg.lat_h + sg.tile_h - 1) / sg.tile_h;
    g.n_w = (sg.lat_w + sg.tile_w - 1) / sg.tile_w;
    g.tiles = ((sg.lat_t + sg.tile_t - 1) / sg.tile_t) * g.n_h * g.n_w;
    g.tile_tokens = sg.tile_t * sg.tile_h * sg.tile_w;
    g.tokens = int64_t(sg.lat_t) * sg.lat_h * sg.lat_w;
    g.tm_tokens = int64_t(g.tiles) * g.tile_tokens;
    const uintptr_t align = reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst) |
                            uintptr_t(row_bytes);
    if (align % 16 == 0) return launch_typed<uint4>(src, dst, outer, row_bytes, g, inverse, stream);
    if (align % 8 == 0) return launch_typed<uint2>(src, dst, outer, row_bytes, g, inverse, stream);
    if (align % 4 == 0) return launch_typed<uint32_t>(src, dst, outer, row_bytes, g, inverse, stream);
    if (align % 2 == 0) return launch_typed<uint16_t>(src, dst, outer, row_bytes, g, inverse, stream);
    return launch_typed<uint8_t>(src, dst, outer, row_bytes, g, inverse, stream);
}

}  // namespace sta
