// sta_api.cu -- host side of the libsta C ABI: argument checks, the plan
// builder, and the launch / status plumbing around the kernels.
//
// The plan follows "Fast Video Generation with Sliding Tile Attention": every
// query tile attends the key tiles of a window of tiles centred on it, shifted
// to stay inside the volume, with one window per head (podcast transcript at
// hotaipapers.com, segments on tiles and on head specialisation; dianyo.github.io
// ICML-2025 post, STA section "Observation & Proposed Method").
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <map>
#include <new>
#include <tuple>
#include <vector>

#include "sta.h"
#include "sta_internal.h"

namespace {

using sta::PlanHost;
using sta::WorkItem;

std::atomic<int> g_inject_timeout{0};
std::atomic<int> g_inject_limit_ms{50};

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per device-side wait

// Name and text of the last CUDA error this library saw in the calling thread.
thread_local char g_detail[256] = "no error";

sta_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return STA_OK;
    snprintf(g_detail, sizeof g_detail, "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    return e == cudaErrorMemoryAllocation ? STA_ERR_OOM : STA_ERR_CUDA;
}

// Launches report their errors through cudaGetLastError, which also returns
// an error left behind by any earlier runtime call of this thread (for
// example one made by the framework on an autograd worker thread).  Entry
// points clear that record before they launch, so a status describes only
// this call.  Sticky errors (a lost context) are reported by the calls that
// follow.
void clear_stale_error() { (void)cudaGetLastError(); }

// The kernels' tensor maps are encoded through the driver API, which needs
// the device's context current in the calling thread; a thread whose first
// CUDA call this is (an autograd worker thread, a thread pool) has none until
// the runtime sets it up.  cudaSetDevice on the current device does.
cudaError_t make_context_current(int dev) { return cudaSetDevice(dev); }

bool geom_valid(const sta_geom* g) {
    if (g == nullptr) return false;
    const int32_t L[3] = {g->lat_t, g->lat_h, g->lat_w};
    const int32_t T[3] = {g->tile_t, g->tile_h, g->tile_w};
    for (int d = 0; d < 3; ++d) {
        if (L[d] <= 0 || T[d] <= 0) return false;
    }
    const int64_t n = int64_t(L[0]) * L[1] * L[2];
    return n <= INT32_MAX;
}

// Window start in tiles along one axis: centred on q, extent e, inside [0, n).
int32_t window_start(int32_t q, int32_t e, int32_t n) {
    return std::min(std::max(q - e / 2, 0), n - e);
}

// Order one-block work items for a persistent grid of `ctas` CTAs, CTA c
// taking items c, c + ctas, c + 2 ctas, ...: the items stay in natural
// (head, block) order round by round, so the CTAs work on neighbouring tiles
// of one head at the same time and share their K/V (or Q/dO) tiles in L2;
// inside each round the longest items go to the CTAs with the least work so
// far, which keeps the CTAs' totals level when list lengths vary.
template <class Len>
void order_rounds(std::vector<WorkItem>& items, const Len& len, int32_t ctas) {
    if (ctas < 1) ctas = 1;
    std::vector<int64_t> load(size_t(ctas), 0);
    std::vector<WorkItem> out(items.size());
    for (size_t r0 = 0; r0 < items.size(); r0 += size_t(ctas)) {
        const size_t n = std::min(size_t(ctas), items.size() - r0);
        std::vector<size_t> idx(n), slot(n);
        for (size_t i = 0; i < n; ++i) idx[i] = slot[i] = i;
        std::stable_sort(idx.begin(), idx.end(),
                         [&](size_t a, size_t b) { return len(items[r0 + a]) > len(items[r0 + b]); });
        std::stable_sort(slot.begin(), slot.end(), [&](size_t a, size_t b) { return load[a] < load[b]; });
        for (size_t i = 0; i < n; ++i) {
            out[r0 + slot[i]] = items[r0 + idx[i]];
            load[slot[i]] += len(items[r0 + idx[i]]);
        }
    }
    items.swap(out);
}

sta_status validate_plan_host(const PlanHost& P);

// `ctas`: the persistent grid the backward work lists are ordered for (the
// device's SM count; 148 for host-only plans).
sta_status build_plan_host(const sta_geom* g, int32_t batch, int32_t heads,
                           const int32_t* window_thw, int32_t ctas, PlanHost& P) {
    if (!geom_valid(g) || batch < 0 || heads < 1 || window_thw == nullptr)
        return STA_ERR_INVALID_ARG;
    const int32_t T[3] = {g->tile_t, g->tile_h, g->tile_w};
    const int32_t L[3] = {g->lat_t, g->lat_h, g->lat_w};
    for (int32_t h = 0; h < heads; ++h)
        for (int d = 0; d < 3; ++d) {
            const int32_t w = window_thw[3 * h + d];
            if (w <= 0 || w % T[d] != 0) return STA_ERR_INVALID_ARG;
        }
    P.g = *g;
    P.batch = batch;
    P.heads = heads;
    // An axis that is not a multiple of the tile is padded at its high end to
    // whole tiles (padding tokens are neither keys nor queries).
    for (int d = 0; d < 3; ++d) P.n_tiles[d] = (L[d] + T[d] - 1) / T[d];
    P.tiles_per_head = P.n_tiles[0] * P.n_tiles[1] * P.n_tiles[2];
    P.tile_tokens = T[0] * T[1] * T[2];
    if (P.tile_tokens % sta::kSubRows != 0) return STA_ERR_UNSUPPORTED;
    P.sub_per_tile = P.tile_tokens / sta::kSubRows;
    const int64_t n_tok = int64_t(P.tiles_per_head) * P.tile_tokens;
    // Row coordinates of the kernel's tensor maps are int32.
    if (int64_t(batch) * heads * n_tok > INT32_MAX) return STA_ERR_UNSUPPORTED;

    // Distinct clamped windows.
    std::map<std::tuple<int32_t, int32_t, int32_t>, int32_t> ids;
    P.head_win.assign(heads, 0);
    P.win_ext.clear();
    for (int32_t h = 0; h < heads; ++h) {
        int32_t e[3];
        for (int d = 0; d < 3; ++d) e[d] = std::min(window_thw[3 * h + d] / T[d], P.n_tiles[d]);
        auto key = std::make_tuple(e[0], e[1], e[2]);
        auto it = ids.find(key);
        if (it == ids.end()) {
            const int32_t id = int32_t(ids.size());
            ids.emplace(key, id);
            P.win_ext.insert(P.win_ext.end(), {e[0], e[1], e[2]});
            P.head_win[h] = id;
        } else {
            P.head_win[h] = it->second;
        }
    }
    const int32_t n_win = int32_t(ids.size());

    // Key-tile lists (CSR), ascending linear tile id.
    const int32_t nt = P.n_tiles[0], nh = P.n_tiles[1], nw = P.n_tiles[2];
    P.csr_off.assign(size_t(n_win) * (P.tiles_per_head + 1), 0);
    P.csr_ids.clear();
    std::vector<int32_t> list_len(n_win, 0);
    for (int32_t w = 0; w < n_win; ++w) {
        const int32_t* e = &P.win_ext[3 * w];
        list_len[w] = e[0] * e[1] * e[2];
        int32_t* off = &P.csr_off[size_t(w) * (P.tiles_per_head + 1)];
        for (int32_t qt = 0; qt < nt; ++qt)
            for (int32_t qh = 0; qh < nh; ++qh)
                for (int32_t qw = 0; qw < nw; ++qw) {
                    const int32_t q = (qt * nh + qh) * nw + qw;
                    off[q] = int32_t(P.csr_ids.size());
                    const int32_t st = window_start(qt, e[0], nt);
                    const int32_t sh = window_start(qh, e[1], nh);
                    const int32_t sw = window_start(qw, e[2], nw);
                    for (int32_t kt = st; kt < st + e[0]; ++kt)
                        for (int32_t kh = sh; kh < sh + e[1]; ++kh)
                            for (int32_t kw = sw; kw < sw + e[2]; ++kw)
                                P.csr_ids.push_back((kt * nh + kh) * nw + kw);
                }
        off[P.tiles_per_head] = int32_t(P.csr_ids.size());
    }

    // Raster origin of every tile (token coordinates of its first token).
    P.tile_origin.assign(size_t(P.tiles_per_head) * 4, 0);
    for (int32_t qt = 0; qt < nt; ++qt)
        for (int32_t qh = 0; qh < nh; ++qh)
            for (int32_t qw = 0; qw < nw; ++qw) {
                int32_t* o = &P.tile_origin[size_t((qt * nh + qh) * nw + qw) * 4];
                o[0] = qw * T[2];
                o[1] = qh * T[1];
                o[2] = qt * T[0];
            }

    // Padded latents: which keys of each 128-key chunk of a tile are real
    // tokens (bit j of word j / 32 for key j of the chunk).  Tiles at the
    // padded edge are the only ones with clear bits.
    P.padded = (L[0] % T[0]) != 0 || (L[1] % T[1]) != 0 || (L[2] % T[2]) != 0;
    P.key_mask.clear();
    if (P.padded) {
        P.key_mask.assign(size_t(P.tiles_per_head) * P.sub_per_tile * 4, 0u);
        for (int32_t tile = 0; tile < P.tiles_per_head; ++tile) {
            const int32_t* o = &P.tile_origin[size_t(tile) * 4];
            const int32_t vt = std::min(T[0], L[0] - o[2]), vh = std::min(T[1], L[1] - o[1]),
                          vw = std::min(T[2], L[2] - o[0]);
            for (int32_t l = 0; l < P.tile_tokens; ++l) {
                const int32_t x = l % T[2], y = (l / T[2]) % T[1], t = l / (T[2] * T[1]);
                if (t < vt && y < vh && x < vw) {
                    const int32_t sub = l / sta::kChunkKeys, j = l % sta::kChunkKeys;
                    P.key_mask[(size_t(tile) * P.sub_per_tile + sub) * 4 + j / 32] |= 1u << (j % 32);
                }
            }
        }
    }

    // Row blocks holding at least one real token (all of them unless the
    // latent is padded: a block of padding rows only has no output and no
    // keys, and is left out of every work list).
    const int32_t S = P.sub_per_tile;
    std::vector<uint8_t> real_block(size_t(P.tiles_per_head) * S, 1);
    if (P.padded)
        for (size_t blk = 0; blk < real_block.size(); ++blk) {
            const uint32_t* m = &P.key_mask[blk * 4];
            real_block[blk] = (m[0] | m[1] | m[2] | m[3]) != 0u;
        }

    P.computed_pairs = 0;
    for (int32_t b = 0; b < batch; ++b)
        for (int32_t h = 0; h < heads; ++h) P.computed_pairs += int64_t(P.tiles_per_head) * list_len[P.head_win[h]];
    // Forward work items (the key-split kernel): every real row block once,
    // head by head, longest lists first (stable sort).
    // Inside a head the query tiles follow a Morton (Z) order of their tile
    // coordinates, so the ~one SM count of blocks in flight at once covers a
    // compact 3D neighbourhood whose key windows overlap most (fewer distinct
    // K / V tiles live in L2 at a time than with raster order).
    std::vector<int32_t> zorder(size_t(P.tiles_per_head));
    {
        std::vector<std::pair<uint64_t, int32_t>> code(zorder.size());
        for (int32_t qt = 0; qt < nt; ++qt)
            for (int32_t qh = 0; qh < nh; ++qh)
                for (int32_t qw = 0; qw < nw; ++qw) {
                    uint64_t c = 0;
                    for (int bit = 0; bit < 21; ++bit)
                        c |= (uint64_t((qw >> bit) & 1) << (3 * bit)) | (uint64_t((qh >> bit) & 1) << (3 * bit + 1)) |
                             (uint64_t((qt >> bit) & 1) << (3 * bit + 2));
                    const int32_t q = (qt * nh + qh) * nw + qw;
                    code[size_t(q)] = {c, q};
                }
        std::sort(code.begin(), code.end());
        for (size_t i = 0; i < code.size(); ++i) zorder[i] = code[i].second;
    }
    P.f1_items.clear();
    for (int32_t b = 0; b < batch; ++b)
        for (int32_t h = 0; h < heads; ++h)
            for (int32_t r = 0; r < P.tiles_per_head; ++r)
                for (int32_t sub = 0; sub < S; ++sub) {
                    const int32_t blk = zorder[size_t(r)] * S + sub;
                    if (real_block[size_t(blk)]) P.f1_items.push_back(WorkItem{b * heads + h, blk, -1, P.head_win[h]});
                }
    std::stable_sort(P.f1_items.begin(), P.f1_items.end(), [&](const WorkItem& a, const WorkItem& b) {
        return list_len[a.win] > list_len[b.win];
    });

    // Backward: transposed lists (query tiles ascending for each key tile).
    const int32_t tph = P.tiles_per_head;
    P.tcsr_off.assign(size_t(n_win) * (tph + 1), 0);
    P.tcsr_ids.assign(P.csr_ids.size(), 0);
    for (int32_t w = 0; w < n_win; ++w) {
        const int32_t* off = &P.csr_off[size_t(w) * (tph + 1)];
        int32_t* toff = &P.tcsr_off[size_t(w) * (tph + 1)];
        std::vector<int32_t> cnt(tph, 0);
        for (int32_t q = 0; q < tph; ++q)
            for (int32_t i = off[q]; i < off[q + 1]; ++i) ++cnt[P.csr_ids[i]];
        toff[0] = off[0];
        for (int32_t kt = 0; kt < tph; ++kt) toff[kt + 1] = toff[kt] + cnt[kt];
        std::vector<int32_t> fill(toff, toff + tph);
        for (int32_t q = 0; q < tph; ++q)
            for (int32_t i = off[q]; i < off[q + 1]; ++i) P.tcsr_ids[fill[P.csr_ids[i]]++] = q;
    }
    // One-block work lists (ordered for the persistent grid below).
    P.bq_items.clear();
    P.bkv_items.clear();
    for (int32_t b = 0; b < batch; ++b)
        for (int32_t h = 0; h < heads; ++h) {
            const int32_t bh = b * heads + h, win = P.head_win[h];
            for (int32_t blk = 0; blk < tph * S; ++blk) {
                if (!real_block[size_t(blk)]) continue;  // padding rows only: no dQ, dK, dV to write
                P.bq_items.push_back(WorkItem{bh, blk, -1, win});
                P.bkv_items.push_back(WorkItem{bh, blk, -1, win});
            }
        }
    auto qlen = [&](const WorkItem& it) { return int64_t(list_len[it.win]); };
    auto tlen = [&](const WorkItem& it) {
        const int32_t* toff = &P.tcsr_off[size_t(it.win) * (tph + 1)];
        const int32_t kt = it.qa / S;
        return int64_t(toff[kt + 1] - toff[kt]);
    };
    order_rounds(P.bq_items, qlen, ctas);
    order_rounds(P.bkv_items, tlen, ctas);
    return validate_plan_host(P);
}

// Every index of the host plan against the plan's extents (see
// sta_plan_validate); on a violation the detail names the array and entry.
sta_status validate_plan_host(const PlanHost& P) {
    auto fail = [](const char* what, int64_t i) {
        snprintf(g_detail, sizeof g_detail, "plan index out of range: %s[%lld]", what, (long long)i);
        return STA_ERR_INVALID_ARG;
    };
    const int32_t T = P.tiles_per_head, S = P.sub_per_tile;
    const int64_t n_win = int64_t(P.win_ext.size() / 3);
    const int64_t n_bh = int64_t(P.batch) * P.heads;
    if (int64_t(P.head_win.size()) != P.heads) return fail("head_win", int64_t(P.head_win.size()));
    for (int32_t h = 0; h < P.heads; ++h)
        if (P.head_win[h] < 0 || P.head_win[h] >= n_win) return fail("head_win", h);
    for (int pass = 0; pass < 2; ++pass) {
        const std::vector<int32_t>& off = pass == 0 ? P.csr_off : P.tcsr_off;
        const std::vector<int32_t>& ids = pass == 0 ? P.csr_ids : P.tcsr_ids;
        const char* on = pass == 0 ? "csr_off" : "tcsr_off";
        const char* in = pass == 0 ? "csr_ids" : "tcsr_ids";
        if (int64_t(off.size()) != n_win * (T + 1)) return fail(on, int64_t(off.size()));
        for (int64_t w = 0; w < n_win; ++w)
            for (int32_t t = 0; t < T; ++t) {
                const int64_t i = w * (T + 1) + t;
                if (off[i] < 0 || off[i] > off[i + 1] || off[i + 1] > int64_t(ids.size())) return fail(on, i);
            }
        for (size_t i = 0; i < ids.size(); ++i)
            if (ids[i] < 0 || ids[i] >= T) return fail(in, int64_t(i));
    }
    // The transposed lists hold exactly the forward pairs: as many pairs,
    // each list strictly ascending, and every (key tile, query tile) pair of
    // them found (binary search) in the query tile's ascending forward list.
    for (int64_t w = 0; w < n_win; ++w) {
        const int32_t* off = &P.csr_off[size_t(w) * (T + 1)];
        const int32_t* toff = &P.tcsr_off[size_t(w) * (T + 1)];
        if (toff[T] - toff[0] != off[T] - off[0]) return fail("tcsr_off", w * (T + 1) + T);
        for (int32_t k = 0; k < T; ++k)
            for (int32_t j = toff[k]; j < toff[k + 1]; ++j) {
                const int32_t q = P.tcsr_ids[j];
                if (j > toff[k] && q <= P.tcsr_ids[j - 1]) return fail("tcsr_ids", j);
                const int32_t* a = P.csr_ids.data() + off[q];
                const int32_t* b = P.csr_ids.data() + off[q + 1];
                if (!std::binary_search(a, b, k)) return fail("tcsr_ids", j);
            }
    }
    const std::vector<WorkItem>* lists[3] = {&P.f1_items, &P.bq_items, &P.bkv_items};
    const char* names[3] = {"f1_items", "bq_items", "bkv_items"};
    for (int l = 0; l < 3; ++l)
        for (size_t i = 0; i < lists[l]->size(); ++i) {
            const WorkItem& it = (*lists[l])[i];
            if (it.bh < 0 || it.bh >= n_bh || it.qa < 0 || it.qa >= T * S || it.win < 0 || it.win >= n_win ||
                it.win != P.head_win[it.bh % P.heads])
                return fail(names[l], int64_t(i));
        }
    const int32_t Lp[3] = {P.n_tiles[0] * P.g.tile_t, P.n_tiles[1] * P.g.tile_h, P.n_tiles[2] * P.g.tile_w};
    for (int32_t t = 0; t < T; ++t) {
        const int32_t* o = &P.tile_origin[size_t(t) * 4];
        if (o[0] < 0 || o[0] >= Lp[2] || o[1] < 0 || o[1] >= Lp[1] || o[2] < 0 || o[2] >= Lp[0])
            return fail("tile_origin", t);
    }
    return STA_OK;
}

void free_device(sta_plan_s* p) {
    if (p->d_off) cudaFree(p->d_off);
    if (p->d_ids) cudaFree(p->d_ids);
    if (p->d_f1_items) cudaFree(p->d_f1_items);
    p->d_f1_items = nullptr;
    if (p->d_status) cudaFree(p->d_status);
    if (p->d_origin) cudaFree(p->d_origin);
    if (p->d_kmask) cudaFree(p->d_kmask);
    p->d_kmask = nullptr;
    if (p->d_counters) cudaFree(p->d_counters);
    p->d_counters = nullptr;
    if (p->d_toff) cudaFree(p->d_toff);
    if (p->d_tids) cudaFree(p->d_tids);
    if (p->d_bq_items) cudaFree(p->d_bq_items);
    if (p->d_bkv_items) cudaFree(p->d_bkv_items);
    p->d_toff = nullptr;
    p->d_tids = nullptr;
    p->d_bq_items = nullptr;
    p->d_bkv_items = nullptr;
    p->d_off = nullptr;
    p->d_ids = nullptr;
    p->d_status = nullptr;
    p->d_origin = nullptr;
    p->on_device = false;
}

template <class T>
cudaError_t upload(T** dst, const std::vector<T>& src, cudaStream_t stream) {
    const size_t bytes = std::max<size_t>(src.size(), 1) * sizeof(T);
    cudaError_t e = cudaMalloc(reinterpret_cast<void**>(dst), bytes);
    if (e != cudaSuccess) return e;
    if (!src.empty()) e = cudaMemcpyAsync(*dst, src.data(), src.size() * sizeof(T),
                                          cudaMemcpyHostToDevice, stream);
    return e;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

sta_status permute_common(const void* src, void* dst, int64_t outer, int32_t row_bytes,
                          const sta_geom* g, void* stream, bool inverse) {
    if (!geom_valid(g) || outer < 0 || row_bytes <= 0) return STA_ERR_INVALID_ARG;
    if (outer == 0) return STA_OK;  // no rows: nothing to move
    if (src == nullptr || dst == nullptr) return STA_ERR_INVALID_ARG;
    const int64_t n_tok = int64_t(g->lat_t) * g->lat_h * g->lat_w;
    int64_t n_pad = 1;  // tile-major rows per slice: whole tiles
    const int32_t L[3] = {g->lat_t, g->lat_h, g->lat_w}, T[3] = {g->tile_t, g->tile_h, g->tile_w};
    for (int d = 0; d < 3; ++d) n_pad *= int64_t((L[d] + T[d] - 1) / T[d]) * T[d];
    const int64_t r_bytes = outer * n_tok * int64_t(row_bytes), t_bytes = outer * n_pad * int64_t(row_bytes);
    const int64_t s_bytes = inverse ? t_bytes : r_bytes, d_bytes = inverse ? r_bytes : t_bytes;
    const uintptr_t s = reinterpret_cast<uintptr_t>(src), d = reinterpret_cast<uintptr_t>(dst);
    if (s < d + uint64_t(d_bytes) && d < s + uint64_t(s_bytes)) return STA_ERR_INVALID_ARG;  // overlap
    clear_stale_error();
    return cuda_status(sta::launch_permute(src, dst, outer, row_bytes, *g, inverse,
                                           static_cast<cudaStream_t>(stream)));
}

sta_status forward_common(sta_plan_t p, const void* q, const void* k, const void* v, void* o, float* lse,
                          int32_t head_dim, float softmax_scale, void* stream, bool raster) {
    if (p == nullptr || !p->on_device) return STA_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale) || !(softmax_scale > 0.0f)) return STA_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return STA_ERR_UNSUPPORTED;
    if (raster && !sta::raster_box(p->h.g).ok) return STA_ERR_UNSUPPORTED;
    if (p->h.batch == 0) return STA_OK;  // no rows: nothing to compute
    if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || lse == nullptr)
        return STA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(lse, 4))
        return STA_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return cuda_status(e);
    if (dev != p->device) return STA_ERR_INVALID_ARG;
    if (cudaError_t e = make_context_current(dev); e != cudaSuccess) return cuda_status(e);
    const int inject = g_inject_timeout.load();
    const uint64_t limit = inject ? uint64_t(g_inject_limit_ms.load()) * 1000000ull
                                  : kDefaultTimeoutNs;
    clear_stale_error();
    return cuda_status(sta::launch_forward(p, q, k, v, o, lse, head_dim, softmax_scale,
                                           static_cast<cudaStream_t>(stream), inject, limit, raster));
}

constexpr int32_t kHostPlanCtas = 148;  // B200 SM count, for plans built without a device

sta_status plan_host_for(const sta_geom* g, int32_t batch, int32_t heads, const int32_t* window_thw,
                         int32_t ctas, sta_plan_t* out) {
    if (out == nullptr) return STA_ERR_INVALID_ARG;
    *out = nullptr;
    sta_plan_s* p = new (std::nothrow) sta_plan_s();
    if (p == nullptr) return STA_ERR_OOM;
    sta_status st;
    try {
        st = build_plan_host(g, batch, heads, window_thw, ctas, p->h);
    } catch (const std::bad_alloc&) {
        st = STA_ERR_OOM;
    }
    if (st != STA_OK) {
        delete p;
        return st;
    }
    *out = p;
    return STA_OK;
}

sta_status backward_common(sta_plan_t p, const void* q, const void* k, const void* v, const void* o,
                           const void* dout, const float* lse, void* dq, void* dk, void* dv, float* workspace,
                           int32_t head_dim, float softmax_scale, void* stream, bool raster) {
    if (p == nullptr || !p->on_device) return STA_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale) || !(softmax_scale > 0.0f)) return STA_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return STA_ERR_UNSUPPORTED;
    if (raster && !sta::raster_box(p->h.g).ok) return STA_ERR_UNSUPPORTED;
    if (p->h.batch == 0) return STA_OK;  // no rows: nothing to compute
    const void* in16[] = {q, k, v, o, dout, dq, dk, dv, workspace};
    for (const void* x : in16)
        if (x == nullptr || !aligned(x, 16)) return STA_ERR_INVALID_ARG;
    if (lse == nullptr || !aligned(lse, 4)) return STA_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return cuda_status(e);
    if (dev != p->device) return STA_ERR_INVALID_ARG;
    if (cudaError_t e = make_context_current(dev); e != cudaSuccess) return cuda_status(e);
    clear_stale_error();
    return cuda_status(sta::launch_backward(p, q, k, v, o, dout, lse, dq, dk, dv, workspace, head_dim,
                                            softmax_scale, static_cast<cudaStream_t>(stream), kDefaultTimeoutNs,
                                            raster));
}

}  // namespace

extern "C" {

const char* sta_status_string(sta_status s) {
    switch (s) {
        case STA_OK: return "STA_OK";
        case STA_ERR_INVALID_ARG: return "STA_ERR_INVALID_ARG";
        case STA_ERR_UNSUPPORTED: return "STA_ERR_UNSUPPORTED";
        case STA_ERR_CUDA: return "STA_ERR_CUDA";
        case STA_ERR_TIMEOUT: return "STA_ERR_TIMEOUT";
        case STA_ERR_OOM: return "STA_ERR_OOM";
        case STA_ERR_BOUNDS: return "STA_ERR_BOUNDS";
    }
    return "STA_ERR_UNKNOWN";
}

sta_status sta_plan_host(const sta_geom* g, int32_t batch, int32_t heads,
                         const int32_t* window_thw, sta_plan_t* out) {
    return plan_host_for(g, batch, heads, window_thw, kHostPlanCtas, out);
}

sta_status sta_plan(const sta_geom* g, int32_t batch, int32_t heads,
                    const int32_t* window_thw, void* stream, sta_plan_t* out) {
    int dev = -1, sms = 0;
    if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return cuda_status(e);
    if (cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev); e != cudaSuccess)
        return cuda_status(e);
    sta_status st = plan_host_for(g, batch, heads, window_thw, sms, out);
    if (st != STA_OK) return st;
    sta_plan_s* p = *out;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaGetDevice(&p->device);
    if (e == cudaSuccess) e = upload(&p->d_off, p->h.csr_off, s);
    if (e == cudaSuccess) e = upload(&p->d_ids, p->h.csr_ids, s);
    if (e == cudaSuccess) e = upload(&p->d_f1_items, p->h.f1_items, s);
    if (e == cudaSuccess) e = upload(&p->d_origin, p->h.tile_origin, s);
    if (e == cudaSuccess && p->h.padded) e = upload(&p->d_kmask, p->h.key_mask, s);
    if (e == cudaSuccess)
        e = cudaMalloc(reinterpret_cast<void**>(&p->d_counters), sta::kCounterPool * sizeof(int32_t));
    if (e == cudaSuccess) e = upload(&p->d_toff, p->h.tcsr_off, s);
    if (e == cudaSuccess) e = upload(&p->d_tids, p->h.tcsr_ids, s);
    if (e == cudaSuccess) e = upload(&p->d_bq_items, p->h.bq_items, s);
    if (e == cudaSuccess) e = upload(&p->d_bkv_items, p->h.bkv_items, s);
    if (e == cudaSuccess) e = cudaMalloc(reinterpret_cast<void**>(&p->d_status), sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaMemsetAsync(p->d_status, 0, sizeof(uint32_t), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) {
        const sta_status st = cuda_status(e);
        cudaGetLastError();
        free_device(p);
        delete p;
        *out = nullptr;
        return st;
    }
    p->on_device = true;
    return STA_OK;
}

sta_status sta_plan_destroy(sta_plan_t p) {
    if (p == nullptr) return STA_OK;
    sta_status st = STA_OK;
    if (p->on_device || p->d_off || p->d_ids || p->d_f1_items || p->d_status || p->d_origin || p->d_kmask ||
        p->d_counters || p->d_toff ||
        p->d_tids || p->d_bq_items || p->d_bkv_items) {
        if (cudaDeviceSynchronize() != cudaSuccess) st = STA_ERR_CUDA;
        free_device(p);
    }
    delete p;
    return st;
}

sta_status sta_plan_query(sta_plan_t p, int32_t head, int32_t q_tile, int32_t* kv_ids,
                          int32_t cap, int32_t* count) {
    if (p == nullptr || count == nullptr || cap < 0 || (cap > 0 && kv_ids == nullptr))
        return STA_ERR_INVALID_ARG;
    const PlanHost& P = p->h;
    if (head < 0 || head >= P.heads || q_tile < 0 || q_tile >= P.tiles_per_head)
        return STA_ERR_INVALID_ARG;
    const int32_t* off = &P.csr_off[size_t(P.head_win[head]) * (P.tiles_per_head + 1)];
    const int32_t n = off[q_tile + 1] - off[q_tile];
    *count = n;
    for (int32_t i = 0; i < std::min(n, cap); ++i) kv_ids[i] = P.csr_ids[off[q_tile] + i];
    return STA_OK;
}

sta_status sta_plan_key_query(sta_plan_t p, int32_t head, int32_t k_tile, int32_t* q_ids,
                              int32_t cap, int32_t* count) {
    if (p == nullptr || count == nullptr || cap < 0 || (cap > 0 && q_ids == nullptr))
        return STA_ERR_INVALID_ARG;
    const PlanHost& P = p->h;
    if (head < 0 || head >= P.heads || k_tile < 0 || k_tile >= P.tiles_per_head)
        return STA_ERR_INVALID_ARG;
    const int32_t* off = &P.tcsr_off[size_t(P.head_win[head]) * (P.tiles_per_head + 1)];
    const int32_t n = off[k_tile + 1] - off[k_tile];
    *count = n;
    for (int32_t i = 0; i < std::min(n, cap); ++i) q_ids[i] = P.tcsr_ids[off[k_tile] + i];
    return STA_OK;
}

sta_status sta_plan_stats(sta_plan_t p, int64_t* computed_tile_pairs, int64_t* work_items) {
    if (p == nullptr) return STA_ERR_INVALID_ARG;
    if (computed_tile_pairs) *computed_tile_pairs = p->h.computed_pairs;
    if (work_items) *work_items = int64_t(p->h.f1_items.size());
    return STA_OK;
}

sta_status sta_plan_work_items(sta_plan_t p, int32_t* items4, int64_t cap, int64_t* count) {
    if (p == nullptr || count == nullptr || cap < 0 || (cap > 0 && items4 == nullptr))
        return STA_ERR_INVALID_ARG;
    const auto& it = p->h.f1_items;
    *count = int64_t(it.size());
    const int64_t n = std::min<int64_t>(cap, int64_t(it.size()));
    for (int64_t i = 0; i < n; ++i) {
        items4[4 * i + 0] = it[i].bh;
        items4[4 * i + 1] = it[i].qa;
        items4[4 * i + 2] = it[i].qb;
        items4[4 * i + 3] = it[i].win;
    }
    return STA_OK;
}

sta_status sta_plan_backward_items(sta_plan_t p, int32_t which, int32_t* items4, int64_t cap, int64_t* count) {
    if (p == nullptr || count == nullptr || cap < 0 || (cap > 0 && items4 == nullptr) || which < 0 || which > 1)
        return STA_ERR_INVALID_ARG;
    const auto& it = which == 0 ? p->h.bq_items : p->h.bkv_items;
    *count = int64_t(it.size());
    const int64_t n = std::min<int64_t>(cap, int64_t(it.size()));
    for (int64_t i = 0; i < n; ++i) {
        items4[4 * i + 0] = it[i].bh;
        items4[4 * i + 1] = it[i].qa;
        items4[4 * i + 2] = it[i].qb;
        items4[4 * i + 3] = it[i].win;
    }
    return STA_OK;
}

sta_status sta_tile_reorder(const void* src, void* dst, int64_t outer, int32_t row_bytes,
                            const sta_geom* g, void* stream) {
    return permute_common(src, dst, outer, row_bytes, g, stream, false);
}

sta_status sta_tile_unreorder(const void* src, void* dst, int64_t outer, int32_t row_bytes,
                              const sta_geom* g, void* stream) {
    return permute_common(src, dst, outer, row_bytes, g, stream, true);
}

sta_status sta_forward(sta_plan_t p, const void* q, const void* k, const void* v, void* o,
                       float* lse, int32_t head_dim, float softmax_scale, void* stream) {
    return forward_common(p, q, k, v, o, lse, head_dim, softmax_scale, stream, false);
}

sta_status sta_forward_raster(sta_plan_t p, const void* q, const void* k, const void* v, void* o,
                              float* lse, int32_t head_dim, float softmax_scale, void* stream) {
    return forward_common(p, q, k, v, o, lse, head_dim, softmax_scale, stream, true);
}

sta_status sta_backward(sta_plan_t p, const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv,
                        float* workspace, int32_t head_dim, float softmax_scale, void* stream) {
    return backward_common(p, q, k, v, o, dout, lse, dq, dk, dv, workspace, head_dim, softmax_scale, stream,
                           false);
}

sta_status sta_backward_raster(sta_plan_t p, const void* q, const void* k, const void* v, const void* o,
                               const void* dout, const float* lse, void* dq, void* dk, void* dv,
                               float* workspace, int32_t head_dim, float softmax_scale, void* stream) {
    return backward_common(p, q, k, v, o, dout, lse, dq, dk, dv, workspace, head_dim, softmax_scale, stream,
                           true);
}

sta_status sta_window_stats(const float* lse_w, const float* lse_full, const void* o_w, const void* o_full,
                            int64_t slices, int64_t tokens, int32_t head_dim, double* recall, double* mse,
                            void* stream) {
    // 8 CTAs per slice in the launch grid
    if (slices < 0 || slices > (int64_t(1) << 28) || tokens < 1 || head_dim < 8 || head_dim % 8 != 0)
        return STA_ERR_INVALID_ARG;
    if (slices == 0) return STA_OK;  // no slices: nothing to reduce
    if (lse_w == nullptr || lse_full == nullptr || o_w == nullptr || o_full == nullptr || recall == nullptr ||
        mse == nullptr)
        return STA_ERR_INVALID_ARG;
    if (!aligned(lse_w, 4) || !aligned(lse_full, 4) || !aligned(o_w, 16) || !aligned(o_full, 16) ||
        !aligned(recall, 8) || !aligned(mse, 8))
        return STA_ERR_INVALID_ARG;
    clear_stale_error();
    return cuda_status(sta::launch_window_stats(lse_w, lse_full, o_w, o_full, slices, tokens, head_dim, recall,
                                                mse, static_cast<cudaStream_t>(stream)));
}

sta_status sta_last_device_status(sta_plan_t p, void* stream) {
    if (p == nullptr || !p->on_device) return STA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaError_t e = cudaStreamSynchronize(s); e != cudaSuccess) return cuda_status(e);
    if (cudaError_t e = cudaGetLastError(); e != cudaSuccess) return cuda_status(e);
    uint32_t word = 0;
    if (cudaError_t e = cudaMemcpy(&word, p->d_status, sizeof word, cudaMemcpyDeviceToHost); e != cudaSuccess)
        return cuda_status(e);
    if (word != 0) {
        if (cudaError_t e = cudaMemset(p->d_status, 0, sizeof word); e != cudaSuccess) return cuda_status(e);
    }
    if (word & sta::kDevBounds) return STA_ERR_BOUNDS;
    if (word & sta::kDevTimeout) return STA_ERR_TIMEOUT;
    return STA_OK;
}

const char* sta_last_error_detail(void) { return g_detail; }

sta_status sta_window_pick(const sta_geom* g, int32_t heads, int32_t n_cand, const int32_t* cand_thw,
                           const double* recall, const double* mse, double max_mse, double min_recall,
                           int32_t* out_thw) {
    if (!geom_valid(g) || heads < 1 || n_cand < 0 || out_thw == nullptr) return STA_ERR_INVALID_ARG;
    if (n_cand > 0 && (cand_thw == nullptr || recall == nullptr || mse == nullptr)) return STA_ERR_INVALID_ARG;
    const int32_t L[3] = {g->lat_t, g->lat_h, g->lat_w}, T[3] = {g->tile_t, g->tile_h, g->tile_w};
    int32_t n[3];
    for (int d = 0; d < 3; ++d) n[d] = (L[d] + T[d] - 1) / T[d];
    std::vector<int64_t> tiles(size_t(n_cand), 1);
    for (int32_t c = 0; c < n_cand; ++c)
        for (int d = 0; d < 3; ++d) {
            const int32_t w = cand_thw[3 * c + d];
            if (w <= 0 || w % T[d] != 0) return STA_ERR_INVALID_ARG;
            tiles[size_t(c)] *= std::min(w / T[d], n[d]);
        }
    std::vector<int32_t> order(static_cast<size_t>(n_cand));
    for (int32_t c = 0; c < n_cand; ++c) order[size_t(c)] = c;
    std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) { return tiles[a] < tiles[b]; });
    for (int32_t h = 0; h < heads; ++h) {
        const int32_t* pick = L;  // the window covering the volume
        for (int32_t c : order) {
            const double r = recall[size_t(c) * heads + h], e = mse[size_t(c) * heads + h];
            if ((max_mse < 0.0 || e <= max_mse) && (min_recall < 0.0 || r >= min_recall)) {
                pick = cand_thw + 3 * c;
                break;
            }
        }
        for (int d = 0; d < 3; ++d) out_thw[3 * h + d] = pick[d];
    }
    return STA_OK;
}

sta_status sta_plan_validate(sta_plan_t p) {
    if (p == nullptr) return STA_ERR_INVALID_ARG;
    return validate_plan_host(p->h);
}

sta_status sta_debug_plan_poke(sta_plan_t p, int32_t which, int64_t index, int32_t value) {
    if (p == nullptr || index < 0) return STA_ERR_INVALID_ARG;
    PlanHost& P = p->h;
    int32_t* host = nullptr;
    void* dev = nullptr;
    int64_t n = 0;
    switch (which) {
        case 0: n = int64_t(P.csr_ids.size()); host = P.csr_ids.data(); dev = p->d_ids; break;
        case 1: n = int64_t(P.f1_items.size()) * 4; host = reinterpret_cast<int32_t*>(P.f1_items.data());
                dev = p->d_f1_items; break;
        case 2: n = int64_t(P.csr_off.size()); host = P.csr_off.data(); dev = p->d_off; break;
        case 3: n = int64_t(P.tcsr_ids.size()); host = P.tcsr_ids.data(); dev = p->d_tids; break;
        default: return STA_ERR_INVALID_ARG;
    }
    if (index >= n) return STA_ERR_INVALID_ARG;
    host[index] = value;
    if (p->on_device && dev != nullptr) {
        if (cudaError_t e = cudaMemcpy(static_cast<int32_t*>(dev) + index, &value, sizeof value,
                                       cudaMemcpyHostToDevice);
            e != cudaSuccess)
            return cuda_status(e);
    }
    return STA_OK;
}

sta_status sta_debug_inject_timeout(int32_t mode, int32_t limit_ms) {
    if (limit_ms < 1 || limit_ms > 10000 || mode < 0 || mode > 2) return STA_ERR_INVALID_ARG;
    g_inject_timeout.store(mode);
    g_inject_limit_ms.store(limit_ms);
    return STA_OK;
}

}  // extern "C"
