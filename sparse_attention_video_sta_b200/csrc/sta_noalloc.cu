// sta_noalloc.cu -- STA forward for callers that cannot allocate device memory.
//
// sta_plan allocates the plan's device arrays with cudaMalloc.  Some callers
// cannot do that: processes whose device memory is owned by another allocator
// or memory pool that forbids outside cudaMalloc calls, deployments that reserve
// every byte at start-up and allow no allocation (and no implicit device
// synchronisation) once serving, and plugin hosts that hand a kernel library
// only the buffers they want it to touch.  sta_forward_noalloc serves them: the
// plan lives in a fixed-size scratch array compiled into this library, so the
// call needs nothing but the caller's own Q, K, V, O and LSE buffers.
//
// The scratch is a file-scope __device__ array (every GPU that loads the library
// holds it until the process exits).  Host code cannot use its name as a device
// address, so its address is looked up once per device with
// cudaGetSymbolAddress and passed to the kernels.  Each call first runs a small
// kernel that writes the plan into the scratch -- key-tile lists, work list,
// a zeroed status word and work counter -- from the per-head windows it takes
// as a kernel parameter, then the forward kernel over that plan.  No host
// buffer is copied to the device.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "sta.h"
#include "sta_internal.h"

namespace {

using sta::WorkItem;

constexpr size_t kScratchBytes = size_t(4) << 20;  // 4 MiB
constexpr size_t kHeaderBytes = 256;               // status word, work counter, padding
constexpr int kMaxHeads = 1024;
constexpr int kMaxDevices = 64;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr int kPlanThreads = 1024;
constexpr int kPlanBlocks = 64;

// The problem, passed by value to the plan-writing kernel (about 6 KB of
// kernel parameters: no host-to-device copy is needed).
struct PlanArgs {
    int32_t batch, heads;
    int32_t n[3];             // tile grid
    int32_t sub_per_tile;     // 128-row blocks per tile
    int32_t tiles;            // tiles per head
    int32_t n_win;            // distinct clamped windows
    uint32_t items_at, off_at, ids_at;  // byte offsets in the scratch
    uint16_t ext[kMaxHeads][3];         // clamped window extent of each head, in tiles
};

}  // namespace

// The scratch the no-allocation forward works in (one copy per device).
static __device__ __align__(256) uint8_t g_scratch[kScratchBytes];

namespace {

__device__ __forceinline__ int32_t window_start_dev(int32_t q, int32_t e, int32_t n) {
    int32_t s = q - e / 2;
    s = s < 0 ? 0 : s;
    return s > n - e ? n - e : s;
}

// Writes the plan of one call into the scratch (every CTA derives the same
// per-head tables, then writes its share of the arrays):
//   - distinct windows in order of first appearance among the heads, each with
//     the ascending key-tile list of every query tile (CSR, the same lists as
//     sta_plan's);
//   - one work item per (b, h, 128-row block), ordered by descending list
//     length, then b, then h (the order sta_plan gives);
//   - the status word and the work counter, zeroed.
__global__ void __launch_bounds__(kPlanThreads) noalloc_plan_kernel(const PlanArgs a, uint8_t* scratch) {
    __shared__ int32_t s_vol[kMaxHeads];   // list length of each head's window
    __shared__ int32_t s_first[kMaxHeads]; // first head with the same window
    __shared__ int32_t s_win[kMaxHeads];   // distinct-window id of each head
    __shared__ int32_t s_rank[kMaxHeads];  // (b, h) order: heads with longer lists, same-length heads
    __shared__ int32_t s_eq[kMaxHeads];    // heads with the same list length
    __shared__ int32_t s_wbase[kMaxHeads + 1];  // CSR start of each distinct window (in ids)
    __shared__ int32_t s_whead[kMaxHeads];      // a head of each distinct window
    const int H = a.heads;
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
        s_vol[h] = int32_t(a.ext[h][0]) * a.ext[h][1] * a.ext[h][2];
        int32_t f = h;
        for (int g = 0; g < h; ++g)
            if (a.ext[g][0] == a.ext[h][0] && a.ext[g][1] == a.ext[h][1] && a.ext[g][2] == a.ext[h][2]) {
                f = g;
                break;
            }
        s_first[h] = f;
    }
    __syncthreads();
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
        int32_t id = 0, gt = 0, eq = 0, eqlt = 0;
        for (int g = 0; g < H; ++g) {
            if (g < s_first[h] && s_first[g] == g) ++id;
            gt += s_vol[g] > s_vol[h];
            eq += s_vol[g] == s_vol[h];
            eqlt += (g < h) && s_vol[g] == s_vol[h];
        }
        s_win[h] = id;
        s_rank[h] = gt * a.batch + eqlt;  // + b * eq for batch b
        s_eq[h] = eq;
        if (s_first[h] == h) s_whead[id] = h;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int32_t acc = 0;
        for (int w = 0; w < a.n_win; ++w) {
            s_wbase[w] = acc;
            acc += a.tiles * s_vol[s_whead[w]];
        }
        s_wbase[a.n_win] = acc;
    }
    __syncthreads();

    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    const int64_t tid = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (tid == 0) {
        reinterpret_cast<uint32_t*>(scratch)[0] = 0u;  // status word
        reinterpret_cast<int32_t*>(scratch)[1] = 0;    // work counter
    }
    // CSR offsets: window w's list of query tile q starts at base(w) + q vol(w).
    int32_t* off = reinterpret_cast<int32_t*>(scratch + a.off_at);
    const int64_t n_off = int64_t(a.n_win) * (a.tiles + 1);
    for (int64_t i = tid; i < n_off; i += stride) {
        const int32_t w = int32_t(i / (a.tiles + 1)), q = int32_t(i % (a.tiles + 1));
        off[i] = s_wbase[w] + q * s_vol[s_whead[w]];
    }
    // Key-tile ids: entry j of query tile q's list, raster order over the
    // window's (t, h, w) offsets, which is ascending tile id.
    int32_t* ids = reinterpret_cast<int32_t*>(scratch + a.ids_at);
    const int64_t n_ids = s_wbase[a.n_win];
    for (int64_t i = tid; i < n_ids; i += stride) {
        int32_t lo = 0, hi = a.n_win - 1;  // the window holding entry i
        while (lo < hi) {
            const int32_t mid = (lo + hi + 1) >> 1;
            if (s_wbase[mid] <= i) lo = mid; else hi = mid - 1;
        }
        const int32_t hw = s_whead[lo];
        const int32_t e0 = a.ext[hw][0], e1 = a.ext[hw][1], e2 = a.ext[hw][2];
        const int32_t vol = e0 * e1 * e2;
        const int32_t r = int32_t(i - s_wbase[lo]);
        const int32_t q = r / vol, j = r % vol;
        const int32_t qw = q % a.n[2], qh = (q / a.n[2]) % a.n[1], qt = q / (a.n[2] * a.n[1]);
        const int32_t jw = j % e2, jh = (j / e2) % e1, jt = j / (e2 * e1);
        const int32_t kt = window_start_dev(qt, e0, a.n[0]) + jt;
        const int32_t kh = window_start_dev(qh, e1, a.n[1]) + jh;
        const int32_t kw = window_start_dev(qw, e2, a.n[2]) + jw;
        ids[i] = (kt * a.n[1] + kh) * a.n[2] + kw;
    }
    // Work items: (b, h) groups in descending list length, then b, then h.
    WorkItem* items = reinterpret_cast<WorkItem*>(scratch + a.items_at);
    const int32_t per_head = a.tiles * a.sub_per_tile;
    const int64_t n_items = int64_t(a.batch) * H * per_head;
    for (int64_t i = tid; i < n_items; i += stride) {
        const int32_t bh = int32_t(i / per_head), blk = int32_t(i % per_head);
        const int32_t b = bh / H, h = bh % H;
        const int64_t rank = int64_t(s_rank[h]) + int64_t(b) * s_eq[h];
        items[rank * per_head + blk] = WorkItem{bh, blk, -1, s_win[h]};
    }
}

std::mutex g_mutex;  // guards g_scratch_ptr
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device (looked up once per device).
cudaError_t scratch_ptr(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" sta_status sta_forward_noalloc(const sta_geom* g, int32_t batch, int32_t heads,
                                          const int32_t* window_thw, const void* q, const void* k,
                                          const void* v, void* o, float* lse, int32_t head_dim,
                                          float softmax_scale, void* stream) {
    // ---- arguments (same rules as sta_plan + sta_forward)
    if (g == nullptr || window_thw == nullptr || batch < 0 || heads < 1) return STA_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale) || !(softmax_scale > 0.0f)) return STA_ERR_INVALID_ARG;
    const int32_t L[3] = {g->lat_t, g->lat_h, g->lat_w};
    const int32_t T[3] = {g->tile_t, g->tile_h, g->tile_w};
    int32_t n[3];
    for (int d = 0; d < 3; ++d) {
        if (L[d] <= 0 || T[d] <= 0) return STA_ERR_INVALID_ARG;
        if (L[d] % T[d] != 0) return STA_ERR_UNSUPPORTED;  // padded latents: sta_plan + sta_forward
        n[d] = L[d] / T[d];
    }
    for (int32_t h = 0; h < heads; ++h)
        for (int d = 0; d < 3; ++d) {
            const int32_t w = window_thw[3 * h + d];
            if (w <= 0 || w % T[d] != 0) return STA_ERR_INVALID_ARG;
        }
    if (head_dim != 64 && head_dim != 128) return STA_ERR_UNSUPPORTED;
    if (heads > kMaxHeads) return STA_ERR_UNSUPPORTED;
    if (n[0] > 65535 || n[1] > 65535 || n[2] > 65535) return STA_ERR_UNSUPPORTED;
    const int64_t n_tok = int64_t(L[0]) * L[1] * L[2];
    const int32_t tile_tokens = T[0] * T[1] * T[2];
    if (tile_tokens % sta::kSubRows != 0) return STA_ERR_UNSUPPORTED;
    if (int64_t(batch) * heads * n_tok > INT32_MAX) return STA_ERR_UNSUPPORTED;
    if (batch == 0) return STA_OK;  // no rows: nothing to compute
    if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || lse == nullptr)
        return STA_ERR_INVALID_ARG;
    auto aligned = [](const void* p, uintptr_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; };
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
        return STA_ERR_INVALID_ARG;
    const int32_t tiles = n[0] * n[1] * n[2];
    const int32_t S = tile_tokens / sta::kSubRows;

    // ---- clamped windows; distinct ones counted for the scratch layout
    PlanArgs a;
    a.batch = batch;
    a.heads = heads;
    for (int d = 0; d < 3; ++d) a.n[d] = n[d];
    a.sub_per_tile = S;
    a.tiles = tiles;
    int32_t n_win = 0;
    int64_t n_ids = 0;
    for (int32_t h = 0; h < heads; ++h) {
        for (int d = 0; d < 3; ++d) {
            const int32_t e = window_thw[3 * h + d] / T[d];
            a.ext[h][d] = uint16_t(e < n[d] ? e : n[d]);
        }
        bool seen = false;
        for (int32_t g2 = 0; g2 < h && !seen; ++g2)
            seen = a.ext[g2][0] == a.ext[h][0] && a.ext[g2][1] == a.ext[h][1] && a.ext[g2][2] == a.ext[h][2];
        if (!seen) {
            ++n_win;
            n_ids += int64_t(tiles) * a.ext[h][0] * a.ext[h][1] * a.ext[h][2];
        }
    }
    a.n_win = n_win;

    // ---- sizes and layout of the scratch
    const int64_t n_items = int64_t(batch) * heads * tiles * S;
    const int64_t n_off = int64_t(n_win) * (tiles + 1);
    const size_t items_at = kHeaderBytes;
    const size_t off_at = items_at + size_t(n_items) * sizeof(WorkItem);
    const size_t ids_at = off_at + size_t(n_off) * sizeof(int32_t);
    const size_t total = ids_at + size_t(n_ids) * sizeof(int32_t);
    if (total > kScratchBytes || n_items > INT32_MAX) return STA_ERR_UNSUPPORTED;
    a.items_at = uint32_t(items_at);
    a.off_at = uint32_t(off_at);
    a.ids_at = uint32_t(ids_at);

    // ---- write the plan into the scratch on the stream, then launch the forward
    void* base = nullptr;
    if (scratch_ptr(&base) != cudaSuccess) return STA_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* dev = static_cast<uint8_t*>(base);
    (void)cudaGetLastError();  // a status describes this call only
    noalloc_plan_kernel<<<kPlanBlocks, kPlanThreads, 0, s>>>(a, dev);
    if (cudaGetLastError() != cudaSuccess) return STA_ERR_CUDA;
    sta::RawPlanView pv;
    pv.batch = batch;
    pv.heads = heads;
    pv.tiles_per_head = tiles;
    pv.tile_tokens = tile_tokens;
    pv.sub_per_tile = S;
    pv.items = reinterpret_cast<const WorkItem*>(dev + items_at);
    pv.n_items = int32_t(n_items);
    pv.item_counter = reinterpret_cast<int32_t*>(dev + 4);
    pv.off = reinterpret_cast<const int32_t*>(dev + off_at);
    pv.ids = reinterpret_cast<const int32_t*>(dev + ids_at);
    pv.status = reinterpret_cast<uint32_t*>(dev);
    pv.timeout_ns = kTimeoutNs;
    pv.n_win = n_win;
    pv.n_ids = int32_t(n_ids);
    const cudaError_t e = sta::launch_forward_raw(pv, q, k, v, o, lse, head_dim, softmax_scale, s);
    return e == cudaSuccess ? STA_OK : STA_ERR_CUDA;
}
