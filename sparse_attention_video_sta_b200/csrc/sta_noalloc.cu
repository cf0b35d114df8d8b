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
// cudaGetSymbolAddress and passed to the kernel.  The plan is written into a
// static host staging buffer (no heap use) and copied into the scratch on the
// caller's stream; that copy also zeroes the kernel's status word.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "sta.h"
#include "sta_internal.h"

namespace {

using sta::WorkItem;

constexpr size_t kScratchBytes = size_t(4) << 20;  // 4 MiB
constexpr size_t kHeaderBytes = 256;               // status word, padded
constexpr int kMaxHeads = 1024;
constexpr int kMaxDevices = 64;
constexpr uint64_t kTimeoutNs = 2000000000ull;

}  // namespace

// The scratch the no-allocation forward works in (one copy per device).
static __device__ __align__(256) uint8_t g_scratch[kScratchBytes];

namespace {

alignas(256) uint8_t g_staging[kScratchBytes];  // host-side image of the scratch
std::mutex g_mutex;                             // guards g_staging and g_scratch_ptr
void* g_scratch_ptr[kMaxDevices] = {};

int32_t window_start(int32_t q, int32_t e, int32_t n) {
    int32_t s = q - e / 2;
    if (s < 0) s = 0;
    if (s > n - e) s = n - e;
    return s;
}

// Device address of g_scratch on the current device (looked up once per device).
cudaError_t scratch_ptr(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
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

    // ---- distinct clamped windows, longest lists first (no heap: fixed arrays)
    static int32_t head_win[kMaxHeads];
    static int32_t win_e[kMaxHeads][3];
    static int32_t order[kMaxHeads];
    std::lock_guard<std::mutex> lock(g_mutex);
    int32_t n_win = 0;
    for (int32_t h = 0; h < heads; ++h) {
        int32_t e[3];
        for (int d = 0; d < 3; ++d) {
            e[d] = window_thw[3 * h + d] / T[d];
            if (e[d] > n[d]) e[d] = n[d];
        }
        int32_t id = -1;
        for (int32_t w = 0; w < n_win && id < 0; ++w)
            if (win_e[w][0] == e[0] && win_e[w][1] == e[1] && win_e[w][2] == e[2]) id = w;
        if (id < 0) {
            id = n_win++;
            for (int d = 0; d < 3; ++d) win_e[id][d] = e[d];
        }
        head_win[h] = id;
    }
    for (int32_t w = 0; w < n_win; ++w) order[w] = w;
    auto vol = [&](int32_t w) { return win_e[w][0] * win_e[w][1] * win_e[w][2]; };
    for (int32_t i = 1; i < n_win; ++i)  // insertion sort, descending list length, stable
        for (int32_t j = i; j > 0 && vol(order[j]) > vol(order[j - 1]); --j) {
            const int32_t t = order[j];
            order[j] = order[j - 1];
            order[j - 1] = t;
        }

    // ---- sizes and layout of the scratch image
    const int64_t items_per_head = int64_t(tiles) * (S / 2) + ((S % 2) ? (tiles + 1) / 2 : 0);
    const int64_t n_items = items_per_head * heads * batch;
    int64_t n_ids = 0;
    for (int32_t w = 0; w < n_win; ++w) n_ids += int64_t(tiles) * vol(w);
    const int64_t n_off = int64_t(n_win) * (tiles + 1);
    const size_t items_at = kHeaderBytes;
    const size_t off_at = items_at + size_t(n_items) * sizeof(WorkItem);
    const size_t ids_at = off_at + size_t(n_off) * sizeof(int32_t);
    const size_t total = ids_at + size_t(n_ids) * sizeof(int32_t);
    if (total > kScratchBytes || n_items > INT32_MAX) return STA_ERR_UNSUPPORTED;

    // ---- write the plan into the host staging image
    std::memset(g_staging, 0, kHeaderBytes);  // status word starts at zero
    int32_t* off = reinterpret_cast<int32_t*>(g_staging + off_at);
    int32_t* ids = reinterpret_cast<int32_t*>(g_staging + ids_at);
    int32_t pos = 0;
    for (int32_t w = 0; w < n_win; ++w) {
        const int32_t* e = win_e[w];
        for (int32_t qt = 0; qt < n[0]; ++qt)
            for (int32_t qh = 0; qh < n[1]; ++qh)
                for (int32_t qw = 0; qw < n[2]; ++qw) {
                    off[int64_t(w) * (tiles + 1) + (qt * n[1] + qh) * n[2] + qw] = pos;
                    const int32_t st = window_start(qt, e[0], n[0]);
                    const int32_t sh = window_start(qh, e[1], n[1]);
                    const int32_t sw = window_start(qw, e[2], n[2]);
                    for (int32_t kt = st; kt < st + e[0]; ++kt)
                        for (int32_t kh = sh; kh < sh + e[1]; ++kh)
                            for (int32_t kw = sw; kw < sw + e[2]; ++kw)
                                ids[pos++] = (kt * n[1] + kh) * n[2] + kw;
                }
        off[int64_t(w) * (tiles + 1) + tiles] = pos;
    }
    WorkItem* items = reinterpret_cast<WorkItem*>(g_staging + items_at);
    int64_t it = 0;
    for (int32_t oi = 0; oi < n_win; ++oi) {
        const int32_t w = order[oi];
        for (int32_t b = 0; b < batch; ++b)
            for (int32_t h = 0; h < heads; ++h) {
                if (head_win[h] != w) continue;
                const int32_t bh = b * heads + h;
                int32_t pending = -1;
                for (int32_t t = 0; t < tiles; ++t) {
                    for (int32_t s = 0; s + 1 < S; s += 2) items[it++] = WorkItem{bh, t * S + s, t * S + s + 1, w};
                    if (S % 2 == 1) {
                        const int32_t blk = t * S + S - 1;
                        if (pending < 0) {
                            pending = blk;
                        } else {
                            items[it++] = WorkItem{bh, pending, blk, w};
                            pending = -1;
                        }
                    }
                }
                if (pending >= 0) items[it++] = WorkItem{bh, pending, -1, w};
            }
    }
    if (it != n_items) return STA_ERR_UNSUPPORTED;  // cannot happen: sizes above match the loops

    // ---- copy into the device scratch and launch
    void* base = nullptr;
    if (scratch_ptr(&base) != cudaSuccess) return STA_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // Returns once the pageable staging image has been taken; the transfer is
    // ordered on `s` before the kernel.
    if (cudaMemcpyAsync(base, g_staging, total, cudaMemcpyHostToDevice, s) != cudaSuccess) return STA_ERR_CUDA;
    uint8_t* dev = static_cast<uint8_t*>(base);
    sta::RawPlanView pv;
    pv.batch = batch;
    pv.heads = heads;
    pv.tiles_per_head = tiles;
    pv.tile_tokens = tile_tokens;
    pv.sub_per_tile = S;
    pv.items = reinterpret_cast<const WorkItem*>(dev + items_at);
    pv.n_items = int32_t(n_items);
    pv.off = reinterpret_cast<const int32_t*>(dev + off_at);
    pv.ids = reinterpret_cast<const int32_t*>(dev + ids_at);
    pv.status = reinterpret_cast<uint32_t*>(dev);
    pv.timeout_ns = kTimeoutNs;
    const cudaError_t e = sta::launch_forward_raw(pv, q, k, v, o, lse, head_dim, softmax_scale, s);
    return e == cudaSuccess ? STA_OK : STA_ERR_CUDA;
}
