// sta_pipe.cu -- STA forward from host memory with the copies overlapped.
//
// A caller whose Q, K, V live in host memory pays two PCIe transfers per call,
// which at the pages' 720p size take longer than the attention itself.  The
// pipeline keeps a ring of `depth` device buffer sets and three streams: the
// copy-in of call i+1, the forward of call i and the copy-out of call i-1 run
// at once (B200 has separate copy engines for each direction).  Ordering per
// slot: copy-in waits until the slot's previous copy-out has finished, the
// forward waits for its copy-in, the copy-out waits for its forward.  Calls
// are asynchronous; sta_pipe_wait blocks until everything submitted is done.
#include <cuda_runtime.h>

#include <cmath>
#include <new>
#include <vector>

#include "sta.h"
#include "sta_internal.h"

namespace {

struct Slot {
    void* q = nullptr;
    void* k = nullptr;
    void* v = nullptr;
    void* o = nullptr;
    float* lse = nullptr;
    cudaEvent_t in_done = nullptr;   // copy-in finished
    cudaEvent_t fwd_done = nullptr;  // forward finished
    cudaEvent_t out_done = nullptr;  // copy-out finished: the slot is free
    bool used = false;
};

}  // namespace

struct sta_pipe_s {
    sta_plan_t plan = nullptr;
    int device = -1;
    int32_t head_dim = 0;
    float scale = 0.0f;
    size_t qkv_bytes = 0, lse_bytes = 0;
    cudaStream_t s_in = nullptr, s_fwd = nullptr, s_out = nullptr;
    std::vector<Slot> slots;
    int64_t next = 0;
};

namespace {

cudaError_t release(sta_pipe_s* p) {
    cudaError_t first = cudaSuccess;
    auto keep = [&](cudaError_t e) {
        if (first == cudaSuccess && e != cudaSuccess) first = e;
    };
    for (Slot& s : p->slots) {
        if (s.q) keep(cudaFree(s.q));
        if (s.k) keep(cudaFree(s.k));
        if (s.v) keep(cudaFree(s.v));
        if (s.o) keep(cudaFree(s.o));
        if (s.lse) keep(cudaFree(s.lse));
        if (s.in_done) keep(cudaEventDestroy(s.in_done));
        if (s.fwd_done) keep(cudaEventDestroy(s.fwd_done));
        if (s.out_done) keep(cudaEventDestroy(s.out_done));
    }
    p->slots.clear();
    if (p->s_in) keep(cudaStreamDestroy(p->s_in));
    if (p->s_fwd) keep(cudaStreamDestroy(p->s_fwd));
    if (p->s_out) keep(cudaStreamDestroy(p->s_out));
    p->s_in = p->s_fwd = p->s_out = nullptr;
    return first;
}

sta_status to_status(cudaError_t e) {
    if (e == cudaSuccess) return STA_OK;
    return e == cudaErrorMemoryAllocation ? STA_ERR_OOM : STA_ERR_CUDA;
}

}  // namespace

extern "C" {

sta_status sta_pipe_create(sta_plan_t plan, int32_t head_dim, float softmax_scale, int32_t depth,
                           sta_pipe_t* out) {
    if (out == nullptr) return STA_ERR_INVALID_ARG;
    *out = nullptr;
    if (plan == nullptr || !plan->on_device || depth < 1 || depth > 8) return STA_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale) || !(softmax_scale > 0.0f)) return STA_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return STA_ERR_UNSUPPORTED;
    // The pipeline keeps raster tensors and runs the fused forward.
    if (!sta::raster_box(plan->h.g).ok) return STA_ERR_UNSUPPORTED;
    if (plan->h.batch == 0) return STA_ERR_INVALID_ARG;  // no rows to pipeline
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return STA_ERR_CUDA;
    if (dev != plan->device) return STA_ERR_INVALID_ARG;
    sta_pipe_s* p = new (std::nothrow) sta_pipe_s();
    if (p == nullptr) return STA_ERR_OOM;
    const sta::PlanHost& P = plan->h;
    const int64_t rows = int64_t(P.batch) * P.heads * P.g.lat_t * P.g.lat_h * P.g.lat_w;
    p->plan = plan;
    p->device = dev;
    p->head_dim = head_dim;
    p->scale = softmax_scale;
    p->qkv_bytes = size_t(rows) * size_t(head_dim) * 2;
    p->lse_bytes = size_t(rows) * sizeof(float);
    cudaError_t e = cudaStreamCreateWithFlags(&p->s_in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p->s_fwd, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p->s_out, cudaStreamNonBlocking);
    if (e == cudaSuccess) {
        try {
            p->slots.resize(size_t(depth));
        } catch (const std::bad_alloc&) {
            release(p);
            delete p;
            return STA_ERR_OOM;
        }
    }
    for (Slot& s : p->slots) {
        if (e != cudaSuccess) break;
        e = cudaMalloc(&s.q, p->qkv_bytes);
        if (e == cudaSuccess) e = cudaMalloc(&s.k, p->qkv_bytes);
        if (e == cudaSuccess) e = cudaMalloc(&s.v, p->qkv_bytes);
        if (e == cudaSuccess) e = cudaMalloc(&s.o, p->qkv_bytes);
        if (e == cudaSuccess) e = cudaMalloc(reinterpret_cast<void**>(&s.lse), p->lse_bytes);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.in_done, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.fwd_done, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.out_done, cudaEventDisableTiming);
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        release(p);
        delete p;
        return to_status(e);
    }
    *out = p;
    return STA_OK;
}

sta_status sta_pipe_submit(sta_pipe_t p, const void* q_host, const void* k_host, const void* v_host, void* o_host,
                           float* lse_host) {
    if (p == nullptr || q_host == nullptr || k_host == nullptr || v_host == nullptr || o_host == nullptr ||
        lse_host == nullptr)
        return STA_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return STA_ERR_CUDA;
    if (dev != p->device) return STA_ERR_INVALID_ARG;
    Slot& s = p->slots[size_t(p->next % int64_t(p->slots.size()))];
    cudaError_t e = cudaSuccess;
    if (s.used) e = cudaStreamWaitEvent(p->s_in, s.out_done, 0);  // the slot's previous output is out
    if (e == cudaSuccess) e = cudaMemcpyAsync(s.q, q_host, p->qkv_bytes, cudaMemcpyHostToDevice, p->s_in);
    if (e == cudaSuccess) e = cudaMemcpyAsync(s.k, k_host, p->qkv_bytes, cudaMemcpyHostToDevice, p->s_in);
    if (e == cudaSuccess) e = cudaMemcpyAsync(s.v, v_host, p->qkv_bytes, cudaMemcpyHostToDevice, p->s_in);
    if (e == cudaSuccess) e = cudaEventRecord(s.in_done, p->s_in);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(p->s_fwd, s.in_done, 0);
    if (e != cudaSuccess) return to_status(e);
    const sta_status st = sta_forward_raster(p->plan, s.q, s.k, s.v, s.o, s.lse, p->head_dim, p->scale, p->s_fwd);
    if (st != STA_OK) return st;
    e = cudaEventRecord(s.fwd_done, p->s_fwd);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(p->s_out, s.fwd_done, 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(o_host, s.o, p->qkv_bytes, cudaMemcpyDeviceToHost, p->s_out);
    if (e == cudaSuccess) e = cudaMemcpyAsync(lse_host, s.lse, p->lse_bytes, cudaMemcpyDeviceToHost, p->s_out);
    if (e == cudaSuccess) e = cudaEventRecord(s.out_done, p->s_out);
    if (e != cudaSuccess) return to_status(e);
    s.used = true;
    ++p->next;
    return STA_OK;
}

sta_status sta_pipe_wait(sta_pipe_t p) {
    if (p == nullptr) return STA_ERR_INVALID_ARG;
    cudaError_t e = cudaStreamSynchronize(p->s_in);
    if (e == cudaSuccess) e = cudaStreamSynchronize(p->s_fwd);
    if (e == cudaSuccess) e = cudaStreamSynchronize(p->s_out);
    if (e != cudaSuccess) return to_status(e);
    return sta_last_device_status(p->plan, p->s_out);
}

sta_status sta_pipe_destroy(sta_pipe_t p) {
    if (p == nullptr) return STA_OK;
    cudaError_t e = cudaSuccess;
    if (p->s_in) {
        e = cudaStreamSynchronize(p->s_in);
        cudaError_t e2 = cudaStreamSynchronize(p->s_fwd), e3 = cudaStreamSynchronize(p->s_out);
        if (e == cudaSuccess) e = e2;
        if (e == cudaSuccess) e = e3;
    }
    const cudaError_t er = release(p);
    if (e == cudaSuccess) e = er;
    delete p;
    return to_status(e);
}

}  // extern "C"
