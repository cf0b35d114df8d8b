// sta_backward.cu -- Sliding Tile Attention backward pass for sm_100a (B200).
//
// Fine-tuning a video DiT with STA in place of full attention ("Fast Video
// Generation with Sliding Tile Attention": podcast transcript at
// hotaipapers.com, fine-tuning segment; dianyo.github.io ICML-2025 post, STA
// section, last paragraph) needs gradients through the sparse attention.  The
// pages give no backward kernel; this one computes the exact gradient of the
// forward's function with the tile window held fixed.  For query row i, key j
// in its window, P_ij = exp(scale q_i.k_j - LSE_i) (LSE from the forward):
//
//   dV_j = sum_i P_ij dO_i,   dP_ij = dO_i . v_j,   D_i = dO_i . O_i,
//   dS_ij = P_ij (dP_ij - D_i),
//   dQ_i = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i.
//
// (D_i = dO_i . O_i equals sum_j P_ij dP_ij because O_i = sum_j P_ij v_j.)
//
// Three launches, no atomics (results are deterministic):
//   1. bwd_prep_kernel: -D_i and -LSE_i log2(e) per row into the workspace.
//   2. sta_bwd_dq_kernel, one 128-row query block per work item, walking the
//      block's key tiles (the forward's lists) in 128-key chunks:
//        S = Q K^T, dP = dO V^T (tcgen05, SMEM operands) -> TMEM;
//        P = exp2(S c - LSE log2 e), dS = P (dP - D) by the elementwise warps,
//        dS as bf16 written back into TMEM over dP;
//        dQ += dS K (tcgen05, A operand from TMEM, K as an MN-major SMEM operand).
//      TMEM: S0 | S1 | dP | dQ; S is double-buffered so the next chunk's
//      scores are computed while the elementwise warps work.
//   3. sta_bwd_dkdv_kernel, one 128-key block per work item, walking the query
//      tiles whose windows hold the block's tile (the lists transposed):
//        S^T = K Q^T, dP^T = V dO^T -> TMEM;  P^T and dS^T by the elementwise
//        warps (per-column LSE and D from shared memory), bf16 over S^T / dP^T;
//        dV += P^T dO, dK += dS^T Q (A from TMEM, B MN-major from SMEM).
//      TMEM: S^T | dP^T | dV | dK.
//
// Both main kernels are persistent (one CTA per SM) with one TMA load warp, one
// tcgen05 issuing warp and two elementwise warpgroups (each owns 64 of the 128
// columns of every row).  Every mbarrier wait is bounded; on expiry the kernel
// records a timeout, drains and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "sta_bounds.cuh"
#include "sta_internal.h"
#include "sta_ptx.cuh"
#include "sta_raster.cuh"
#include "sta_wait.cuh"

namespace sta {
namespace {

constexpr int kBwThreads = 320;  // warps 0-7 elementwise, 8 load, 9 MMA
constexpr int kBwLoadWarp = 8;
constexpr int kBwMmaWarp = 9;
constexpr int kEwWarps = 8;
constexpr uint32_t kBwTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kBoxBytes = 128 * 128;  // one TMA box: 128 rows x 128 bytes (64 bf16)
// Work items are handed out at run time, as in the forward: the load warp
// takes the next item from a per-launch global counter and passes it to the
// MMA thread and the eight elementwise warps through a queue in shared memory.
constexpr int kItemQ = 4;
constexpr int kItemConsumers = 1 + kEwWarps;
// Shared memory requested at launch is at least this, so one CTA holds an SM
// alone: a second CTA on the SM would wait in tcgen05.alloc for the 512 TMEM
// columns until the first one exits.
constexpr int kMinSmemLaunch = 120 * 1024;
constexpr int smem_launch(int bytes) { return bytes > kMinSmemLaunch ? bytes : kMinSmemLaunch; }

struct BwdParams {
    const WorkItem* items;
    int32_t n_items;
    const int32_t* off;  // CSR offsets [n_win][tiles + 1]: key tiles per query tile (dQ), or query tiles per key tile (dK/dV)
    const int32_t* ids;
    int32_t tiles_per_head;
    int32_t sub_per_tile;
    int32_t tile_tokens;
    int32_t tokens;
    const float* neg_d;  // workspace plane 0: -D per row
    const float* neg_l;  // workspace plane 1: -LSE log2(e) per row
    __nv_bfloat16* out_a;  // dQ (dQ kernel) or dK (dK/dV kernel)
    __nv_bfloat16* out_b;  // dV (dK/dV kernel)
    float scale_log2;      // softmax_scale * log2(e)
    float scale;
    uint32_t* status;
    uint64_t timeout_ns;
    RasterGeom rg;          // raster layout only
    int32_t* item_counter;  // next item to hand out (zeroed before the launch); null: fixed stride
    PlanBounds pb;          // extents of the plan arrays (checked by the debug build)
};

__device__ __forceinline__ bool wait_bw(uint32_t bar, uint32_t parity, volatile int* abort_flag, const BwdParams& p) {
    return wait_bar_limited(bar, parity, abort_flag, p.status, p.timeout_ns);
}

// One 128-row block of a tile-major [rows, D] bf16 tensor: D / 64 boxes.
template <int D>
__device__ __forceinline__ void load_rows(uint32_t dst, const CUtensorMap* m, uint32_t bar, int32_t row) {
#pragma unroll
    for (int cb = 0; cb < D / 64; ++cb) ptx::tma_load_2d(dst + cb * kBoxBytes, m, bar, cb * 64, row);
}

// Producer side of the item queue (one thread): publish this CTA's k-th item
// (-1: none left) in entry k % kItemQ once that entry's previous item has been
// taken by every consumer.  Returns the item, or -2 when the CTA is aborting.
__device__ __forceinline__ int32_t put_item(uint32_t k, uint32_t full0, uint32_t empty0, volatile int32_t* q,
                                            volatile int* abort_flag, const BwdParams& p) {
    int32_t u = p.item_counter != nullptr ? atomicAdd(p.item_counter, 1) : int32_t(blockIdx.x + k * gridDim.x);
    if (u >= p.n_items) u = -1;
    if (kDebugBounds && u >= 0 && !item_in_bounds(p.items, p.n_items, u, p.off, p.ids, p.pb, p.status)) {
        *abort_flag = 1;  // no more items: every role leaves its loop
        u = -1;
    }
    const uint32_t e = k % kItemQ;
    if (k >= uint32_t(kItemQ) && !wait_bw(empty0 + 8u * e, ((k / kItemQ) - 1) & 1u, abort_flag, p)) return -2;
    q[e] = u;
    ptx::mbar_arrive(full0 + 8u * e);
    return u;
}

// Consumer side: wait for entry k and read it; false when the CTA is aborting.
__device__ __forceinline__ bool get_item(uint32_t k, uint32_t full0, volatile int32_t* q, volatile int* abort_flag,
                                        const BwdParams& p, int32_t& u) {
    if (!wait_bw(full0 + 8u * (k % kItemQ), (k / kItemQ) & 1u, abort_flag, p)) return false;
    u = q[k % kItemQ];
    return true;
}

// 128-row block `sub` of tile `tile` of head bh: tile-major rows (2D map) or
// a raster box (5D map).
template <int D, bool kRaster>
__device__ __forceinline__ void load_blk(uint32_t dst, const CUtensorMap* m, uint32_t bar, const BwdParams& p,
                                         int32_t bh, int32_t tile, int32_t sub) {
    if (!kRaster)
        load_rows<D>(dst, m, bar, bh * p.tokens + tile * p.tile_tokens + sub * 128);
    else
        raster_load(dst, m, bar, p.rg, bh, tile, sub, D / 64, kBoxBytes);
}

// Output row of row `r` of block `blk` of head bh; -1 for a padding row of a
// raster output.
template <bool kRaster, bool kPadded>
__device__ __forceinline__ int64_t bwd_out_row(const BwdParams& p, int32_t bh, int32_t blk, int32_t r) {
    if (!kRaster) return int64_t(bh) * p.tokens + int64_t(blk) * 128 + r;
    return raster_row<kPadded>(p.rg, bh, blk, r);
}

// 64 fp32 values -> 32 bf16 pairs.
__device__ __forceinline__ void pack64(const float (&x)[64], uint32_t (&pk)[32]) {
#pragma unroll
    for (int i = 0; i < 32; ++i) pk[i] = ptx::pack_bf16x2(x[2 * i], x[2 * i + 1]);
}

// Epilogue: `cols` fp32 TMEM columns of this thread's lane (starting at taddr),
// times `mul`, as bf16 to dst (16-byte aligned, cols contiguous elements).
// Every lane loads (the TMEM access is warp-wide); only lanes with `store` write.
template <int kCols>
__device__ __forceinline__ void store_cols(uint32_t taddr, float mul, __nv_bfloat16* dst, bool store) {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll 1
    for (int cb = 0; cb < kCols / 32; ++cb) {
        uint32_t r[32];
        ptx::tmem_ld32(taddr + cb * 32, r);
        if (!store) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint4 v;
            v.x = ptx::pack_bf16x2(__uint_as_float(r[8 * j + 0]) * mul, __uint_as_float(r[8 * j + 1]) * mul);
            v.y = ptx::pack_bf16x2(__uint_as_float(r[8 * j + 2]) * mul, __uint_as_float(r[8 * j + 3]) * mul);
            v.z = ptx::pack_bf16x2(__uint_as_float(r[8 * j + 4]) * mul, __uint_as_float(r[8 * j + 5]) * mul);
            v.w = ptx::pack_bf16x2(__uint_as_float(r[8 * j + 6]) * mul, __uint_as_float(r[8 * j + 7]) * mul);
            d4[cb * 4 + j] = v;
        }
    }
}

// A-operand column of K-step kk (16 keys / queries) of a bf16 matrix that the
// two elementwise warpgroups wrote into TMEM: warpgroup h packs its 64 columns
// into columns [64 h, 64 h + 32) of the region.
__device__ __forceinline__ uint32_t a_col(int kk) { return uint32_t((kk >> 2) * 64 + (kk & 3) * 8); }

// ---------------------------------------------------------------- prep
// neg_d[r] = -sum_c dO[r, c] O[r, c];  neg_l[r] = -lse[r] log2(e), for every
// tile-major row r (the planes are tile-major in both layouts, so a 128-row
// block's values are one contiguous 512-byte copy).  kRaster: O, dO and LSE
// are raster tensors, read at the row's raster token; a padding row gets 0
// for both (its dO is 0, so it adds nothing to dK or dV).
// D / 8 threads per row, 16 bytes of each tensor per thread.
template <int D, bool kRaster, bool kPadded>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const uint4* __restrict__ o, const uint4* __restrict__ dout,
                                                       const float* __restrict__ lse, float* __restrict__ neg_d,
                                                       float* __restrict__ neg_l, int64_t rows, int32_t tokens,
                                                       const RasterGeom rg) {
    constexpr int kTpr = D / 8;
    const int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t row = t / kTpr;
    const int part = int(t % kTpr);
    int64_t src = row;
    if ((kRaster || kPadded) && row < rows) {
        // raster layout: the row's raster position; padded latents: -1 for a
        // padding row, whose O and LSE rows may be unwritten (the forward skips
        // blocks of padding rows only) and which gets 0 in both planes
        const int32_t bh = int32_t(row / tokens), within = int32_t(row % tokens);
        const int64_t r = raster_row<kPadded>(rg, bh, within / 128, within % 128);
        src = kRaster ? r : (r < 0 ? -1 : row);
    }
    float acc = 0.0f;
    if (row < rows && src >= 0) {
        const uint4 a = __ldg(o + src * kTpr + part), b = __ldg(dout + src * kTpr + part);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc = fmaf(__uint_as_float(aw[i] << 16), __uint_as_float(bw[i] << 16), acc);
            acc = fmaf(__uint_as_float(aw[i] & 0xffff0000u), __uint_as_float(bw[i] & 0xffff0000u), acc);
        }
    }
#pragma unroll
    for (int s = kTpr / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if (row < rows && part == 0) {
        neg_d[row] = -acc;
        neg_l[row] = src >= 0 ? -lse[src] * kLog2e : 0.0f;
    }
}

// ---------------------------------------------------------------- dQ
template <int D>
struct DqCfg {
    static constexpr int kBlk = 128 * D * 2;  // one 128-row bf16 block
    static constexpr int kKStages = 3, kVStages = 2;
    static constexpr int kQOff = 0, kDOOff = kBlk;
    static constexpr int kKOff = 2 * kBlk;
    static constexpr int kVOff = kKOff + kKStages * kBlk;
    static constexpr int kBarOff = kVOff + kVStages * kBlk;
    // k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], q_full, q_empty,
    // s_full[2], dp_full, ds_full, dq_full, drain, item_full[Q], item_empty[Q]
    static constexpr int kNumBars = 2 * kKStages + 2 * kVStages + 9 + 2 * kItemQ;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem slot, abort flag, item queue
    static constexpr int kSmemBytes = kMiscOff + 8 + 4 * kItemQ + 1024;
    static constexpr uint32_t kColS0 = 0, kColDP = 256, kColDQ = 384;
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
    static_assert(kColDQ + D <= kBwTmemCols, "TMEM budget");
};

template <int D, bool kRaster, bool kPadded>
__global__ void __launch_bounds__(kBwThreads, 1)
sta_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const BwdParams p) {
    using C = DqCfg<D>;
    constexpr int KS = C::kKStages, VS = C::kVStages;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const uint32_t bar0 = base + C::kBarOff;
    auto k_full = [&](int r) { return bar0 + 8u * r; };
    auto k_empty = [&](int r) { return bar0 + 8u * (KS + r); };
    auto v_full = [&](int r) { return bar0 + 8u * (2 * KS + r); };
    auto v_empty = [&](int r) { return bar0 + 8u * (2 * KS + VS + r); };
    const uint32_t xb = bar0 + 8u * (2 * KS + 2 * VS);
    const uint32_t q_full = xb, q_empty = xb + 8;
    auto s_full = [&](int b) { return xb + 16 + 8u * b; };
    const uint32_t dp_full = xb + 32, ds_full = xb + 40, dq_full = xb + 48, drain = xb + 56;
    const uint32_t item_full0 = xb + 64, item_empty0 = xb + 64 + 8 * kItemQ;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
    volatile int32_t* item_q = reinterpret_cast<volatile int32_t*>(smem + C::kMiscOff + 8);

    if (threadIdx.x == 0) {
        for (int r = 0; r < KS; ++r) {
            ptx::mbar_init(k_full(r), 1);
            ptx::mbar_init(k_empty(r), 1);
        }
        for (int r = 0; r < VS; ++r) {
            ptx::mbar_init(v_full(r), 1);
            ptx::mbar_init(v_empty(r), 1);
        }
        ptx::mbar_init(q_full, 1);
        ptx::mbar_init(q_empty, 1);
        ptx::mbar_init(s_full(0), 1);
        ptx::mbar_init(s_full(1), 1);
        ptx::mbar_init(dp_full, 1);
        ptx::mbar_init(ds_full, kEwWarps);
        ptx::mbar_init(dq_full, 1);
        ptx::mbar_init(drain, 1);
        for (int q = 0; q < kItemQ; ++q) {
            ptx::mbar_init(item_full0 + 8u * q, 1);
            ptx::mbar_init(item_empty0 + 8u * q, kItemConsumers);
        }
        *abort_flag = 0;
        ptx::fence_barrier_init();
        ptx::fence_proxy_async_smem();
    }
    if (warp == kBwLoadWarp && lane == 0) {
        ptx::prefetch_tensormap(&tm_q);
        ptx::prefetch_tensormap(&tm_k);
        ptx::prefetch_tensormap(&tm_v);
        ptx::prefetch_tensormap(&tm_do);
    }
    if (warp == kBwMmaWarp) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kBwTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int32_t SPT = p.sub_per_tile;

    if (warp == kBwLoadWarp) {
        if (lane == 0) {
            // ------------------------------------------------------------ load
            uint32_t kit = 0, vit = 0, qc = 0;
            bool ok = true;
            for (uint32_t kq = 0; ok; ++kq) {
                const int32_t u = put_item(kq, item_full0, item_empty0, item_q, abort_flag, p);
                if (u == -2) { ok = false; break; }
                if (u < 0) break;
                const WorkItem w = p.items[u];
                const int32_t tile = w.qa / SPT;
                const int32_t* off = p.off + int64_t(w.win) * (p.tiles_per_head + 1);
                const int32_t* list = p.ids + off[tile];
                const int32_t n_kt = off[tile + 1] - off[tile];
                if (!wait_bw(q_empty, (qc & 1u) ^ 1u, abort_flag, p)) { ok = false; break; }
                ptx::mbar_arrive_expect_tx(q_full, 2 * C::kBlk);
                load_blk<D, kRaster>(base + C::kQOff, &tm_q, q_full, p, w.bh, tile, w.qa - tile * SPT);
                load_blk<D, kRaster>(base + C::kDOOff, &tm_do, q_full, p, w.bh, tile, w.qa - tile * SPT);
                ++qc;
                for (int32_t kt = 0; ok && kt < n_kt; ++kt) {
                    const int32_t t = __ldg(list + kt);
                    for (int32_t kc = 0; ok && kc < SPT; ++kc) {
                        const int rk = int(kit % KS);
                        if (kit >= uint32_t(KS) && !wait_bw(k_empty(rk), ((kit / KS) - 1) & 1u, abort_flag, p)) {
                            ok = false;
                            break;
                        }
                        ptx::mbar_arrive_expect_tx(k_full(rk), C::kBlk);
                        load_blk<D, kRaster>(base + C::kKOff + rk * C::kBlk, &tm_k, k_full(rk), p, w.bh, t, kc);
                        ++kit;
                        const int rv = int(vit % VS);
                        if (vit >= uint32_t(VS) && !wait_bw(v_empty(rv), ((vit / VS) - 1) & 1u, abort_flag, p)) {
                            ok = false;
                            break;
                        }
                        ptx::mbar_arrive_expect_tx(v_full(rv), C::kBlk);
                        load_blk<D, kRaster>(base + C::kVOff + rv * C::kBlk, &tm_v, v_full(rv), p, w.bh, t, kc);
                        ++vit;
                    }
                }
            }
            // Drain the copies still in flight.
            for (uint32_t it = kit > uint32_t(KS) ? kit - KS : 0u; it < kit; ++it)
                drain_bar(k_full(int(it % KS)), (it / KS) & 1u, p.timeout_ns);
            for (uint32_t it = vit > uint32_t(VS) ? vit - VS : 0u; it < vit; ++it)
                drain_bar(v_full(int(it % VS)), (it / VS) & 1u, p.timeout_ns);
            if (qc > 0) drain_bar(q_full, (qc - 1) & 1u, p.timeout_ns);
        }
    } else if (warp == kBwMmaWarp) {
        if (lane == 0) {
            // ------------------------------------------------------------- MMA
            constexpr uint32_t idesc_s = ptx::idesc_bf16(128, 128, false);
            constexpr uint32_t idesc_dq = ptx::idesc_bf16(128, D, true);
            const uint32_t qaddr = base + C::kQOff, doaddr = base + C::kDOOff;
            uint32_t kbase = 0, vbase = 0, gs = 0, qc = 0;
            bool ok = true;
            for (uint32_t kq = 0; ok; ++kq) {
                int32_t u;
                if (!get_item(kq, item_full0, item_q, abort_flag, p, u)) { ok = false; break; }
                ptx::mbar_arrive(item_empty0 + 8u * (kq % kItemQ));
                if (u < 0) break;
                const WorkItem w = p.items[u];
                const int32_t tile = w.qa / SPT;
                const int32_t* off = p.off + int64_t(w.win) * (p.tiles_per_head + 1);
                const int32_t n = (off[tile + 1] - off[tile]) * SPT;
                if (!wait_bw(q_full, qc & 1u, abort_flag, p)) { ok = false; break; }
                ++qc;
                ptx::tc_fence_after();
                // S_j = Q K_j^T into S buffer (gs + j) & 1
                auto issue_s = [&](int32_t j) -> bool {
                    const uint32_t it = kbase + uint32_t(j);
                    if (!wait_bw(k_full(int(it % KS)), (it / KS) & 1u, abort_flag, p)) return false;
                    ptx::tc_fence_after();
                    const uint32_t kaddr = base + C::kKOff + (it % KS) * C::kBlk;
                    const uint32_t tS = tmem + C::kColS0 + ((gs + uint32_t(j)) & 1u) * 128u;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t coff = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
                        ptx::mma_ss(tS, ptx::desc_k_sw128(qaddr + coff), ptx::desc_k_sw128(kaddr + coff), idesc_s,
                                    kk > 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(s_full(int((gs + uint32_t(j)) & 1u)));
                    return true;
                };
                // dP_j = dO V_j^T; V_j is then free
                auto issue_dp = [&](int32_t j) -> bool {
                    const uint32_t it = vbase + uint32_t(j);
                    if (!wait_bw(v_full(int(it % VS)), (it / VS) & 1u, abort_flag, p)) return false;
                    ptx::tc_fence_after();
                    const uint32_t vaddr = base + C::kVOff + (it % VS) * C::kBlk;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t coff = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
                        ptx::mma_ss(tmem + C::kColDP, ptx::desc_k_sw128(doaddr + coff),
                                    ptx::desc_k_sw128(vaddr + coff), idesc_s, kk > 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(dp_full);
                    ptx::mma_commit(v_empty(int(it % VS)));
                    return true;
                };
                ok = issue_s(0) && issue_dp(0) && (n < 2 || issue_s(1));
                for (int32_t j = 0; ok && j < n; ++j) {
                    if (!wait_bw(ds_full, (gs + uint32_t(j)) & 1u, abort_flag, p)) { ok = false; break; }
                    ptx::tc_fence_after();
                    // dQ += dS_j K_j (dS from TMEM over dP; K_j MN-major)
                    const uint32_t it = kbase + uint32_t(j);
                    const uint32_t kaddr = base + C::kKOff + (it % KS) * C::kBlk;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        ptx::mma_ts(tmem + C::kColDQ, tmem + C::kColDP + a_col(kk),
                                    ptx::desc_mn_sw128(kaddr + kk * 16 * 128, kBoxBytes), idesc_dq,
                                    (j > 0 || kk > 0) ? 1u : 0u);
                    ptx::mma_commit(k_empty(int(it % KS)));
                    // in issue order after dQ_j, which reads the dS this dP overwrites
                    if (j + 1 < n && !issue_dp(j + 1)) { ok = false; break; }
                    if (j + 2 < n && !issue_s(j + 2)) { ok = false; break; }
                }
                if (!ok) break;
                ptx::mma_commit(dq_full);
                ptx::mma_commit(q_empty);
                kbase += uint32_t(n);
                vbase += uint32_t(n);
                gs += uint32_t(n);
            }
            ptx::mma_commit(drain);
            drain_bar(drain, 0, p.timeout_ns);
        }
    } else {
        // ------------------------------------------------------- elementwise
        const int h = warp >> 2;  // column half
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_addr = uint32_t((warp & 3) * 32) << 16;
        const uint64_t c2 = ptx::f2(p.scale_log2, p.scale_log2);
        uint32_t gs = 0, dqc = 0;
        bool ok = true;
        for (uint32_t kq = 0; ok; ++kq) {
            int32_t u = -1;
            if (!__all_sync(0xffffffffu, get_item(kq, item_full0, item_q, abort_flag, p, u))) break;
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(item_empty0 + 8u * (kq % kItemQ));
            if (u < 0) break;
            const WorkItem w = p.items[u];
            const int32_t tile = w.qa / SPT;
            const int32_t* off = p.off + int64_t(w.win) * (p.tiles_per_head + 1);
            const int32_t n = (off[tile + 1] - off[tile]) * SPT;
            const int64_t grow = int64_t(w.bh) * p.tokens + int64_t(w.qa) * 128 + row;
            const float nl = __ldg(p.neg_l + grow), nd = __ldg(p.neg_d + grow);
            const uint64_t nl2 = ptx::f2(nl, nl), nd2 = ptx::f2(nd, nd);
            for (int32_t j = 0; j < n; ++j) {
                const uint32_t step = gs + uint32_t(j);
                if (!__all_sync(0xffffffffu, wait_bw(s_full(int(step & 1u)), (step >> 1) & 1u, abort_flag, p))) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                float pr[64];
                {
                    uint32_t sr[64];
                    ptx::tmem_ld64(tmem + lane_addr + C::kColS0 + (step & 1u) * 128u + 64u * h, sr);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        float x0, x1;
                        ptx::f2_split(ptx::f2_fma(ptx::f2(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])),
                                                  c2, nl2),
                                      x0, x1);
                        pr[2 * i] = ptx::ex2(x0);
                        pr[2 * i + 1] = ptx::ex2(x1);
                    }
                }
                if (!__all_sync(0xffffffffu, wait_bw(dp_full, step & 1u, abort_flag, p))) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t tdp = tmem + lane_addr + C::kColDP + 64u * h;
                uint32_t pk[32];
                {
                    uint32_t dr[64];
                    ptx::tmem_ld64(tdp, dr);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        float t0, t1;
                        ptx::f2_split(ptx::f2_mul(ptx::f2(pr[2 * i], pr[2 * i + 1]),
                                                  ptx::f2_add(ptx::f2(__uint_as_float(dr[2 * i]),
                                                                      __uint_as_float(dr[2 * i + 1])),
                                                              nd2)),
                                      t0, t1);
                        pk[i] = ptx::pack_bf16x2(t0, t1);
                    }
                }
                ptx::tmem_st32(tdp, pk);
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ds_full);
            }
            if (!ok) break;
            if (!__all_sync(0xffffffffu, wait_bw(dq_full, dqc & 1u, abort_flag, p))) break;
            ++dqc;
            ptx::tc_fence_after();
            const int64_t orow = bwd_out_row<kRaster, kPadded>(p, w.bh, w.qa, row);
            store_cols<D / 2>(tmem + lane_addr + C::kColDQ + uint32_t(D / 2) * h, p.scale,
                              p.out_a + (orow < 0 ? 0 : orow) * D + (D / 2) * h, orow >= 0);
            ptx::tc_fence_before();
            gs += uint32_t(n);
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kBwMmaWarp) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kBwTmemCols);
    }
}

// ---------------------------------------------------------------- dK / dV
template <int D>
struct DkvCfg {
    static constexpr int kBlk = 128 * D * 2;
    static constexpr int kStages = 2;
    static constexpr int kKOff = 0, kVOff = kBlk;
    // stage: Q block, dO block, -LSE log2(e) [128], -D [128]
    static constexpr int kStQ = 0, kStDO = kBlk, kStL = 2 * kBlk, kStD = 2 * kBlk + 512;
    static constexpr int kStageBytes = 2 * kBlk + 1024;
    static constexpr int kStageOff = 2 * kBlk;
    static constexpr int kBarOff = kStageOff + kStages * kStageBytes;
    // st_full[2], st_empty[2], kv_full, kv_empty, s_full, dp_full, p_full,
    // ds_full, dkv_full, drain, item_full[Q], item_empty[Q]
    static constexpr int kNumBars = 2 * kStages + 8 + 2 * kItemQ;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem slot, abort flag, item queue
    static constexpr int kSmemBytes = kMiscOff + 8 + 4 * kItemQ + 1024;
    static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
    static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
    static_assert(kColDK + D <= kBwTmemCols, "TMEM budget");
};

template <int D, bool kRaster, bool kPadded>
__global__ void __launch_bounds__(kBwThreads, 1)
sta_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const BwdParams p) {
    using C = DkvCfg<D>;
    constexpr int NS = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const uint32_t bar0 = base + C::kBarOff;
    auto st_full = [&](int r) { return bar0 + 8u * r; };
    auto st_empty = [&](int r) { return bar0 + 8u * (NS + r); };
    const uint32_t xb = bar0 + 8u * (2 * NS);
    const uint32_t kv_full = xb, kv_empty = xb + 8, s_full = xb + 16, dp_full = xb + 24, p_full = xb + 32,
                   ds_full = xb + 40, dkv_full = xb + 48, drain = xb + 56;
    const uint32_t item_full0 = xb + 64, item_empty0 = xb + 64 + 8 * kItemQ;
    auto stage = [&](int r) { return base + C::kStageOff + uint32_t(r) * C::kStageBytes; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
    volatile int32_t* item_q = reinterpret_cast<volatile int32_t*>(smem + C::kMiscOff + 8);

    if (threadIdx.x == 0) {
        for (int r = 0; r < NS; ++r) {
            ptx::mbar_init(st_full(r), 1);
            ptx::mbar_init(st_empty(r), 1);
        }
        ptx::mbar_init(kv_full, 1);
        ptx::mbar_init(kv_empty, 1);
        ptx::mbar_init(s_full, 1);
        ptx::mbar_init(dp_full, 1);
        ptx::mbar_init(p_full, kEwWarps);
        ptx::mbar_init(ds_full, kEwWarps);
        ptx::mbar_init(dkv_full, 1);
        ptx::mbar_init(drain, 1);
        for (int q = 0; q < kItemQ; ++q) {
            ptx::mbar_init(item_full0 + 8u * q, 1);
            ptx::mbar_init(item_empty0 + 8u * q, kItemConsumers);
        }
        *abort_flag = 0;
        ptx::fence_barrier_init();
        ptx::fence_proxy_async_smem();
    }
    if (warp == kBwLoadWarp && lane == 0) {
        ptx::prefetch_tensormap(&tm_q);
        ptx::prefetch_tensormap(&tm_k);
        ptx::prefetch_tensormap(&tm_v);
        ptx::prefetch_tensormap(&tm_do);
    }
    if (warp == kBwMmaWarp) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kBwTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int32_t SPT = p.sub_per_tile;

    if (warp == kBwLoadWarp) {
        if (lane == 0) {
            // ------------------------------------------------------------ load
            uint32_t sit = 0, kvc = 0;
            bool ok = true;
            for (uint32_t kq = 0; ok; ++kq) {
                const int32_t u = put_item(kq, item_full0, item_empty0, item_q, abort_flag, p);
                if (u == -2) { ok = false; break; }
                if (u < 0) break;
                const WorkItem w = p.items[u];
                const int32_t ktile = w.qa / SPT;
                const int32_t* off = p.off + int64_t(w.win) * (p.tiles_per_head + 1);
                const int32_t* list = p.ids + off[ktile];
                const int32_t n_qt = off[ktile + 1] - off[ktile];
                if (!wait_bw(kv_empty, (kvc & 1u) ^ 1u, abort_flag, p)) { ok = false; break; }
                ptx::mbar_arrive_expect_tx(kv_full, 2 * C::kBlk);
                load_blk<D, kRaster>(base + C::kKOff, &tm_k, kv_full, p, w.bh, ktile, w.qa - ktile * SPT);
                load_blk<D, kRaster>(base + C::kVOff, &tm_v, kv_full, p, w.bh, ktile, w.qa - ktile * SPT);
                ++kvc;
                for (int32_t qt = 0; ok && qt < n_qt; ++qt) {
                    const int32_t t = __ldg(list + qt);
                    for (int32_t sub = 0; ok && sub < SPT; ++sub) {
                        const int r = int(sit % NS);
                        if (sit >= uint32_t(NS) && !wait_bw(st_empty(r), ((sit / NS) - 1) & 1u, abort_flag, p)) {
                            ok = false;
                            break;
                        }
                        const int32_t row = w.bh * p.tokens + t * p.tile_tokens + sub * 128;
                        ptx::mbar_arrive_expect_tx(st_full(r), C::kStageBytes);
                        load_blk<D, kRaster>(stage(r) + C::kStQ, &tm_q, st_full(r), p, w.bh, t, sub);
                        load_blk<D, kRaster>(stage(r) + C::kStDO, &tm_do, st_full(r), p, w.bh, t, sub);
                        ptx::bulk_load(stage(r) + C::kStL, p.neg_l + row, 512, st_full(r));
                        ptx::bulk_load(stage(r) + C::kStD, p.neg_d + row, 512, st_full(r));
                        ++sit;
                    }
                }
            }
            for (uint32_t it = sit > uint32_t(NS) ? sit - NS : 0u; it < sit; ++it)
                drain_bar(st_full(int(it % NS)), (it / NS) & 1u, p.timeout_ns);
            if (kvc > 0) drain_bar(kv_full, (kvc - 1) & 1u, p.timeout_ns);
        }
    } else if (warp == kBwMmaWarp) {
        if (lane == 0) {
            // ------------------------------------------------------------- MMA
            constexpr uint32_t idesc_s = ptx::idesc_bf16(128, 128, false);
            constexpr uint32_t idesc_acc = ptx::idesc_bf16(128, D, true);
            const uint32_t kaddr = base + C::kKOff, vaddr = base + C::kVOff;
            uint32_t sbase = 0, gs = 0, kvc = 0;
            bool ok = true;
            for (uint32_t kq = 0; ok; ++kq) {
                int32_t u;
                if (!get_item(kq, item_full0, item_q, abort_flag, p, u)) { ok = false; break; }
                ptx::mbar_arrive(item_empty0 + 8u * (kq % kItemQ));
                if (u < 0) break;
                const WorkItem w = p.items[u];
                const int32_t ktile = w.qa / SPT;
                const int32_t* off = p.off + int64_t(w.win) * (p.tiles_per_head + 1);
                const int32_t n = (off[ktile + 1] - off[ktile]) * SPT;
                if (!wait_bw(kv_full, kvc & 1u, abort_flag, p)) { ok = false; break; }
                ++kvc;
                ptx::tc_fence_after();
                // S^T_j = K Q_j^T (waits for stage j)
                auto issue_s = [&](int32_t j) -> bool {
                    const uint32_t it = sbase + uint32_t(j);
                    if (!wait_bw(st_full(int(it % NS)), (it / NS) & 1u, abort_flag, p)) return false;
                    ptx::tc_fence_after();
                    const uint32_t qaddr = stage(int(it % NS)) + C::kStQ;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t coff = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
                        ptx::mma_ss(tmem + C::kColS, ptx::desc_k_sw128(kaddr + coff), ptx::desc_k_sw128(qaddr + coff),
                                    idesc_s, kk > 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(s_full);
                    return true;
                };
                // dP^T_j = V dO_j^T (stage j already waited for by issue_s)
                auto issue_dp = [&](int32_t j) {
                    const uint32_t it = sbase + uint32_t(j);
                    const uint32_t doaddr = stage(int(it % NS)) + C::kStDO;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t coff = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
                        ptx::mma_ss(tmem + C::kColDP, ptx::desc_k_sw128(vaddr + coff),
                                    ptx::desc_k_sw128(doaddr + coff), idesc_s, kk > 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(dp_full);
                };
                ok = issue_s(0);
                if (ok) issue_dp(0);
                for (int32_t j = 0; ok && j < n; ++j) {
                    const uint32_t it = sbase + uint32_t(j);
                    const uint32_t st = stage(int(it % NS));
                    if (!wait_bw(p_full, (gs + uint32_t(j)) & 1u, abort_flag, p)) { ok = false; break; }
                    ptx::tc_fence_after();
                    // dV += P^T_j dO_j
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        ptx::mma_ts(tmem + C::kColDV, tmem + C::kColS + a_col(kk),
                                    ptx::desc_mn_sw128(st + C::kStDO + kk * 16 * 128, kBoxBytes), idesc_acc,
                                    (j > 0 || kk > 0) ? 1u : 0u);
                    // in issue order after dV_j, which reads the P^T this S^T overwrites
                    if (j + 1 < n && !issue_s(j + 1)) { ok = false; break; }
                    if (!wait_bw(ds_full, (gs + uint32_t(j)) & 1u, abort_flag, p)) { ok = false; break; }
                    ptx::tc_fence_after();
                    // dK += dS^T_j Q_j
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        ptx::mma_ts(tmem + C::kColDK, tmem + C::kColDP + a_col(kk),
                                    ptx::desc_mn_sw128(st + C::kStQ + kk * 16 * 128, kBoxBytes), idesc_acc,
                                    (j > 0 || kk > 0) ? 1u : 0u);
                    ptx::mma_commit(st_empty(int(it % NS)));
                    // after dK_j, which reads the dS^T this dP^T overwrites
                    if (j + 1 < n) issue_dp(j + 1);
                }
                if (!ok) break;
                ptx::mma_commit(dkv_full);
                ptx::mma_commit(kv_empty);
                sbase += uint32_t(n);
                gs += uint32_t(n);
            }
            ptx::mma_commit(drain);
            drain_bar(drain, 0, p.timeout_ns);
        }
    } else {
        // ------------------------------------------------------- elementwise
        const int h = warp >> 2;  // query-column half
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_addr = uint32_t((warp & 3) * 32) << 16;
        const uint64_t c2 = ptx::f2(p.scale_log2, p.scale_log2);
        uint32_t gs = 0, sbase = 0, kvc = 0;
        bool ok = true;
        for (uint32_t kq = 0; ok; ++kq) {
            int32_t u = -1;
            if (!__all_sync(0xffffffffu, get_item(kq, item_full0, item_q, abort_flag, p, u))) break;
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(item_empty0 + 8u * (kq % kItemQ));
            if (u < 0) break;
            const WorkItem w = p.items[u];
            const int32_t ktile = w.qa / SPT;
            const int32_t* off = p.off + int64_t(w.win) * (p.tiles_per_head + 1);
            const int32_t n = (off[ktile + 1] - off[ktile]) * SPT;
            for (int32_t j = 0; j < n; ++j) {
                const uint32_t step = gs + uint32_t(j), it = sbase + uint32_t(j);
                const int r = int(it % NS);
                // the stage's per-column constants (TMA-written) and the scores
                if (!__all_sync(0xffffffffu, wait_bw(st_full(r), (it / NS) & 1u, abort_flag, p) &&
                                                 wait_bw(s_full, step & 1u, abort_flag, p))) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                // per-column constants, 16-byte broadcast loads
                const float4* cl = reinterpret_cast<const float4*>(smem + (stage(r) - base) + C::kStL) + 16 * h;
                const float4* cd = reinterpret_cast<const float4*>(smem + (stage(r) - base) + C::kStD) + 16 * h;
                const uint32_t ts = tmem + lane_addr + C::kColS + 64u * h;
                float pr[64];
                uint32_t pk[32];
                {
                    uint32_t sr[64];
                    ptx::tmem_ld64(ts, sr);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float4 l = cl[i];
                        float x0, x1, x2, x3;
                        ptx::f2_split(ptx::f2_fma(ptx::f2(__uint_as_float(sr[4 * i]), __uint_as_float(sr[4 * i + 1])),
                                                  c2, ptx::f2(l.x, l.y)),
                                      x0, x1);
                        ptx::f2_split(ptx::f2_fma(ptx::f2(__uint_as_float(sr[4 * i + 2]), __uint_as_float(sr[4 * i + 3])),
                                                  c2, ptx::f2(l.z, l.w)),
                                      x2, x3);
                        pr[4 * i] = ptx::ex2(x0);
                        pr[4 * i + 1] = ptx::ex2(x1);
                        pr[4 * i + 2] = ptx::ex2(x2);
                        pr[4 * i + 3] = ptx::ex2(x3);
                    }
                }
                pack64(pr, pk);
                ptx::tmem_st32(ts, pk);
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(p_full);
                if (!__all_sync(0xffffffffu, wait_bw(dp_full, step & 1u, abort_flag, p))) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t tdp = tmem + lane_addr + C::kColDP + 64u * h;
                {
                    uint32_t dr[64];
                    ptx::tmem_ld64(tdp, dr);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float4 dd = cd[i];
                        float t0, t1, t2, t3;
                        ptx::f2_split(ptx::f2_mul(ptx::f2(pr[4 * i], pr[4 * i + 1]),
                                                  ptx::f2_add(ptx::f2(__uint_as_float(dr[4 * i]),
                                                                      __uint_as_float(dr[4 * i + 1])),
                                                              ptx::f2(dd.x, dd.y))),
                                      t0, t1);
                        ptx::f2_split(ptx::f2_mul(ptx::f2(pr[4 * i + 2], pr[4 * i + 3]),
                                                  ptx::f2_add(ptx::f2(__uint_as_float(dr[4 * i + 2]),
                                                                      __uint_as_float(dr[4 * i + 3])),
                                                              ptx::f2(dd.z, dd.w))),
                                      t2, t3);
                        pk[2 * i] = ptx::pack_bf16x2(t0, t1);
                        pk[2 * i + 1] = ptx::pack_bf16x2(t2, t3);
                    }
                }
                ptx::tmem_st32(tdp, pk);
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ds_full);
            }
            if (!ok) break;
            if (!__all_sync(0xffffffffu, wait_bw(dkv_full, kvc & 1u, abort_flag, p))) break;
            ++kvc;
            ptx::tc_fence_after();
            const int64_t orow = bwd_out_row<kRaster, kPadded>(p, w.bh, w.qa, row);
            const int64_t safe = orow < 0 ? 0 : orow;
            store_cols<D / 2>(tmem + lane_addr + C::kColDV + uint32_t(D / 2) * h, 1.0f,
                              p.out_b + safe * D + (D / 2) * h, orow >= 0);
            store_cols<D / 2>(tmem + lane_addr + C::kColDK + uint32_t(D / 2) * h, p.scale,
                              p.out_a + safe * D + (D / 2) * h, orow >= 0);
            ptx::tc_fence_before();
            gs += uint32_t(n);
            sbase += uint32_t(n);
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kBwMmaWarp) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kBwTmemCols);
    }
}

// ---------------------------------------------------------------- host
using EncodeTiled = PFN_cuTensorMapEncodeTiled_v12000;

cudaError_t encode_fn(EncodeTiled* out) {
    static EncodeTiled fn = nullptr;
    static cudaError_t err = cudaSuccess;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q);
        if (err == cudaSuccess && q != cudaDriverEntryPointSuccess) err = cudaErrorNotSupported;
        fn = reinterpret_cast<EncodeTiled>(f);
    });
    *out = fn;
    return err;
}

// [rows, d] bf16, box 64 x 128, 128-byte swizzle.
cudaError_t make_rows_map(CUtensorMap* m, const void* ptr, int64_t rows, int d) {
    EncodeTiled fn;
    if (cudaError_t e = encode_fn(&fn); e != cudaSuccess) return e;
    cuuint64_t dims[2] = {cuuint64_t(d), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(d) * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The three launches of one (layout, padding) variant.
template <int D, bool kRaster, bool kPadded>
cudaError_t launch_bwd_variant(const sta_plan_s* pl, const CUtensorMap& mq, const CUtensorMap& mk,
                               const CUtensorMap& mv, const CUtensorMap& mdo, BwdParams bp, const void* o,
                               const void* dout, const float* lse, void* dq, void* dk, void* dv, float* ws,
                               int64_t rows, int sms, cudaStream_t stream) {
    const PlanHost& P = pl->h;
    {
        const int64_t threads = rows * (D / 8);
        const int64_t blocks = (threads + 255) / 256;
        // Tile-major tensors of a padded latent: the row pass writes 0 for
        // padding rows instead of reading them (the main kernels need no mask:
        // padding rows of K, V and dO are zero).
        if (!kRaster && P.padded)
            bwd_prep_kernel<D, false, true><<<dim3(uint32_t(blocks)), 256, 0, stream>>>(
                static_cast<const uint4*>(o), static_cast<const uint4*>(dout), lse, ws, ws + rows, rows, bp.tokens,
                bp.rg);
        else
            bwd_prep_kernel<D, kRaster, kPadded><<<dim3(uint32_t(blocks)), 256, 0, stream>>>(
                static_cast<const uint4*>(o), static_cast<const uint4*>(dout), lse, ws, ws + rows, rows, bp.tokens,
                bp.rg);
        if (cudaError_t e = cudaGetLastError(); e != cudaSuccess) return e;
    }
    // dQ
    bp.item_counter = pl->d_counters + pl->launch_seq.fetch_add(1) % uint32_t(kCounterPool);
    if (cudaError_t e = cudaMemsetAsync(bp.item_counter, 0, sizeof(int32_t), stream); e != cudaSuccess) return e;
    bp.items = pl->d_bq_items;
    bp.n_items = int32_t(P.bq_items.size());
    bp.off = pl->d_off;
    bp.ids = pl->d_ids;
    bp.out_a = static_cast<__nv_bfloat16*>(dq);
    bp.out_b = nullptr;
    int grid = bp.n_items < sms ? bp.n_items : sms;
    if (grid <= 0) return cudaSuccess;
    constexpr int kSmemDq = smem_launch(DqCfg<D>::kSmemBytes);
    cudaError_t e = cudaFuncSetAttribute(sta_bwd_dq_kernel<D, kRaster, kPadded>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemDq);
    if (e != cudaSuccess) return e;
    sta_bwd_dq_kernel<D, kRaster, kPadded><<<grid, kBwThreads, kSmemDq, stream>>>(mq, mk, mv, mdo, bp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // dK, dV
    bp.item_counter = pl->d_counters + pl->launch_seq.fetch_add(1) % uint32_t(kCounterPool);
    if ((e = cudaMemsetAsync(bp.item_counter, 0, sizeof(int32_t), stream)) != cudaSuccess) return e;
    bp.items = pl->d_bkv_items;
    bp.n_items = int32_t(P.bkv_items.size());
    bp.off = pl->d_toff;
    bp.ids = pl->d_tids;
    bp.out_a = static_cast<__nv_bfloat16*>(dk);
    bp.out_b = static_cast<__nv_bfloat16*>(dv);
    grid = bp.n_items < sms ? bp.n_items : sms;
    constexpr int kSmemDkv = smem_launch(DkvCfg<D>::kSmemBytes);
    e = cudaFuncSetAttribute(sta_bwd_dkdv_kernel<D, kRaster, kPadded>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemDkv);
    if (e != cudaSuccess) return e;
    sta_bwd_dkdv_kernel<D, kRaster, kPadded><<<grid, kBwThreads, kSmemDkv, stream>>>(mq, mk, mv, mdo, bp);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_bwd_d(const sta_plan_s* pl, const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv, float* ws,
                         float scale, cudaStream_t stream, uint64_t timeout_ns, bool raster) {
    const PlanHost& P = pl->h;
    // tile-major rows (whole tiles): the workspace planes are tile-major in both layouts
    const int64_t rows = int64_t(P.batch) * P.heads * P.tiles_per_head * P.tile_tokens;
    if (rows == 0) return cudaSuccess;
    CUtensorMap mq, mk, mv, mdo;
    cudaError_t e;
    if (raster) {
        const RasterBox rb = raster_box(P.g);
        if (!rb.ok) return cudaErrorInvalidValue;
        EncodeTiled fn;
        if ((e = encode_fn(&fn)) != cudaSuccess) return e;
        const int64_t bh = int64_t(P.batch) * P.heads;
        e = make_raster_map(fn, &mq, q, P.g, bh, D, rb.box_t, rb.box_h);
        if (e == cudaSuccess) e = make_raster_map(fn, &mk, k, P.g, bh, D, rb.box_t, rb.box_h);
        if (e == cudaSuccess) e = make_raster_map(fn, &mv, v, P.g, bh, D, rb.box_t, rb.box_h);
        if (e == cudaSuccess) e = make_raster_map(fn, &mdo, dout, P.g, bh, D, rb.box_t, rb.box_h);
    } else {
        e = make_rows_map(&mq, q, rows, D);
        if (e == cudaSuccess) e = make_rows_map(&mk, k, rows, D);
        if (e == cudaSuccess) e = make_rows_map(&mv, v, rows, D);
        if (e == cudaSuccess) e = make_rows_map(&mdo, dout, rows, D);
    }
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;

    BwdParams bp{};
    bp.tiles_per_head = P.tiles_per_head;
    bp.sub_per_tile = P.sub_per_tile;
    bp.tile_tokens = P.tile_tokens;
    bp.tokens = P.tiles_per_head * P.tile_tokens;
    bp.neg_d = ws;
    bp.neg_l = ws + rows;
    bp.scale = scale;
    bp.scale_log2 = scale * kLog2e;
    bp.status = pl->d_status;
    bp.timeout_ns = timeout_ns;
    bp.rg = raster_geom(pl);
    // the forward lists and their transpose have the same extents
    bp.pb = PlanBounds{int32_t(int64_t(P.batch) * P.heads), P.tiles_per_head, P.sub_per_tile, P.tile_tokens,
                       int32_t(P.win_ext.size() / 3), int32_t(P.csr_ids.size())};
    if (raster)
        return P.padded ? launch_bwd_variant<D, true, true>(pl, mq, mk, mv, mdo, bp, o, dout, lse, dq, dk, dv, ws, rows,
                                                            sms, stream)
                        : launch_bwd_variant<D, true, false>(pl, mq, mk, mv, mdo, bp, o, dout, lse, dq, dk, dv,
                                                             ws, rows, sms, stream);
    return launch_bwd_variant<D, false, false>(pl, mq, mk, mv, mdo, bp, o, dout, lse, dq, dk, dv, ws, rows, sms,
                                               stream);
}

}  // namespace

cudaError_t launch_backward(const sta_plan_s* p, const void* q, const void* k, const void* v, const void* o,
                            const void* dout, const float* lse, void* dq, void* dk, void* dv, float* workspace,
                            int head_dim, float softmax_scale, cudaStream_t stream, uint64_t timeout_ns,
                            bool raster) {
    if (head_dim == 128)
        return launch_bwd_d<128>(p, q, k, v, o, dout, lse, dq, dk, dv, workspace, softmax_scale, stream, timeout_ns,
                                 raster);
    return launch_bwd_d<64>(p, q, k, v, o, dout, lse, dq, dk, dv, workspace, softmax_scale, stream, timeout_ns,
                            raster);
}

}  // namespace sta
