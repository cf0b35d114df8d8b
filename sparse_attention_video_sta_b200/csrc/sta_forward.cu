// sta_forward.cu -- Sliding Tile Attention forward for sm_100a (B200).
//
// Method ("Fast Video Generation with Sliding Tile Attention"): each query tile
// attends, with exact softmax, to the key tiles listed by the plan (a window of
// tiles centred on it); because the window slides tile by tile, every computed
// (query tile, key tile) block is dense and needs no mask (podcast transcript at
// hotaipapers.com, segments on tiles and on dense / empty / mixed blocks).  The
// pages' own kernel splits a thread block into data warpgroups that load K/V and
// manage the sparse tile list, and compute warpgroups doing dense attention math
// (same transcript, segment on ThunderKittens); the kernel below keeps that
// split but is built for Blackwell: one 128-row query block per work item,
// every 128-key chunk split between two softmax warpgroups, S triple buffered
// in TMEM (see the kernel's own comment).
//
// The kernel is persistent (one CTA per SM) over the plan's work list, longest
// key lists first, items handed out at run time.  Every mbarrier wait has a
// time limit; on expiry the kernel records STA timeout status, drains its
// copies and MMAs, frees TMEM and exits.
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

constexpr int kThreads = 384;  // 3 warpgroups: softmax half A, softmax half B, producers
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp0 = 9;  // PV issuer; also allocates TMEM.  S issuer: warp 10.
// Registers per thread: launched at 168 (384 threads, 3 warps per SM
// sub-partition); the producer warpgroup (warps 8-11, warp 11 idle) gives
// registers to the two softmax warpgroups.  128 * (208 + 208 + 88) is within the
// launch's 384 * 168, so the increase never waits on registers that are not there
// (88 keeps the producer code free of spills).
constexpr uint32_t kRegsSoftmax = 208;
constexpr uint32_t kRegsProducer = 88;
static_assert(128 * (2 * kRegsSoftmax + kRegsProducer) <= kThreads * 168, "register split exceeds the launch");
constexpr uint32_t kTmemCols = 512;

// Work items are handed out at run time: the load warp takes the next item
// index from a global counter and passes it to the other roles through a
// queue of this many entries in shared memory.  CTAs that run slower (their
// SM's share of L2 and HBM, their items' tiles) then take fewer items.
constexpr int kItemQ = 4;

struct FwdParams {
    const WorkItem* items;
    int32_t n_items;
    int32_t* item_counter;  // next item to hand out (zeroed before the launch); null: static striding
    const int32_t* off;  // CSR offsets [n_win][tiles + 1]
    const int32_t* ids;  // CSR key-tile ids
    int32_t tiles_per_head;
    int32_t sub_per_tile;  // 128-row blocks (= 128-key chunks) per tile
    int32_t tile_tokens;
    int32_t tokens;  // tile-major rows per (b, h): whole tiles
    __nv_bfloat16* o;
    float* lse;
    float scale_log2;  // softmax_scale * log2(e)
    float scale;
    uint32_t* status;
    uint64_t timeout_ns;
    // Debug: 1 = the load warp's first wait runs out before any copy is
    // issued; 2 = the S issuer's wait at the start of its CTA's second work
    // item runs out, with that item's query block and K/V chunks already
    // issued (copies in flight or landed, nothing consuming them).
    int32_t inject;
    RasterGeom rg;  // raster layout only
    // Padded latents (an axis not a multiple of the tile): real-key bits of
    // every 128-key chunk, [tiles][sub_per_tile] x 4 words; null otherwise.
    const uint4* key_mask;
    PlanBounds pb;  // extents of the plan arrays (checked by the debug build)
};

// Load 128-row block `sub` of tile `tile` of head bh.  Tile-major layout: one
// 2D row coordinate.  Raster layout: the (w, h, t) origin of the block's box
// inside the tile (tile origin from the plan's table), whose rows TMA lays out
// in tile-major order.
// `org`: the tile's raster origin (raster layout only; read ahead by the caller).
template <bool kRaster>
__device__ __forceinline__ void load_block(uint32_t dst, const CUtensorMap* m, uint32_t bar, const FwdParams& p,
                                           int32_t bh, int32_t tile, int4 org, int32_t sub, int col_blocks,
                                           int box_bytes) {
    if (!kRaster) {
        const int32_t row = bh * p.tokens + tile * p.tile_tokens + sub * kSubRows;
        for (int cb = 0; cb < col_blocks; ++cb) ptx::tma_load_2d(dst + cb * box_bytes, m, bar, cb * 64, row);
    } else {
        raster_load_at(dst, m, bar, p.rg, bh, org, sub, col_blocks, box_bytes);
    }
}

// Raster origin of a tile (zeros for the tile-major layout, which has none).
template <bool kRaster>
__device__ __forceinline__ int4 tile_org(const FwdParams& p, int32_t tile) {
    return kRaster ? __ldg(p.rg.tile_origin + tile) : make_int4(0, 0, 0, 0);
}

// Row of the output tensors that holds row `r` of block `blk` of head bh; -1
// for a padding row of a raster output (a token past the latent; kPadded only).
template <bool kRaster, bool kPadded>
__device__ __forceinline__ int64_t out_row(const FwdParams& p, int32_t bh, int32_t blk, int32_t r) {
    if (!kRaster) return int64_t(bh) * p.tokens + int64_t(blk) * kSubRows + r;
    return raster_row<kPadded>(p.rg, bh, blk, r);
}

// Bounded wait with this launch's status word and time limit.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         const FwdParams& p) {
    return wait_bar_limited(bar, parity, abort_flag, p.status, p.timeout_ns);
}

// The same for one 64-score half row (key-split kernel): `lo`, `hi` hold the
// real-key bits of the half's 64 keys.
__device__ __forceinline__ void mask_scores64(uint32_t (&sr)[64], uint32_t lo, uint32_t hi) {
#pragma unroll
    for (int j = 0; j < 64; ++j)
        if (!(((j < 32 ? lo : hi) >> (j & 31)) & 1u)) sr[j] = 0xff800000u;
}

// P = exp2(S * c - m * c) for one 64-score half row, packed to bf16 pairs;
// returns the fp32 sum of the bf16 values, the ones P V multiplies.  Summing
// the rounded values keeps O / l a convex combination of V rows: with the
// unrounded sum, a row dominated by one key whose P rounds by up to 2^-9 (the
// running max is only updated lazily, so that P is rarely exactly 1) would
// carry that rounding into O on top of O's own bf16 rounding.
__device__ __forceinline__ float softmax_exp64(const uint32_t (&sr)[64], float c, float m, uint32_t (&pk)[32]) {
    const uint64_t c2 = ptx::f2(c, c);
    const uint64_t nmc2 = ptx::f2(-m * c, -m * c);
    uint64_t acc0 = ptx::f2(0.0f, 0.0f), acc1 = acc0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const float s0 = __uint_as_float(sr[2 * j]), s1 = __uint_as_float(sr[2 * j + 1]);
        float x0, x1, p0, p1;
        ptx::f2_split(ptx::f2_fma(ptx::f2(s0, s1), c2, nmc2), x0, x1);
        p0 = ptx::ex2(x0);
        p1 = ptx::ex2(x1);
        pk[j] = ptx::pack_bf16x2(p0, p1);
        const uint64_t pr = ptx::f2(__uint_as_float(pk[j] << 16), __uint_as_float(pk[j] & 0xffff0000u));
        if (j & 1)
            acc1 = ptx::f2_add(acc1, pr);
        else
            acc0 = ptx::f2_add(acc0, pr);
    }
    float r0, r1, r2, r3;
    ptx::f2_split(acc0, r0, r1);
    ptx::f2_split(acc1, r2, r3);
    return (r0 + r1) + (r2 + r3);
}

__device__ __forceinline__ float row_max64(const uint32_t (&sr)[64]) {
    float a0 = __uint_as_float(sr[0]), a1 = __uint_as_float(sr[1]);
    float a2 = __uint_as_float(sr[2]), a3 = __uint_as_float(sr[3]);
#pragma unroll
    for (int j = 4; j < 60; j += 8) {
        a0 = ptx::max3(a0, __uint_as_float(sr[j]), __uint_as_float(sr[j + 1]));
        a1 = ptx::max3(a1, __uint_as_float(sr[j + 2]), __uint_as_float(sr[j + 3]));
        a2 = ptx::max3(a2, __uint_as_float(sr[j + 4]), __uint_as_float(sr[j + 5]));
        a3 = ptx::max3(a3, __uint_as_float(sr[j + 6]), __uint_as_float(sr[j + 7]));
    }
    a0 = ptx::max3(a0, __uint_as_float(sr[60]), __uint_as_float(sr[61]));
    a1 = ptx::max3(a1, __uint_as_float(sr[62]), __uint_as_float(sr[63]));
    return ptx::max3(a0, a1, fmaxf(a2, a3));
}

// ---------------------------------------------------------------------------
// Key-split forward kernel.
//
// One work item is one 128-row query block.  Every 128-key chunk is split in
// two halves of 64 keys: softmax warpgroup A (warps 0-3) exponentiates keys
// 0-63 of each chunk, warpgroup B (warps 4-7) keys 64-127, so both halves'
// exponentials run at once, two warps per SM sub-partition, which keeps the
// MUFU pipe busier than one warp can (measured: 0.91 of its rate against
// 0.82).  The two warps that own the same 32 rows (warp w of A, warp w + 4 of
// B) keep one running maximum per row between them, so both halves' P V
// products accumulate into one O; each keeps its own row sum, added in the
// epilogue.  S is triple buffered in TMEM: the S of chunk c + 3 only waits for
// the P V of chunk c, whose P it overwrites, so the tensor pipe runs up to
// three chunks ahead of the softmax.
//
//   warp 8 (load)   : TMA loads of the query block (two buffers: the next
//                     block's query loads while the current one runs) and of
//                     K(0), K(1), K(2), then V(i), K(i + 3) for i = 0, 1, ...
//                     into the ring, the order in which they are consumed
//   warp 9 (PV)     : O += P_A V_A, then O += P_B V_B (keys 64 h .. 64 h + 63
//                     of the chunk) as each half's P lands in TMEM
//   warp 10 (S)     : S(c) = Q K(c)^T into buffer c % 3, once the PVs of chunk
//                     c - 3, which read that buffer, have completed
//   warps 0-7       : softmax halves and the epilogue
//
// TMEM (512 columns): S0 | S1 | S2 | O (d = 128).  P_A (bf16) is written over
// the first 32 columns of its half of S, P_B over the first 32 of its.
//
// Shared running maximum.  A chunk is exponentiated against the row's running
// maximum m without a max pass; the warp pair meets once per chunk on a named
// barrier whose reduction says whether either warp needs the slow path: the
// block's first chunk (m is set from both halves' maxima), a chunk whose
// half-row sum exceeds kRescaleRowSum (m is raised to the maximum of both
// halves' scores, and O and both row sums are rescaled, each half rescaling
// its own half of O's columns), or an abort (both warps leave together, so
// neither is left waiting at a later barrier).  Row sums add the bf16 P values
// (see softmax_exp64).  Padded latents (kPadded): each half masks its padding
// keys from the chunk's real-key bits; a first chunk without a real key in
// either half starts from a finite stand-in maximum of 0, which the rescale
// moves once real keys arrive.
namespace split {

constexpr int kItemConsumers = 2 + 8;  // the two issuing threads and the eight softmax warps
constexpr int kSBufs = 3;              // S buffers in TMEM
// A half-row sum above this (the scores grew far past the running maximum,
// or an exponential overflowed) takes the slow path.  The sums add bf16 P
// values, whose rounding is relative, so P far above 1 costs no accuracy;
// the bound only keeps O and l far from fp32 overflow.
constexpr float kRescaleRowSum = 65536.0f;

template <int D>
struct Cfg {
    static constexpr int kColBlocks = D / 64;
    static constexpr int kBoxBytes = 128 * 128;
    static constexpr int kQBytes = kSubRows * D * 2;
    static constexpr int kKVBytes = kChunkKeys * D * 2;
    static constexpr int kStages = (D == 128) ? 5 : 8;
    static constexpr int kQOff = 0;
    static constexpr int kRingOff = 2 * kQBytes;
    static constexpr int kBarOff = kRingOff + kStages * kKVBytes;
    // full[S], empty[S], q_full[2], q_empty[2], s_full[3], p_full[2][3], pv_buf[3],
    // o_full, o_empty, dead, drain[2], item_full[Q], item_empty[Q]
    static constexpr int kNumBars = 2 * kStages + 2 + 2 + kSBufs + 2 * kSBufs + kSBufs + 1 + 1 + 1 + 2 +
                                    2 * kItemQ;
    static constexpr int kXchOff = kBarOff + kNumBars * 8;  // [2 halves][128 rows] fp32 exchange
    static constexpr int kMiscOff = kXchOff + 2 * kSubRows * 4;  // tmem base slot, abort flag, item queue
    static constexpr int kSmemBytes = kMiscOff + 8 + 4 * kItemQ + 1024;
    __host__ __device__ static constexpr uint32_t col_s(int buf) { return uint32_t(buf) * 128u; }
    static constexpr uint32_t kColO = kSBufs * 128u;
    static_assert(kSBufs * 128 + D <= int(kTmemCols), "TMEM budget");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

// kPadded: the latent has padding tokens; padding keys are masked per chunk
// and raster padding rows are not stored.
template <int D, bool kRaster, bool kPadded>
__global__ void __launch_bounds__(kThreads, 1)
sta_fwd_split_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const uint32_t bar0 = base + C::kBarOff;
    constexpr int S = C::kStages;
    constexpr int NB = kSBufs;
    auto bar_full = [&](int r) { return bar0 + 8u * r; };
    auto bar_empty = [&](int r) { return bar0 + 8u * (S + r); };
    auto bar_q_full = [&](int b) { return bar0 + 8u * (2 * S + b); };
    auto bar_q_empty = [&](int b) { return bar0 + 8u * (2 * S + 2 + b); };
    auto bar_s_full = [&](int b) { return bar0 + 8u * (2 * S + 4 + b); };
    auto bar_p_full = [&](int h, int b) { return bar0 + 8u * (2 * S + 4 + NB + NB * h + b); };
    auto bar_pv_buf = [&](int b) { return bar0 + 8u * (2 * S + 4 + 3 * NB + b); };
    const uint32_t bar_o_full = bar0 + 8u * (2 * S + 4 + 4 * NB);
    const uint32_t bar_o_empty = bar0 + 8u * (2 * S + 5 + 4 * NB);
    const uint32_t bar_dead = bar0 + 8u * (2 * S + 6 + 4 * NB);
    auto bar_drain = [&](int h) { return bar0 + 8u * (2 * S + 7 + 4 * NB + h); };
    auto bar_item_full = [&](int q) { return bar0 + 8u * (2 * S + 9 + 4 * NB + q); };
    auto bar_item_empty = [&](int q) { return bar0 + 8u * (2 * S + 9 + 4 * NB + kItemQ + q); };
    static_assert(2 * S + 9 + 4 * NB + 2 * kItemQ == C::kNumBars, "barrier count");
    float* xch = reinterpret_cast<float*>(smem + C::kXchOff);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
    volatile int32_t* item_q = reinterpret_cast<volatile int32_t*>(smem + C::kMiscOff + 8);
    auto take_item = [&](uint32_t k, int32_t& u) -> bool {
        const int q = int(k % kItemQ);
        if (!wait_bar(bar_item_full(q), (k / kItemQ) & 1u, abort_flag, p)) return false;
        u = item_q[q];
        return true;
    };

    if (threadIdx.x == 0) {
        for (int r = 0; r < S; ++r) {
            ptx::mbar_init(bar_full(r), 1);
            ptx::mbar_init(bar_empty(r), 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(bar_q_full(b), 1);
            ptx::mbar_init(bar_q_empty(b), 1);  // the block's last S products completed
            ptx::mbar_init(bar_drain(b), 1);
        }
        for (int b = 0; b < NB; ++b) {
            ptx::mbar_init(bar_s_full(b), 1);
            ptx::mbar_init(bar_p_full(0, b), 4);  // one arrival per softmax warp of the half
            ptx::mbar_init(bar_p_full(1, b), 4);
            ptx::mbar_init(bar_pv_buf(b), 1);
        }
        ptx::mbar_init(bar_o_full, 1);
        ptx::mbar_init(bar_o_empty, 8);
        ptx::mbar_init(bar_dead, 1);
        for (int q = 0; q < kItemQ; ++q) {
            ptx::mbar_init(bar_item_full(q), 1);
            ptx::mbar_init(bar_item_empty(q), kItemConsumers);
        }
        *abort_flag = 0;
        ptx::fence_barrier_init();
        ptx::fence_proxy_async_smem();
    }
    if (warp == kLoadWarp && lane == 0) {
        ptx::prefetch_tensormap(&tm_q);
        ptx::prefetch_tensormap(&tm_k);
        ptx::prefetch_tensormap(&tm_v);
    }
    if (warp == kMmaWarp0) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int32_t SPT = p.sub_per_tile;

    if (warp == kLoadWarp) {
        ptx::regs_dec<kRegsProducer>();
        if (lane == 0) {
            // ------------------------------------------------------------ load
            // Ring entries in the order the issuing threads consume them: per
            // block, K(0), K(1), K(2), then V(i), K(i + 3) for i = 0, 1, ...
            uint32_t ring = 0;
            uint32_t q_loads[2] = {0u, 0u};  // query loads issued into each buffer
            bool ok = true;
            if (p.inject == 1) ok = wait_bar(bar_dead, 0, abort_flag, p);
            auto issue = [&](const CUtensorMap* m, int32_t bh, int32_t tile, int4 org, int32_t sub) -> bool {
                const int r = int(ring % S);
                if (ring >= uint32_t(S) && !wait_bar(bar_empty(r), ((ring / S) - 1) & 1u, abort_flag, p))
                    return false;
                ptx::mbar_arrive_expect_tx(bar_full(r), C::kKVBytes);
                load_block<kRaster>(base + C::kRingOff + r * C::kKVBytes, m, bar_full(r), p, bh, tile, org, sub,
                                    C::kColBlocks, C::kBoxBytes);
                ++ring;
                return true;
            };
            for (uint32_t k = 0; ok; ++k) {
                int32_t u = p.item_counter != nullptr ? atomicAdd(p.item_counter, 1)
                                                      : int32_t(blockIdx.x + k * gridDim.x);
                if (u >= p.n_items) u = -1;
                if (kDebugBounds && u >= 0 && !item_in_bounds(p.items, p.n_items, u, p.off, p.ids, p.pb, p.status)) {
                    *abort_flag = 1;  // no more items: every role leaves its loop
                    u = -1;
                }
                const int qe = int(k % kItemQ);
                if (k >= uint32_t(kItemQ) &&
                    !wait_bar(bar_item_empty(qe), ((k / kItemQ) - 1) & 1u, abort_flag, p)) {
                    ok = false;
                    break;
                }
                item_q[qe] = u;
                ptx::mbar_arrive(bar_item_full(qe));
                if (u < 0) break;
                const WorkItem w = p.items[u];
                const int32_t tile_q = w.qa / SPT;
                const int32_t* off = p.off + int64_t(w.win) * (p.tiles_per_head + 1);
                const int32_t* list = p.ids + off[tile_q];
                const int32_t n = (off[tile_q + 1] - off[tile_q]) * SPT;
                // query block into buffer k % 2 (free once block k - 2's S products completed)
                const int qb = int(k & 1u);
                if (!wait_bar(bar_q_empty(qb), ((k >> 1) & 1u) ^ 1u, abort_flag, p)) { ok = false; break; }
                ptx::mbar_arrive_expect_tx(bar_q_full(qb), C::kQBytes);
                load_block<kRaster>(base + C::kQOff + qb * C::kQBytes, &tm_q, bar_q_full(qb), p, w.bh, tile_q,
                                    tile_org<kRaster>(p, tile_q), w.qa - tile_q * SPT, C::kColBlocks, C::kBoxBytes);
                ++q_loads[qb];
                // chunk c of the list is block c % SPT of key tile list[c / SPT]
                auto load_chunk = [&](const CUtensorMap* m, int32_t c) -> bool {
                    const int32_t kt = __ldg(list + c / SPT);
                    return issue(m, w.bh, kt, tile_org<kRaster>(p, kt), c % SPT);
                };
                for (int32_t c = 0; ok && c < n && c < NB; ++c) ok = load_chunk(&tm_k, c);
                for (int32_t i = 0; ok && i < n; ++i) {
                    ok = load_chunk(&tm_v, i);
                    if (ok && i + NB < n) ok = load_chunk(&tm_k, i + NB);
                }
            }
            // Drain before exit (after an abort some copies may still be in
            // flight): the last copy into each ring stage and the last query
            // block loaded into each buffer.
            const uint32_t first = ring > uint32_t(S) ? ring - S : 0u;
            for (uint32_t it = first; it < ring; ++it)
                drain_bar(bar_full(int(it % S)), (it / S) & 1u, p.timeout_ns);
            for (int b = 0; b < 2; ++b)
                if (q_loads[b] > 0) drain_bar(bar_q_full(b), (q_loads[b] - 1u) & 1u, p.timeout_ns);
        }
    } else if (warp == kMmaWarp0 + 2) {
        ptx::regs_dec<kRegsProducer>();  // idle: completes the producer warpgroup for the register hand-over
    } else if (warp == kMmaWarp0 || warp == kMmaWarp0 + 1) {
        ptx::regs_dec<kRegsProducer>();
        if (lane == 0) {
            // ------------------------------------------------------------- MMA
            // Two issuing threads.  Warp 9 issues O += P_h V_h as soon as a
            // half's P is in TMEM; warp 10 issues S = Q K^T for chunk c + 3 once
            // both PVs of chunk c (which read the S buffer S(c + 3) overwrites)
            // have completed.  A tcgen05.mma issue holds its thread until the
            // pipe takes it, so with one thread for both kinds the P hand-off
            // waited behind the previous step's S batch.
            const bool pv_role = warp == kMmaWarp0;
            constexpr uint32_t idesc_qk = ptx::idesc_bf16(128, kChunkKeys, false);
            constexpr uint32_t idesc_pv = ptx::idesc_bf16(128, D, true);
            uint32_t e0 = 0, g = 0;  // ring entries and chunks of the blocks before this one
            bool ok = true;
            // Ring entry of chunk c's K and V in a block of n chunks (the load
            // order: K(0), K(1), K(2), then V(i), K(i + 3) for i = 0, 1, ...).
            auto entry_k = [](uint32_t c) { return c < uint32_t(NB) ? c : 2u * c - uint32_t(NB - 1); };
            auto entry_v = [](uint32_t i, uint32_t n) {
                return i + uint32_t(NB) <= n ? uint32_t(NB) + 2u * i : n + i;
            };
            auto wait_entry = [&](uint32_t e, uint32_t& addr) -> bool {
                const int r = int(e % S);
                if (!wait_bar(bar_full(r), (e / S) & 1u, abort_flag, p)) return false;
                addr = base + C::kRingOff + r * C::kKVBytes;
                return true;
            };
            for (uint32_t kq = 0; ok; ++kq) {
                int32_t u;
                if (!take_item(kq, u)) { ok = false; break; }
                ptx::mbar_arrive(bar_item_empty(int(kq % kItemQ)));
                if (u < 0) break;
                const WorkItem w = p.items[u];
                const int32_t tile_q = w.qa / SPT;
                const int32_t* off = p.off + int64_t(w.win) * (p.tiles_per_head + 1);
                const uint32_t n = uint32_t(off[tile_q + 1] - off[tile_q]) * uint32_t(SPT);
                const uint32_t g0 = g;
                if (pv_role) {
                    const uint32_t tO = tmem + C::kColO;
                    for (uint32_t i = 0; ok && i < n; ++i) {
                        const uint32_t gi = g0 + i, bb = gi % uint32_t(NB), e = e0 + entry_v(i, n);
                        uint32_t vaddr;
                        if (!wait_entry(e, vaddr)) { ok = false; break; }
                        if (i == 0 && !wait_bar(bar_o_empty, (kq & 1u) ^ 1u, abort_flag, p)) { ok = false; break; }
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            // O += P_h(gi) V_h(gi): keys 64 h .. 64 h + 63 of the chunk
                            if (!wait_bar(bar_p_full(h, int(bb)), (gi / uint32_t(NB)) & 1u, abort_flag, p)) {
                                ok = false;
                                break;
                            }
                            ptx::tc_fence_after();
                            const uint32_t tP = tmem + C::col_s(int(bb)) + uint32_t(h) * 64u;
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                ptx::mma_ts(tO, tP + kk * 8,
                                            ptx::desc_mn_sw128(vaddr + (h * 4 + kk) * 16 * 128, C::kBoxBytes),
                                            idesc_pv, (i > 0 || h > 0 || kk > 0) ? 1u : 0u);
                        }
                        if (!ok) break;
                        ptx::mma_commit(bar_pv_buf(int(bb)));  // S buffer bb is free again; O holds P(.. gi) V
                        ptx::mma_commit(bar_empty(int(e % S)));
                    }
                    if (!ok) break;
                    ptx::mma_commit(bar_o_full);
                } else {
                    const int qb = int(kq & 1u);
                    const uint32_t qaddr = base + C::kQOff + qb * C::kQBytes;
                    if (p.inject == 2 && kq == 1u) {
                        // Debug: wait on a barrier nothing arrives at; the limit runs out
                        // while this item's loads are issued and nothing consumes them.
                        wait_bar(bar_dead, 0, abort_flag, p);
                        ok = false;
                        break;
                    }
                    if (!wait_bar(bar_q_full(qb), (kq >> 1) & 1u, abort_flag, p)) { ok = false; break; }
                    for (uint32_t c = 0; ok && c < n; ++c) {
                        const uint32_t gc = g0 + c, bb = gc % uint32_t(NB), e = e0 + entry_k(c);
                        // S(gc) overwrites buffer bb, read by the PVs of chunk gc - 3
                        if (gc >= uint32_t(NB) &&
                            !wait_bar(bar_pv_buf(int(bb)), ((gc / uint32_t(NB)) - 1u) & 1u, abort_flag, p)) {
                            ok = false;
                            break;
                        }
                        uint32_t kaddr;
                        if (!wait_entry(e, kaddr)) { ok = false; break; }
                        ptx::tc_fence_after();
                        const uint32_t tS = tmem + C::col_s(int(bb));
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t coff = (kk >> 2) * C::kBoxBytes + (kk & 3) * 32;
                            ptx::mma_ss(tS, ptx::desc_k_sw128(qaddr + coff), ptx::desc_k_sw128(kaddr + coff),
                                        idesc_qk, kk > 0 ? 1u : 0u);
                        }
                        ptx::mma_commit(bar_s_full(int(bb)));
                        ptx::mma_commit(bar_empty(int(e % S)));
                    }
                    if (!ok) break;
                    ptx::mma_commit(bar_q_empty(qb));  // the query buffer is free once these S products complete
                }
                g = g0 + n;
                e0 += 2u * n;
            }
            const int dr = pv_role ? 0 : 1;
            ptx::mma_commit(bar_drain(dr));
            drain_bar(bar_drain(dr), 0, p.timeout_ns);
        }
    } else {
        // ------------------------------------------------------------- softmax
        ptx::regs_inc<kRegsSoftmax>();
        const int half = warp >> 2;  // 0: keys 0-63 of every chunk, 1: keys 64-127
        const int row = threadIdx.x & 127;
        const uint32_t pair_bar = 1u + uint32_t(warp & 3);  // named barrier of warps w and w + 4
        const uint32_t lane_addr = uint32_t((warp & 3) * 32) << 16;
        const uint32_t tOh = tmem + lane_addr + C::kColO + uint32_t(half) * (D / 2);  // this half's O columns
        float* x_mine = xch + half * kSubRows + row;
        const float* x_other = xch + (1 - half) * kSubRows + row;
        const float c = p.scale_log2;
        uint32_t g = 0;
        bool ok = true;
        for (uint32_t kq = 0; ok; ++kq) {
            int32_t u = -1;
            const bool took = __all_sync(0xffffffffu, take_item(kq, u));
            __syncwarp();
            if (took && lane == 0) ptx::mbar_arrive(bar_item_empty(int(kq % kItemQ)));
            if (ptx::bar_red_or(pair_bar, 64, !took)) {  // leave together
                ok = false;
                break;
            }
            if (u < 0) break;
            const WorkItem w = p.items[u];
            const int32_t tile_q = w.qa / SPT;
            const int32_t* off = p.off + int64_t(w.win) * (p.tiles_per_head + 1);
            const uint32_t n = uint32_t(off[tile_q + 1] - off[tile_q]) * uint32_t(SPT);
            const int32_t kbeg = off[tile_q];  // this block's key tiles (padded latents: their masks)
            float m_used = 0.0f, l = 0.0f;
            // The scores of the next chunk are loaded while this chunk's P is
            // stored and handed over (`pre`: sr already holds S(g)).
            uint32_t sr[64];
            bool pre = false;
            for (uint32_t i = 0; i < n; ++i, ++g) {
                const uint32_t b = g % uint32_t(NB), b1 = (g + 1u) % uint32_t(NB);
                const uint32_t tS = tmem + lane_addr + C::col_s(int(b)) + uint32_t(half) * 64u;
                const uint32_t tS1 = tmem + lane_addr + C::col_s(int(b1)) + uint32_t(half) * 64u;
                bool wok = true;
                if (!pre) {
                    wok = __all_sync(0xffffffffu,
                                     wait_bar(bar_s_full(int(b)), (g / uint32_t(NB)) & 1u, abort_flag, p));
                    if (wok) {
                        ptx::tc_fence_after();
                        ptx::tmem_ld64(tS, sr);
                    }
                }
                pre = false;
                uint32_t mlo = ~0u, mhi = ~0u;  // real-key bits of this half's 64 keys
                if (kPadded) {
                    const uint4 m4 = __ldg(p.key_mask + int64_t(__ldg(p.ids + kbeg + int32_t(i) / SPT)) * SPT +
                                           int32_t(i) % SPT);
                    mlo = half == 0 ? m4.x : m4.z;
                    mhi = half == 0 ? m4.y : m4.w;
                }
                if (wok && kPadded && (mlo & mhi) != ~0u) mask_scores64(sr, mlo, mhi);  // warp-uniform
                // Is S(g + 1) of this block complete?  If so, its load starts
                // right after the exponentials and overlaps the P hand-over.
                const bool can_pre = wok && i > 0 && i + 1 < n;
                const bool t_next =
                    can_pre && ptx::mbar_test_wait(bar_s_full(int(b1)), ((g + 1u) / uint32_t(NB)) & 1u);
                uint32_t pk[32];
                float rowsum = 0.0f;
                bool need = false;
                if (wok && i > 0) {
                    // Exponentiate against the running max (no max pass).
                    rowsum = softmax_exp64(sr, c, m_used, pk);
                    need = !(rowsum <= kRescaleRowSum);  // also catches inf
                }
                const bool nxt = can_pre && __all_sync(0xffffffffu, t_next);
                if (nxt) {
                    ptx::tc_fence_after();
                    ptx::tmem_ld64_start(tS1, sr);
                }
                if (ptx::bar_red_or(pair_bar, 64, !wok || need || i == 0)) {
                    // ---- slow path: the block's first chunk, a rescale, or an abort.
                    // Both warps of the pair take it, exchange this chunk's
                    // maxima of their rows and agree on the new running max.
                    if (nxt) {
                        ptx::tmem_wait_ld(sr);
                        ptx::tmem_ld64(tS, sr);  // S(g) again: P(g) is not stored yet
                        if (kPadded && (mlo & mhi) != ~0u) mask_scores64(sr, mlo, mhi);
                    }
                    *x_mine = wok ? row_max64(sr) : -INFINITY;
                    if (ptx::bar_red_or(pair_bar, 64, !wok)) {
                        ok = false;
                        break;
                    }
                    const float mx = fmaxf(*x_mine, *x_other);
                    float alpha = 1.0f;
                    if (i == 0) {
                        // padded latents: a first chunk without a real key in this
                        // row's window takes a finite stand-in, moved later
                        m_used = mx == -INFINITY ? 0.0f : mx;
                    } else if ((mx - m_used) * c > 0.0f) {
                        alpha = ptx::ex2((m_used - mx) * c);
                        m_used = mx;
                    }
                    rowsum = softmax_exp64(sr, c, m_used, pk);
                    ptx::tmem_st32(tS, pk);
                    l = l * alpha + rowsum;
                    bool pv_ok = true;
                    if (i > 0) {
                        // O holds P(.. g - 1) V: wait for PV(g - 1), the one that
                        // may still run, then rescale this half's columns of O.
                        // Its buffer's barrier is at most one phase behind here
                        // (S(g) waited for PV(g - 3)), so the parity wait is exact.
                        const uint32_t gp = g - 1u;
                        pv_ok = __all_sync(0xffffffffu, wait_bar(bar_pv_buf(int(gp % uint32_t(NB))),
                                                                 (gp / uint32_t(NB)) & 1u, abort_flag, p));
                        if (pv_ok && __any_sync(0xffffffffu, alpha != 1.0f)) {
                            ptx::tc_fence_after();
                            const uint64_t alpha2 = ptx::f2(alpha, alpha);
#pragma unroll 1
                            for (int cb = 0; cb < D / 64; ++cb) {
                                uint32_t orr[32];
                                ptx::tmem_ld32(tOh + cb * 32, orr);
#pragma unroll
                                for (int j = 0; j < 16; ++j) {
                                    float o0, o1;
                                    ptx::f2_split(ptx::f2_mul(ptx::f2(__uint_as_float(orr[2 * j]),
                                                                      __uint_as_float(orr[2 * j + 1])), alpha2),
                                                  o0, o1);
                                    orr[2 * j] = __float_as_uint(o0);
                                    orr[2 * j + 1] = __float_as_uint(o1);
                                }
                                ptx::tmem_st32(tOh + cb * 32, orr);
                            }
                        }
                    }
                    ptx::tmem_wait_st();
                    ptx::tc_fence_before();
                    // both halves' rescales of O are done before either half's P is signalled
                    if (ptx::bar_red_or(pair_bar, 64, !pv_ok)) {
                        ok = false;
                        break;
                    }
                    if (nxt) ptx::tmem_ld64(tS1, sr);  // S(g + 1) again
                } else {
                    ptx::tmem_st32(tS, pk);
                    l += rowsum;
                    ptx::tmem_wait_st();
                    ptx::tc_fence_before();
                    if (nxt) ptx::tmem_wait_ld(sr);
                }
                pre = nxt;
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar_p_full(half, int(b)));
            }
            if (!ok) break;
            // ---- epilogue: O / (l_A + l_B) -> bf16, LSE.  Each half stores its
            // half of the columns.
            const bool ook = __all_sync(0xffffffffu, wait_bar(bar_o_full, kq & 1u, abort_flag, p));
            *x_mine = l;
            if (ptx::bar_red_or(pair_bar, 64, !ook)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const float l_sum = l + *x_other;
            const float inv_l = 1.0f / l_sum;
            const uint64_t f2inv = ptx::f2(inv_l, inv_l);
            const int64_t grow = out_row<kRaster, kPadded>(p, w.bh, w.qa, row);
            uint4* dst = reinterpret_cast<uint4*>(p.o + (grow < 0 ? 0 : grow) * D + half * (D / 2));
#pragma unroll 1
            for (int cb = 0; cb < D / 64; ++cb) {
                uint32_t orr[32];
                ptx::tmem_ld32(tOh + cb * 32, orr);  // every lane loads: the access is warp-wide
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    float o0, o1;
                    ptx::f2_split(ptx::f2_mul(ptx::f2(__uint_as_float(orr[2 * j]), __uint_as_float(orr[2 * j + 1])),
                                              f2inv),
                                  o0, o1);
                    pk[j] = ptx::pack_bf16x2(o0, o1);
                }
                if (grow >= 0) {  // a padding row of a raster output stores nothing
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        dst[cb * 4 + j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                }
            }
            if (half == 0 && grow >= 0) p.lse[grow] = m_used * p.scale + logf(l_sum);
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar_o_empty);
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp0) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace split

struct EncodeFn {
    PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    cudaError_t err = cudaSuccess;
};

const EncodeFn& encode_fn() {
    static EncodeFn e;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        e.err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q);
        if (e.err == cudaSuccess && q != cudaDriverEntryPointSuccess) e.err = cudaErrorNotSupported;
        e.fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return e;
}

// 2D map over a [rows, d] bf16 matrix: box of 64 elements (128 bytes) x 128 rows,
// 128-byte swizzle (the layout the tcgen05 shared-memory descriptors expect).
cudaError_t make_map(CUtensorMap* m, const void* ptr, int64_t rows, int d) {
    const EncodeFn& e = encode_fn();
    if (e.err != cudaSuccess) return e.err;
    cuuint64_t dims[2] = {cuuint64_t(d), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(d) * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = e.fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
                      estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D, bool kRaster, bool kPadded>
cudaError_t launch_split_kernel(int grid, cudaStream_t stream, const CUtensorMap& mq, const CUtensorMap& mk,
                                const CUtensorMap& mv, const FwdParams& fp) {
    constexpr int kSmem = split::Cfg<D>::kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(split::sta_fwd_split_kernel<D, kRaster, kPadded>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    split::sta_fwd_split_kernel<D, kRaster, kPadded><<<grid, kThreads, kSmem, stream>>>(mq, mk, mv, fp);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const sta_plan_s* pl, const void* q, const void* k, const void* v, void* o,
                     float* lse, float scale, cudaStream_t stream, int inject, uint64_t timeout_ns,
                     bool raster) {
    const PlanHost& P = pl->h;
    const int64_t bh = int64_t(P.batch) * P.heads;
    const int64_t rows = bh * P.tiles_per_head * P.tile_tokens;
    const RasterBox rb = raster_box(P.g);
    if (raster && !rb.ok) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv;
    cudaError_t e;
    if (raster) {
        const EncodeFn& ef = encode_fn();
        if (ef.err != cudaSuccess) return ef.err;
        e = make_raster_map(ef.fn, &mq, q, P.g, bh, D, rb.box_t, rb.box_h);
        if (e == cudaSuccess) e = make_raster_map(ef.fn, &mk, k, P.g, bh, D, rb.box_t, rb.box_h);
        if (e == cudaSuccess) e = make_raster_map(ef.fn, &mv, v, P.g, bh, D, rb.box_t, rb.box_h);
    } else {
        e = make_map(&mq, q, rows, D);
        if (e == cudaSuccess) e = make_map(&mk, k, rows, D);
        if (e == cudaSuccess) e = make_map(&mv, v, rows, D);
    }
    if (e != cudaSuccess) return e;
    // One-block work items, longest key lists first.
    FwdParams fp{};
    fp.items = pl->d_f1_items;
    fp.n_items = int32_t(P.f1_items.size());
    fp.off = pl->d_off;
    fp.ids = pl->d_ids;
    fp.tiles_per_head = P.tiles_per_head;
    fp.sub_per_tile = P.sub_per_tile;
    fp.tile_tokens = P.tile_tokens;
    fp.tokens = P.tiles_per_head * P.tile_tokens;
    fp.o = static_cast<__nv_bfloat16*>(o);
    fp.lse = lse;
    fp.scale = scale;
    fp.scale_log2 = scale * 1.4426950408889634f;
    fp.status = pl->d_status;
    fp.timeout_ns = timeout_ns;
    fp.inject = inject;
    fp.rg = raster_geom(pl);
    fp.key_mask = reinterpret_cast<const uint4*>(pl->d_kmask);
    fp.pb = PlanBounds{int32_t(bh), P.tiles_per_head, P.sub_per_tile, P.tile_tokens,
                       int32_t(P.win_ext.size() / 3), int32_t(P.csr_ids.size())};
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int grid = fp.n_items < sms ? fp.n_items : sms;
    if (grid <= 0) return cudaSuccess;
    fp.item_counter = pl->d_counters + pl->launch_seq.fetch_add(1) % uint32_t(kCounterPool);
    if ((e = cudaMemsetAsync(fp.item_counter, 0, sizeof(int32_t), stream)) != cudaSuccess) return e;
    if (raster)
        return P.padded ? launch_split_kernel<D, true, true>(grid, stream, mq, mk, mv, fp)
                        : launch_split_kernel<D, true, false>(grid, stream, mq, mk, mv, fp);
    return P.padded ? launch_split_kernel<D, false, true>(grid, stream, mq, mk, mv, fp)
                    : launch_split_kernel<D, false, false>(grid, stream, mq, mk, mv, fp);
}

}  // namespace

RasterBox raster_box(const sta_geom& g) {
    RasterBox rb{0, 0, 0, false};
    const int32_t hw = g.tile_h * g.tile_w;
    if (hw <= 0 || g.tile_w > 256 || g.tile_w > g.lat_w) return rb;
    if (kSubRows % hw == 0) {  // a block is whole (h, w) slices: box_t of them
        rb.box_t = kSubRows / hw;
        rb.box_h = g.tile_h;
        rb.blocks_per_slice = 1;
        rb.ok = g.tile_h <= 256 && g.tile_t % rb.box_t == 0 && rb.box_t <= g.lat_t && rb.box_h <= g.lat_h;
    } else if (hw % kSubRows == 0 && kSubRows % g.tile_w == 0) {  // a block is part of one slice
        rb.box_t = 1;
        rb.box_h = kSubRows / g.tile_w;
        rb.blocks_per_slice = hw / kSubRows;
        rb.ok = rb.box_h <= g.lat_h;  // boxes never wider than the latent (edge boxes read past it: zero fill)
    }
    return rb;
}

cudaError_t launch_forward(const sta_plan_s* p, const void* q, const void* k, const void* v, void* o,
                           float* lse, int head_dim, float softmax_scale, cudaStream_t stream,
                           int inject_timeout, uint64_t timeout_ns, bool raster) {
    if (head_dim == 128)
        return launch_d<128>(p, q, k, v, o, lse, softmax_scale, stream, inject_timeout, timeout_ns, raster);
    return launch_d<64>(p, q, k, v, o, lse, softmax_scale, stream, inject_timeout, timeout_ns, raster);
}

cudaError_t launch_forward_raw(const RawPlanView& pv, const void* q, const void* k, const void* v,
                               void* o, float* lse, int head_dim, float softmax_scale,
                               cudaStream_t stream) {
    const int64_t rows = int64_t(pv.batch) * pv.heads * pv.tiles_per_head * pv.tile_tokens;
    CUtensorMap mq, mk, mv;
    cudaError_t e = make_map(&mq, q, rows, head_dim);
    if (e == cudaSuccess) e = make_map(&mk, k, rows, head_dim);
    if (e == cudaSuccess) e = make_map(&mv, v, rows, head_dim);
    if (e != cudaSuccess) return e;
    FwdParams fp{};
    fp.items = pv.items;
    fp.n_items = pv.n_items;
    fp.item_counter = pv.item_counter;
    fp.off = pv.off;
    fp.ids = pv.ids;
    fp.tiles_per_head = pv.tiles_per_head;
    fp.sub_per_tile = pv.sub_per_tile;
    fp.tile_tokens = pv.tile_tokens;
    fp.tokens = pv.tiles_per_head * pv.tile_tokens;
    fp.o = static_cast<__nv_bfloat16*>(o);
    fp.lse = lse;
    fp.scale = softmax_scale;
    fp.scale_log2 = softmax_scale * 1.4426950408889634f;
    fp.status = pv.status;
    fp.timeout_ns = pv.timeout_ns;
    fp.inject = 0;
    fp.pb = PlanBounds{pv.batch * pv.heads, pv.tiles_per_head, pv.sub_per_tile, pv.tile_tokens, pv.n_win, pv.n_ids};
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int grid = fp.n_items < sms ? fp.n_items : sms;
    if (grid <= 0) return cudaSuccess;
    if (head_dim == 128) return launch_split_kernel<128, false, false>(grid, stream, mq, mk, mv, fp);
    return launch_split_kernel<64, false, false>(grid, stream, mq, mk, mv, fp);
}

}  // namespace sta
