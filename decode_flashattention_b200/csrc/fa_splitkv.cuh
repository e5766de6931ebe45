// fa_splitkv.cuh -- split-KV decode / small-Q attention kernel (both variants).
//
// One CTA per SM.  Its producer warp walks the CTA's piece of the key-tile
// space (the Partition in fa_common.cuh) and feeds a ring of STAGES
// shared-memory stages: per tile it issues TMA loads of K and V (128 keys x 64
// elements per box, 128-byte swizzle, no multicast); at the first tile of a
// unit's segment it also copies that unit's 8 packed query rows into the
// stage's Q slot with cp.async, tracked by the same barrier; and it publishes
// the tile's coordinates in the stage header.  (K-outer blocking with the next
// tiles prefetched while the current one is consumed: "SmallQ FlashAttention
// for Ascend 910B", section "算法要点"; the CSDN "FlashAttention on Ascend
// CANN" post, section on pipelining HBM prefetch with compute.)
//
// The four consumer warps take 32 of the 128 keys of each tile.  Two ways to
// do the products, chosen at compile time (FMA):
//  - tensor cores (FMA = false): S^T = K Q^T with mma.sync m16n8k16 (keys as
//    M, the 8 packed query rows as N, fp32 accumulation), P turned into the B
//    operand with movmatrix, O^T += V^T P^T with a second m16n8k16;
//  - fp32 FMA (FMA = true, one packed query row): each lane owns one key and
//    forms its score as an fp32 dot product with the query (held in fp32 in
//    shared memory, read by broadcast), then each lane accumulates Dv/32
//    output dims over the warp's 32 keys, the weights passed by warp shuffle
//    ("SmallQ FlashAttention for Ascend 910B", section "算法要点": fp32 scalar
//    dot products and fp32 accumulation for a few query rows).
// Either way the scores go through masking and the base-2 online softmax
// (running max m and sum l in fp32; the accumulator is rescaled by
// 2^(m_old - m_new) when the max grows: "昇腾CANN上的FlashAttention工程实战",
// tiling + online softmax section).  At the last tile of a segment the warps
// merge their (m, l, O) through shared memory and write the final O / lse
// (unit finished inside this piece) or a normalised partial and its
// log2-sum-exp (unit shared with other pieces; merged by the combine kernel).
//
// Launched with programmatic dependent launch: barrier set-up, tensor-map
// prefetch and (for dense K/V) the schedule run before the kernel waits for
// the previous kernel in the stream; nothing in global memory is touched
// before that wait.  Every wait is bounded (see mbar_wait).
#pragma once

#include "fa_common.cuh"
#include "fa_internal.h"

namespace fa {

// Stage header written by the producer, read by every consumer warp.
struct StageMeta {
    int b, rb, hkv, tile;  // unit and key tile (keys tile * TK ...)
    int flags, piece, slot, pad;
};
constexpr int kMetaFirst = 1;  // first tile of a segment: Q is in the stage, reset state
constexpr int kMetaLast = 2;   // last tile of a segment: run the epilogue
constexpr int kMetaWhole = 4;  // the segment is the whole unit: write O / lse
constexpr int kMetaDone = 8;   // no more work
constexpr int kMetaFinal = 16; // the CTA's last tile


// KB: 16-key blocks per consumer warp per tile (2: 128-key tiles; 1: 64-key
// tiles, for head dims whose 128-key stage would not leave room for a ring).
// ILV: paged K / V with pages smaller than a tile, each page gathered in one
// 5-D box with all its 64-column chunks (Params::kv_ilv).
template <int DQK, int DV, int STAGES, bool FMA, int KB = 2, bool ILV_ = false>
struct SplitCfg {
    static constexpr bool ILV = ILV_;
    static constexpr int KEYS_PER_WARP = 16 * KB;
    static constexpr int TK = KEYS_PER_WARP * kConsumerWarps;  // keys per tile
    static constexpr int TK_SHIFT = KB == 2 ? 7 : 6;
    static_assert((1 << TK_SHIFT) == TK, "TK is 2^TK_SHIFT");
    static constexpr int KBOX = DQK / 64;
    static constexpr int VBOX = DV / 64;
    static constexpr int BOX_BYTES = TK * 128;  // TK keys x 64 elements x 2 bytes
    static constexpr int STAGE_BYTES = (KBOX + VBOX) * BOX_BYTES;  // K and V of one tile
    static constexpr int Q_STRIDE = DQK + 8;    // padded Q row (elements): conflict-free fragment loads
    static constexpr int Q_BYTES = kRowsPerCta * Q_STRIDE * 2;
    static constexpr int RED_STRIDE = DV + 4;   // padded row: conflict-free scatter
    static constexpr int RED_BYTES = kConsumerWarps * kRowsPerCta * RED_STRIDE * 4;
    static constexpr int OFF_Q = STAGES * STAGE_BYTES;
    static constexpr int QF_BYTES = FMA ? kConsumerWarps * DQK * 4 : 0;  // per-warp fp32 query row
    static constexpr int OFF_QF = OFF_Q + STAGES * Q_BYTES;
    static constexpr int OFF_RED = OFF_QF + QF_BYTES;
    static constexpr int OFF_M = OFF_RED + RED_BYTES;
    static constexpr int OFF_L = OFF_M + kConsumerWarps * kRowsPerCta * 4;
    static constexpr int OFF_META = OFF_L + kConsumerWarps * kRowsPerCta * 4;
    static constexpr int OFF_BAR = OFF_META + STAGES * (int)sizeof(StageMeta);
    static constexpr int OFF_MISC = OFF_BAR + (2 * STAGES + 1) * 8;
    static constexpr int OFF_SCRATCH = (OFF_MISC + 16 + 15) & ~15;  // sink of the warm-up pass's stores
    static constexpr int SMEM_USED = OFF_SCRATCH + 64;
    static constexpr int SMEM = SMEM_USED + 1024;  // slack to align the base to 1024 B
    static_assert(DQK % 64 == 0 && DV % 64 == 0, "head dims are multiples of 64");
    static_assert(OFF_QF % 16 == 0 && OFF_RED % 16 == 0 && OFF_BAR % 8 == 0, "aligned regions");
    static_assert(SMEM <= 232448, "fits the 227 KB per-CTA shared memory limit");
    // paged K/V: pages of >= 16 keys give at most TK / 16 boxes per column
    // chunk; the producer's lanes loop over them
    static_assert((KBOX + VBOX) * (TK / 16) <= 64, "paged boxes per tile: at most two per lane");
};


// Tiles of a CTA's piece the producer asks L2 for before waiting on the
// previous kernel (dense K / V).
#ifndef FA_PREFETCH_TILES
#define FA_PREFETCH_TILES 2
#endif
constexpr int kPrefetchTiles = FA_PREFETCH_TILES;
// Tile-by-tile cursor over a piece: a SegmentWalker plus the tile within the
// current segment (device code, any single lane).
struct TileCursor {
    SegmentWalker w;
    int tt, t1;
    __device__ __forceinline__ void start(const SegmentWalker &wk) {
        w = wk;
        tt = w.done() ? 0 : w.pos - w.u0;
        t1 = w.done() ? 0 : w.seg_end() - w.u0;
    }
    __device__ __forceinline__ bool done() const { return w.done(); }
    __device__ __forceinline__ void next(const Params &p) {
        if (++tt < t1) return;
        w.advance(p);
        if (!w.done()) {
            tt = w.pos - w.u0;
            t1 = w.seg_end() - w.u0;
        }
    }
};

// L2 prefetch of the K and V boxes of the cursor's tile (dense K / V).
template <class C>
__device__ __forceinline__ void prefetch_tile(const CUtensorMap *tmK, const CUtensorMap *tmV, const Params &p,
                                              const TileCursor &pc) {
    const int b = pc.w.b(p);
    const BatchGeom G = batch_geom(p, b);
    const int kb = p.cu_q ? 0 : b;
    const int key = G.k0 + pc.tt * C::TK;
#pragma unroll
    for (int c = 0; c < C::KBOX; ++c) tma_prefetch_4d(tmK, c * 64, key, pc.w.hkv, kb);
#pragma unroll
    for (int c = 0; c < C::VBOX; ++c) tma_prefetch_4d(tmV, c * 64, key, pc.w.hkv, kb);
}

// The producer warp's loop, shared by the split-KV kernels: walks the CTA's
// piece of the key-tile space (the Partition) segment by segment and feeds the
// copy ring(s) -- per tile the TMA loads of K and V (C::KBOX and C::VBOX
// boxes of C::TK keys x 64 elements, 128-byte swizzle, L2 evict-first, no
// multicast; a paged cache gathered page by page) and the tile header (in
// meta[stage], or meta[it % kMetaRing] with separate rings); at the first tile of each segment q_write(s, seg, b, rb, hkv,
// G) (all 32 lanes, s the K slot) stages the unit's query rows and returns
// false if a wait gave up.  Ends with the end-of-work marker and a bounded
// wait for every copy still in flight.  Must be called by all 32 lanes of the
// warp.
//
// Where a tile's K and V go.  Joint stages (VS == 0 in splitkv_produce): K
// and V of tile it share stage it % KS (V right after K) and its full / empty
// barriers.  Separate rings (VS > 0): K goes to K slot it % KS and V to V slot
// it % VS, each with its own full / empty barriers, so K can be released as
// soon as the products that read it are done while V waits for its own.
// With separate rings the tile headers have a ring of their own,
// meta[it % kMetaRing]: the producer can run at most KS tiles ahead of the S
// products and those at most two tiles ahead of the softmax, so a header is
// read before its entry comes round again as long as KS + 3 <= kMetaRing.
constexpr int kMetaRing = 8;

struct RingLayout {
    uint32_t k_base, k_stride;  // shared address of K slot 0, bytes between slots
    uint32_t v_base, v_stride;  // V slot 0 (joint: stage 0's V boxes), bytes between slots
    uint32_t kfull0, kempty0;   // barrier arrays of the K slots / joint stages (8 bytes apart)
    uint32_t vfull0, vempty0;   // barrier arrays of the V slots (separate rings only)
};

template <class C, int KS, int VS, class QW>
__device__ __forceinline__ void splitkv_produce(const CUtensorMap *tmK, const CUtensorMap *tmV, const Params &p,
                                                const RingLayout &R, StageMeta *meta, volatile int *abort_flag,
                                                QW &&q_write) {
    constexpr bool kJoint = VS == 0;
    static_assert(kJoint || KS + 3 <= kMetaRing, "header ring deep enough for the K ring");
    constexpr uint32_t kKBytes = C::KBOX * C::BOX_BYTES, kVBytes = C::VBOX * C::BOX_BYTES;
    const int lane = threadIdx.x & 31;
    auto kfull = [&](int s) { return R.kfull0 + 8u * s; };
    auto kempty = [&](int s) { return R.kempty0 + 8u * s; };
    auto vfull = [&](int s) { return R.vfull0 + 8u * s; };
    auto vempty = [&](int s) { return R.vempty0 + 8u * s; };
    // Dense inputs: the schedule needs only the kernel's parameters, so it
    // is worked out before the wait and overlaps the previous kernel; cache
    // or sequence lengths are read only after the wait.
    Partition pt = {0, 1};
    SegmentWalker wk;
    bool active = false;
    const int cta = blockIdx.x;
    auto plan = [&]() {
        pt = make_partition(warp_total_tiles(p), p.P, p.min_share);
        active = pt.W > 0 && cta < pt.P;
        if (active) wk.init(p, piece_start(pt, cta), piece_end(pt, cta));
    };
    if (uniform_batches(p)) {
        plan();
        // While the previous kernel in the stream finishes, ask L2 for the
        // first tiles of this CTA's piece (dense K / V only: the addresses
        // need no memory reads).  A prefetch hands no data to this CTA --
        // the loads below still run after the wait and read L2, where any
        // write of the previous kernel lands -- so it cannot see stale data;
        // it only moves the first HBM reads ahead, into the previous
        // kernel's tail, where the memory system is mostly idle.
        if (active && lane == 0 && !p.block_table) {
            TileCursor pc;
            pc.start(wk);
            for (int n = 0; n < kPrefetchTiles && !pc.done(); ++n, pc.next(p)) prefetch_tile<C>(tmK, tmV, p, pc);
        }
        __syncwarp();
    }
    pdl_wait_primary();
    // The combine kernel's CTAs may be scheduled now (they wait for this
    // grid to complete before reading anything it writes).
    pdl_launch_dependents();
    if (!uniform_batches(p)) plan();

    const uint64_t policy = l2_policy_evict_first();
    // Issues the boxes of one tile's K (V_PART false) or V (true) -- or both,
    // for joint stages -- completing on `bar`.  Paged K / V: the tile is
    // gathered page by page.  A page of at least TK keys gives one box of TK
    // rows; a smaller page gives TK / page boxes of `page` rows, stacked in
    // the slot exactly where one TK-row box would put them (a box of 8 or more
    // rows starts on a 1024-byte swizzle period).  The lanes share the boxes;
    // a page past the table or an invalid block number reads as zeros
    // (out-of-range coordinates).
    auto issue = [&](bool do_k, bool do_v, uint32_t kdst, uint32_t vdst, uint32_t bar, int b, int hkv,
                     const BatchGeom &G, int j) {
        const int kb = p.cu_q ? 0 : b;  // K / V batch coordinate (packed inputs: one batch of tokens)
        if (lane == 0) mbar_expect_tx(bar, (do_k ? kKBytes : 0u) + (do_v ? kVBytes : 0u));
        if (!p.block_table) {
            if (lane == 0) {
                if (do_k) {
#pragma unroll
                    for (int c = 0; c < C::KBOX; ++c)
                        tma_load_4d(kdst + c * C::BOX_BYTES, tmK, bar, c * 64, G.k0 + j, hkv, kb, policy);
                }
                if (do_v) {
#pragma unroll
                    for (int c = 0; c < C::VBOX; ++c)
                        tma_load_4d(vdst + c * C::BOX_BYTES, tmV, bar, c * 64, G.k0 + j, hkv, kb, policy);
                }
            }
        } else if constexpr (C::ILV) {
            // pages smaller than a tile, each page's K / V rows with all their
            // chunks in one 5-D box: the page's rows land at sub * page * 128
            // * chunks in the slot, chunk after chunk
            __syncwarp();
            const int nsub = C::TK >> p.page_shift;
            const int count = (do_k ? nsub : 0) + (do_v ? nsub : 0);
            for (int idx = lane; idx < count; idx += 32) {
                const bool is_k = do_k && idx < nsub;
                const int sub = do_k ? (is_k ? idx : idx - nsub) : idx;
                const int key = j + (sub << p.page_shift);
                const int page = key >> p.page_shift;
                int blk = p.num_blocks;
                if (page < p.max_pages) {
                    const int e = __ldg(p.block_table + (long long)b * p.bt_stride + page);
                    if (e >= 0 && e < p.num_blocks) blk = e;
                }
                const uint32_t off = (uint32_t)(sub << p.page_shift) * 128u * (is_k ? C::KBOX : C::VBOX);
                if (is_k) tma_load_5d(kdst + off, tmK, bar, 0, 0, 0, hkv, blk, policy);
                else tma_load_5d(vdst + off, tmV, bar, 0, 0, 0, hkv, blk, policy);
            }
        } else {
            __syncwarp();
            const int sub_shift = p.page_shift < C::TK_SHIFT ? p.page_shift : C::TK_SHIFT;
            const int nsub = C::TK >> sub_shift;
            const int c0 = do_k ? 0 : C::KBOX, c1 = do_v ? C::KBOX + C::VBOX : C::KBOX;
            for (int idx = lane; idx < (c1 - c0) * nsub; idx += 32) {
                const int c = c0 + idx / nsub, sub = idx % nsub;
                const int key = j + (sub << sub_shift);
                const int page = key >> p.page_shift;
                int blk = p.num_blocks;
                if (page < p.max_pages) {
                    const int e = __ldg(p.block_table + (long long)b * p.bt_stride + page);
                    if (e >= 0 && e < p.num_blocks) blk = e;
                }
                const int row = key & ((1 << p.page_shift) - 1);
                const uint32_t off = (uint32_t)(sub << sub_shift) * 128u;
                if (c < C::KBOX)
                    tma_load_4d(kdst + c * C::BOX_BYTES + off, tmK, bar, c * 64, row, hkv, blk, policy);
                else
                    tma_load_4d(vdst + (c - C::KBOX) * C::BOX_BYTES + off, tmV, bar, (c - C::KBOX) * 64, row, hkv,
                                blk, policy);
            }
        }
    };
    int it = 0, itv = 0, seg = 0;  // tiles whose K (joint: K and V) / separate V were issued
    bool stop = !active;
    for (; active && !wk.done() && !stop; wk.advance(p), ++seg) {
        const int b = wk.b(p), rb = wk.rb(p), hkv = wk.hkv;
        const BatchGeom G = batch_geom(p, b);
        const int t0 = wk.pos - wk.u0, t1 = wk.seg_end() - wk.u0;
        const bool whole = (wk.pos == wk.u0) && (wk.seg_end() == wk.u0 + wk.t);
        const int slot = seg == 0 ? 0 : 1;  // partial slot: the CTA's first segment, or a later one
        for (int tt = t0; tt < t1 && !stop; ++tt, ++it) {
            const int s = it % KS, use = it / KS;
            // test hook: the first CTA leaves its first tile's slots empty (no
            // copy, no arrival), so the consumers' wait on it runs out
            if (p.stall && cta == 0 && it == 0) {
                if (!kJoint) ++itv;
                continue;
            }
            bool ok = use == 0 || mbar_wait(kempty(s), (use - 1) & 1, abort_flag, p.status, p.wait_limit_ns);
            if (!__all_sync(0xffffffffu, ok)) {  // keep the warp's control flow uniform
                stop = true;
                break;
            }
            const uint32_t kdst = R.k_base + s * R.k_stride;
            // (one piece per CTA: the piece's last tile is the CTA's last tile)
            const int flags = (tt == t0 ? kMetaFirst : 0) | (tt == t1 - 1 ? kMetaLast : 0) |
                              (whole ? kMetaWhole : 0) | (tt == t1 - 1 && wk.last_segment() ? kMetaFinal : 0);
            const int j = tt * C::TK;
            issue(true, kJoint, kdst, R.v_base + s * R.v_stride, kfull(s), b, hkv, G, j);
            // separate rings: V's copy goes out too before the query rows are
            // staged (a synchronous copy at a segment's first tile)
            int vs = 0;
            bool vok = true;
            if constexpr (!kJoint) {
                const int vuse = itv / VS;
                vs = itv % VS;
                vok = vuse == 0 || mbar_wait(vempty(vs), (vuse - 1) & 1, abort_flag, p.status, p.wait_limit_ns);
                vok = __all_sync(0xffffffffu, vok);
                if (vok) issue(false, true, 0u, R.v_base + vs * R.v_stride, vfull(vs), b, hkv, G, j);
            }
            if (lane == 0) {
                StageMeta m = {b, rb, hkv, tt, flags, cta, slot, 0};
                meta[kJoint ? s : it % kMetaRing] = m;
            }
            const bool qok = vok && (!(flags & kMetaFirst) || __all_sync(0xffffffffu, q_write(s, seg, b, rb, hkv, G)));
            __syncwarp();
            if (lane == 0) mbar_arrive(kfull(s));
            if constexpr (!kJoint) {
                if (vok) {
                    if (lane == 0) mbar_arrive(vfull(vs));
                    ++itv;
                }
            }
            if (!qok) {  // a wait gave up (the CTA is aborting): the slots still complete, then stop
                stop = true;
                ++it;
                break;
            }
        }
    }
    // end-of-work marker in the next K slot / stage (its previous load was
    // consumed: the empty barrier says so); with separate rings it completes
    // the next V slot's phase as well, since consumers may take the tile
    // header from either ring's barrier
    const int s_done = it % KS, v_done = itv % (kJoint ? 1 : VS);
    bool done_sent = false, vdone_sent = false;
    {
        const int use = it / KS;
        bool ok = use == 0 || mbar_wait(kempty(s_done), (use - 1) & 1, abort_flag, p.status, p.wait_limit_ns);
        bool vok = kJoint;
        if constexpr (!kJoint) {
            const int vuse = itv / VS;
            vok = ok && (vuse == 0 || mbar_wait(vempty(v_done), (vuse - 1) & 1, abort_flag, p.status, p.wait_limit_ns));
        }
        ok = __all_sync(0xffffffffu, ok);
        vok = __all_sync(0xffffffffu, vok);
        if (lane == 0) {
            StageMeta m = {0, 0, 0, 0, kMetaDone, 0, 0, 0};
            meta[kJoint ? s_done : it % kMetaRing] = m;
        }
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(kfull(s_done));
        if constexpr (!kJoint) {
            if (lane == 0 && vok) mbar_arrive(vfull(v_done));
        }
        done_sent = ok;
        vdone_sent = !kJoint && vok;
    }
    // Never leave the CTA with copies in flight: wait (bounded, whatever
    // the abort state) for the last load issued into each slot.  The
    // marker's slot needs no wait once the marker went out.
    if (lane == 0) {
        volatile int no_abort = 0;
        for (int s = 0; s < KS && s < it; ++s) {
            if (s == s_done && done_sent) continue;
            const int last_use = (it - 1 - s) / KS;
            mbar_wait(kfull(s), last_use & 1, &no_abort, p.status, p.wait_limit_ns / 8);
        }
        if constexpr (!kJoint) {
            for (int s = 0; s < VS && s < itv; ++s) {
                if (s == v_done && vdone_sent) continue;
                const int last_use = (itv - 1 - s) / VS;
                mbar_wait(vfull(s), last_use & 1, &no_abort, p.status, p.wait_limit_ns / 8);
            }
        }
    }
}


template <typename T, int DQK, int DV, int STAGES, bool FMA, int KB = 2, bool ILV = false>
__global__ void __launch_bounds__(kThreads, 1)
    splitkv_kernel(const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const Params p) {
    using C = SplitCfg<DQK, DV, STAGES, FMA, KB, ILV>;
    static_assert(!ILV || !FMA, "the page-interleaved layout is read by the mma.sync consumer only");
    static_assert(!FMA || KB == 2, "the FMA consumer gives each lane one of 32 keys per warp");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    float *red = reinterpret_cast<float *>(smem + C::OFF_RED);
    float *sm_m = reinterpret_cast<float *>(smem + C::OFF_M);
    float *sm_l = reinterpret_cast<float *>(smem + C::OFF_L);
    StageMeta *meta = reinterpret_cast<StageMeta *>(smem + C::OFF_META);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t smem_base = smem_u32(smem);
    auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
    auto empty_bar = [&](int s) { return smem_u32(&bars[STAGES + s]); };
    const uint32_t ep_bar = smem_u32(&bars[2 * STAGES]);

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), kConsumerWarps);
        }
        mbar_init(ep_bar, kConsumerWarps);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kConsumerWarps && lane == 0) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    __syncthreads();  // barriers initialised

    if (warp == kConsumerWarps) {
        // ============================================================ producer warp
        // At the first tile of a segment the unit's 8 packed query rows (rows
        // past g*Lq are zero) go into the stage's Q slot, copied
        // asynchronously and counted on the same stage barrier.
        const T *__restrict__ qg = reinterpret_cast<const T *>(p.q);
        auto q_write = [&](int s, int seg, int b, int rb, int hkv, const BatchGeom &G) {
            (void)seg;
            const uint32_t qs = smem_base + C::OFF_Q + s * C::Q_BYTES;
            for (int idx = lane; idx < kRowsPerCta * (DQK / 8); idx += 32) {
                const int r = idx / (DQK / 8), c = idx % (DQK / 8);
                const int rq = rb * kRowsPerCta + r;
                const T *src = qg;
                uint32_t nbytes = 0;
                if (rq < G.R && c * 8 < p.dqk) {  // dims past the call's head dim stay zero
                    const int hq = hkv * p.g + rq / G.Lq, i = rq % G.Lq;
                    src = qg + b * p.q_sb + (long long)(G.q0 + i) * p.q_sl + (long long)hq * p.q_sh + c * 8;
                    nbytes = 16;
                }
                cp_async_16(qs + (r * C::Q_STRIDE + c * 8) * 2, src, nbytes);
            }
            cp_async_mbar_arrive(full_bar(s));
            return true;
        };
        const RingLayout ring = {smem_base, (uint32_t)C::STAGE_BYTES, smem_base + C::KBOX * C::BOX_BYTES,
                                 (uint32_t)C::STAGE_BYTES, full_bar(0), empty_bar(0), 0u, 0u};
        splitkv_produce<C, STAGES, 0>(&tmK, &tmV, p, ring, meta, abort_flag, q_write);
        return;
    }

    // ================================================================ consumer warps
    // The loop below starts with two warm-up passes (it = -2, -1) that run
    // before the wait for the previous kernel: the tile body and the epilogue
    // (its partial-output and its final-output form) execute once on a stage
    // that holds no data yet, with every store sent to a shared-memory sink.
    // Their results are discarded (the first real tile resets the state).  They
    // bring the code into the instruction caches while nothing else is waiting
    // on these warps; otherwise the first epilogue of a CTA can stall for
    // microseconds on instruction fetches queued behind the K/V stream.
    T *__restrict__ og = reinterpret_cast<T *>(p.o);
    void *const sink = smem + C::OFF_SCRATCH;
    const int kw = warp * C::KEYS_PER_WARP;  // this warp's first key within a tile
    const int r_lo = 2 * (lane & 3);         // accumulator rows of this lane: r_lo, r_lo + 1
    uint32_t ep_phase = 0;

    // Where the 16-key blocks and 64-column chunks of a stage's K and V sit:
    // block kb of this warp at kblk[kb] / vblk[kb] from the slot, chunk c at
    // c * chs further (the whole tile's chunks one after the other, or, for
    // pages smaller than a tile gathered in 5-D boxes, each page's chunks
    // one after the other -- Params::kv_ilv).
    const uint32_t chs = ILV ? (128u << p.page_shift) : (uint32_t)C::BOX_BYTES;
    uint32_t kblk[KB], vblk[KB];  // (ILV only; the plain layout's are kw * 128 + kb * 2048)
#pragma unroll
    for (int kb = 0; kb < KB; ++kb) {
        const int r = kw + kb * 16;  // the block's first key within the tile
        const uint32_t in_page = (uint32_t)(r & ((1 << p.page_shift) - 1)) * 128u;
        const uint32_t page0 = (uint32_t)(r >> p.page_shift) * chs;
        kblk[kb] = page0 * C::KBOX + in_page;
        vblk[kb] = page0 * C::VBOX + in_page;
    }
    // Per-lane ldmatrix offsets inside a block (the 128-byte swizzle XORs the
    // 16-byte chunk index with key & 7, and key & 7 == lane & 7 here).
    uint32_t koff[DQK / 16], voff[DV / 16];
    {
        const int sw = lane & 7;
        const int kkey = (lane & 7) + ((lane >> 3) & 1) * 8;  // A = K block: matrices (k0-7|k8-15) x (d lo|hi)
#pragma unroll
        for (int kk = 0; kk < DQK / 16; ++kk) {
            const int d = kk * 16 + ((lane >> 4) & 1) * 8;
            koff[kk] = (d >> 6) * chs + ((((d & 63) >> 3) ^ sw) << 4) + kkey * 128;
        }
        const int vkey = (lane & 7) + ((lane >> 4) & 1) * 8;  // A = V^T block: (d lo|hi) x (k0-7|k8-15)
#pragma unroll
        for (int t = 0; t < DV / 16; ++t) {
            const int d = t * 16 + ((lane >> 3) & 1) * 8;
            voff[t] = (d >> 6) * chs + ((((d & 63) >> 3) ^ sw) << 4) + vkey * 128;
        }
    }

    // Merge of the four warps' (m, l, O) published in shared memory, then the
    // store of the final O / lse (unit finished here) or of the partial and its
    // log2-sum-exp.  Shared by both variants.
    auto merge_store = [&](const StageMeta &md, bool warm, const BatchGeom &cg) {
        // thread -> (row, 8 consecutive dims); weights 2^(m_w - M) of the warps' partials
        constexpr int EPT = DV * kRowsPerCta / (32 * kConsumerWarps);
        constexpr int TPR = DV / EPT;
        const int r = tid / TPR;
        const int d0 = (tid % TPR) * EPT;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm_m[w * kRowsPerCta + r]);
        float wt[kConsumerWarps];
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const float mw = sm_m[w * kRowsPerCta + r];
            wt[w] = (M == -INFINITY || mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
            L += wt[w] * sm_l[w * kRowsPerCta + r];
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        float v[EPT];
#pragma unroll
        for (int e = 0; e < EPT; ++e) v[e] = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const float *src = red + (w * kRowsPerCta + r) * C::RED_STRIDE + d0;
#pragma unroll
            for (int e = 0; e < EPT; e += 4) {
                const float4 x = *reinterpret_cast<const float4 *>(src + e);
                v[e] += wt[w] * x.x;
                v[e + 1] += wt[w] * x.y;
                v[e + 2] += wt[w] * x.z;
                v[e + 3] += wt[w] * x.w;
            }
        }
#pragma unroll
        for (int e = 0; e < EPT; ++e) v[e] *= inv;
        const float lse2 = L > 0.f ? M + log2f(L) : -INFINITY;
        const int rr = md.rb * kRowsPerCta + r;
        if (md.flags & kMetaWhole) {
            if (rr < cg.R) {
                const int hq = md.hkv * p.g + rr / cg.Lq, i = rr % cg.Lq;
                T *op = warm ? static_cast<T *>(sink)
                             : og + md.b * p.o_sb + (long long)(cg.q0 + i) * p.o_sl + (long long)hq * p.o_sh + d0;
                // only the call's Dv dims (a multiple of 8) are written
                const int dmax = warm ? DV : p.dv;
                if constexpr (EPT % 8 == 0) {
#pragma unroll
                    for (int e = 0; e < EPT; e += 8)
                        if (d0 + e < dmax) store_row8<T>(op + e, v + e);
                } else {
                    if (d0 < dmax) {
#pragma unroll
                        for (int e = 0; e < EPT; e += 2)
                            *reinterpret_cast<uint32_t *>(op + e) = Mma<T>::pack(v[e], v[e + 1]);
                    }
                }
                if (p.lse && (tid % TPR) == 0)
                    *(warm ? static_cast<float *>(sink)
                           : p.lse + md.b * p.lse_sb + hq * p.lse_sh + cg.q0 + i) = lse2 * 0.69314718055994531f;
            }
        } else {
            const long long base = ((long long)md.piece * 2 + md.slot) * kRowsPerCta + r;
            float *wo = warm ? static_cast<float *>(sink) : p.ws_o + base * DV + d0;
#pragma unroll
            for (int e = 0; e < EPT; e += 4)
                *reinterpret_cast<float4 *>(wo + (warm ? 0 : e)) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
            if ((tid % TPR) == 0) *(warm ? static_cast<float *>(sink) : p.ws_lse + base) = lse2;
        }
    };

    if constexpr (FMA) {
        // ========================================================= fp32 FMA consumer
        // One packed query row (g * Lq == 1, so Lq == 1 and the causal mask
        // hides nothing: key j is visible iff j < n).
        float *qf32 = reinterpret_cast<float *>(smem + C::OFF_QF) + warp * DQK;  // this warp's fp32 query
        const uint32_t qf_addr = smem_u32(qf32);
        const int kkey = kw + lane;            // this lane's key within a tile (scores)
        const uint32_t krow = kkey * 128;      // its row inside a K box
        const int ksw = kkey & 7;              // the row's 128-byte swizzle phase
        constexpr int EPL = DV / 32;           // output dims per lane
        const int dl = lane * EPL;
        // byte offset of this lane's dims inside a V row, per swizzle phase (key & 7)
        uint32_t vsw[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) vsw[j] = (dl >> 6) * C::BOX_BYTES + ((((dl & 63) >> 3) ^ j) << 4) + (dl & 7) * 2;
        int n = 0;
        BatchGeom cg = {p.Lq, p.R, 0, 0, 0};
        float m = -INFINITY;  // running max of the warp's scores (base 2)
        float l = 0.f;        // this lane's share of the running sum
        float acc[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = 0.f;

        for (int it = -2;; ++it) {
            const bool warm = it < 0;
            if (it == 0) pdl_wait_primary();  // outputs and workspace are written below
            const int s = warm ? 0 : it % STAGES, use = warm ? 0 : it / STAGES;
            const bool ok = warm || mbar_wait(full_bar(s), use & 1, abort_flag, p.status, p.wait_limit_ns);
            if (__any_sync(0xffffffffu, !ok || *abort_flag)) break;
            StageMeta md = {0, 0, 0, 0, kMetaFirst | kMetaLast | (it == -1 ? kMetaWhole : 0), 0, 0, 0};
            if (!warm) md = meta[s];
            if (md.flags & kMetaDone) break;
            const uint32_t kst = smem_base + s * C::STAGE_BYTES;  // the stage's K boxes
            const uint32_t vst = kst + C::KBOX * C::BOX_BYTES;    // and V boxes

            if (md.flags & kMetaFirst) {
                // packed row 0 of the stage's Q slot, converted once into fp32
                const T *qs = reinterpret_cast<const T *>(smem + C::OFF_Q + s * C::Q_BYTES);
                for (int d = lane; d < DQK; d += 32) qf32[d] = Cvt<T>::f1(qs[d]);
                __syncwarp();
                cg = warm ? BatchGeom{p.Lq, p.R, 1 << 30, 0, 0} : batch_geom(p, md.b);
                n = cg.n;
                m = -INFINITY;
                l = 0.f;
#pragma unroll
                for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
            }
            const int jbase = md.tile * C::TK + kw;

            // ---- this lane's score: fp32 dot product of its key with the query
            float sa = 0.f, sb = 0.f;
#pragma unroll
            for (int c = 0; c < C::KBOX; ++c) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint32_t k0, k1, k2, k3;
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(k0), "=r"(k1), "=r"(k2), "=r"(k3)
                                 : "r"(kst + c * C::BOX_BYTES + krow + ((ch ^ ksw) << 4)));
                    float4 qa, qb;
                    const uint32_t qaddr = qf_addr + (c * 64 + ch * 8) * 4;
                    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                 : "=f"(qa.x), "=f"(qa.y), "=f"(qa.z), "=f"(qa.w) : "r"(qaddr));
                    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                 : "=f"(qb.x), "=f"(qb.y), "=f"(qb.z), "=f"(qb.w) : "r"(qaddr + 16));
                    const float2 x0 = Cvt<T>::f2(k0), x1 = Cvt<T>::f2(k1);
                    const float2 x2 = Cvt<T>::f2(k2), x3 = Cvt<T>::f2(k3);
                    sa = fmaf(qa.x, x0.x, sa);
                    sb = fmaf(qa.y, x0.y, sb);
                    sa = fmaf(qa.z, x1.x, sa);
                    sb = fmaf(qa.w, x1.y, sb);
                    sa = fmaf(qb.x, x2.x, sa);
                    sb = fmaf(qb.y, x2.y, sb);
                    sa = fmaf(qb.z, x3.x, sa);
                    sb = fmaf(qb.w, x3.y, sb);
                }
            }
            const float sv = jbase + lane < n ? (sa + sb) * p.scale_log2 : -INFINITY;

            // ---- online softmax (base 2); the running max is warp-wide
            float mx = sv;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float mn = fmaxf(m, mx);
            const float base = mn == -INFINITY ? 0.f : mn;
            const float pj = fast_exp2(sv - base);
            if (mn != m) {  // warp-uniform
                const float al = fast_exp2(m - base);
                l *= al;
#pragma unroll
                for (int e = 0; e < EPL; ++e) acc[e] *= al;
                m = mn;
            }
            l += pj;

            // ---- cache slots at or beyond this batch's length may hold anything
            // (NaN included): zero those V rows so 0 * V stays 0.
            const uint32_t vbase = vst + kw * 128;
            if ((p.seqlens || p.cu_q) && jbase + C::KEYS_PER_WARP > n) {
                for (int idx = lane; idx < C::KEYS_PER_WARP * C::VBOX * 8; idx += 32) {
                    const int key = idx / (C::VBOX * 8);
                    const int rem = idx % (C::VBOX * 8);
                    if (jbase + key >= n) {
                        const uint32_t a = vbase + (rem >> 3) * C::BOX_BYTES + key * 128 + (rem & 7) * 16;
                        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
            }
            // ---- O += sum over the warp's 32 keys of p_j v_j (this lane's EPL dims)
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
                const float w = __shfl_sync(0xffffffffu, pj, jj);
                const uint32_t a = vbase + jj * 128 + vsw[jj & 7];
                if constexpr (EPL == 4) {
                    uint32_t v0, v1;
                    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v0), "=r"(v1) : "r"(a));
                    const float2 y0 = Cvt<T>::f2(v0), y1 = Cvt<T>::f2(v1);
                    acc[0] = fmaf(w, y0.x, acc[0]);
                    acc[1] = fmaf(w, y0.y, acc[1]);
                    acc[2] = fmaf(w, y1.x, acc[2]);
                    acc[3] = fmaf(w, y1.y, acc[3]);
                } else {
                    uint32_t v0;
                    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v0) : "r"(a));
                    const float2 y0 = Cvt<T>::f2(v0);
                    acc[0] = fmaf(w, y0.x, acc[0]);
                    acc[1] = fmaf(w, y0.y, acc[1]);
                }
            }
            __syncwarp();
            if (lane == 0 && !warm) mbar_arrive(empty_bar(s));  // the stage (K, V, Q) is free again
            if (!(md.flags & kMetaLast)) continue;

            // ---- epilogue: publish this warp's (m, l, O) as packed row 0
            float lt = l;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) lt += __shfl_xor_sync(0xffffffffu, lt, off);
            if (lane < kRowsPerCta) {
                sm_m[warp * kRowsPerCta + lane] = lane == 0 ? m : -INFINITY;
                sm_l[warp * kRowsPerCta + lane] = lane == 0 ? lt : 0.f;
            }
            float *dst = red + warp * kRowsPerCta * C::RED_STRIDE + dl;
            if constexpr (EPL == 4) {
                *reinterpret_cast<float4 *>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
            } else {
                *reinterpret_cast<float2 *>(dst) = make_float2(acc[0], acc[1]);
            }
            if (!consumer_sync_bounded(ep_bar, ep_phase, abort_flag, p.status, p.wait_limit_ns)) break;
            merge_store(md, warm, cg);
            // red / sm_m / sm_l are reused by the next segment, if there is one
            if (md.flags & kMetaFinal) break;
            if (!consumer_sync_bounded(ep_bar, ep_phase, abort_flag, p.status, p.wait_limit_ns)) break;
        }
    } else {
        // ========================================================= tensor-core consumer
        uint32_t qf[DQK / 16][2];
        int lim[2] = {0, 0};
        int n = 0;
        BatchGeom cg = {p.Lq, p.R, 0, 0, 0};
        float m[2] = {-INFINITY, -INFINITY};
        float l[2] = {0.f, 0.f};
        float acc[DV / 16][4];

        for (int it = -2;; ++it) {
            const bool warm = it < 0;
            if (it == 0) pdl_wait_primary();  // outputs and workspace are written below
            const int s = warm ? 0 : it % STAGES, use = warm ? 0 : it / STAGES;
            const bool ok = warm || mbar_wait(full_bar(s), use & 1, abort_flag, p.status, p.wait_limit_ns);
            if (__any_sync(0xffffffffu, !ok || *abort_flag)) break;
            StageMeta md = {0, 0, 0, 0, kMetaFirst | kMetaLast | (it == -1 ? kMetaWhole : 0), 0, 0, 0};
            if (!warm) md = meta[s];
            if (md.flags & kMetaDone) break;
            const uint32_t kst = smem_base + s * C::STAGE_BYTES;  // the stage's K
            const uint32_t vst = kst + C::KBOX * C::BOX_BYTES;    // and V
            const uint32_t kbase = kst + kw * 128;                // this warp's keys (plain layout)
            const uint32_t vbase = vst + kw * 128;

            if (md.flags & kMetaFirst) {
                // Q as the B operand: lane holds row (lane >> 2), dims 2*(lane & 3) + {0, 1} (+8).
                const uint32_t qrow =
                    smem_base + C::OFF_Q + s * C::Q_BYTES + ((lane >> 2) * C::Q_STRIDE + 2 * (lane & 3)) * 2;
    #pragma unroll
                for (int kk = 0; kk < DQK / 16; ++kk) {
                    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(qf[kk][0]) : "r"(qrow + kk * 32));
                    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(qf[kk][1]) : "r"(qrow + kk * 32 + 16));
                }
                cg = warm ? BatchGeom{p.Lq, p.R, 1 << 30, 0, 0} : batch_geom(p, md.b);
                n = cg.n;
                // last visible key of this lane's two accumulator rows (bottom-right causal)
    #pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int r = md.rb * kRowsPerCta + r_lo + e;
                    int lm = n - 1;
                    if (p.causal && r < cg.R) {
                        const int c = r % cg.Lq + n - cg.Lq;
                        lm = c < lm ? c : lm;
                    }
                    lim[e] = lm;
                }
                m[0] = m[1] = -INFINITY;
                l[0] = l[1] = 0.f;
    #pragma unroll
                for (int t = 0; t < DV / 16; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
            }
            const int jbase = md.tile * C::TK + kw;

            // ---- S^T (16 keys x 8 rows per block) = K Q^T, two independent chains per block
            float sc[KB][4], sd[KB][4];
    #pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
    #pragma unroll
                for (int e = 0; e < 4; ++e) sc[kb][e] = sd[kb][e] = 0.f;
    #pragma unroll
                for (int kk = 0; kk < DQK / 16; ++kk) {
                    uint32_t a0, a1, a2, a3;
                    ldmatrix_x4((ILV ? kst + kblk[kb] : kbase + kb * 16 * 128) + koff[kk], a0, a1, a2, a3);
                    if (kk & 1) Mma<T>::run(sd[kb], a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
                    else Mma<T>::run(sc[kb], a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
                }
            }
            // ---- mask + online softmax (base 2)
            float sv[KB][4];
            float mx0 = -INFINITY, mx1 = -INFINITY;
    #pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
                const int j0 = jbase + kb * 16 + (lane >> 2), j1 = j0 + 8;
                sv[kb][0] = j0 <= lim[0] ? (sc[kb][0] + sd[kb][0]) * p.scale_log2 : -INFINITY;
                sv[kb][1] = j0 <= lim[1] ? (sc[kb][1] + sd[kb][1]) * p.scale_log2 : -INFINITY;
                sv[kb][2] = j1 <= lim[0] ? (sc[kb][2] + sd[kb][2]) * p.scale_log2 : -INFINITY;
                sv[kb][3] = j1 <= lim[1] ? (sc[kb][3] + sd[kb][3]) * p.scale_log2 : -INFINITY;
                mx0 = fmaxf(mx0, fmaxf(sv[kb][0], sv[kb][2]));
                mx1 = fmaxf(mx1, fmaxf(sv[kb][1], sv[kb][3]));
            }
    #pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
            }
            const float mn0 = fmaxf(m[0], mx0), mn1 = fmaxf(m[1], mx1);
            const float base0 = mn0 == -INFINITY ? 0.f : mn0;
            const float base1 = mn1 == -INFINITY ? 0.f : mn1;
            uint32_t pb[KB][2];
            float ps0 = 0.f, ps1 = 0.f;
    #pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
                const float p0 = fast_exp2(sv[kb][0] - base0), p2 = fast_exp2(sv[kb][2] - base0);
                const float p1 = fast_exp2(sv[kb][1] - base1), p3 = fast_exp2(sv[kb][3] - base1);
                ps0 += p0 + p2;
                ps1 += p1 + p3;
                pb[kb][0] = movmatrix_trans(Mma<T>::pack(p0, p1));  // keys 0-7 of the block
                pb[kb][1] = movmatrix_trans(Mma<T>::pack(p2, p3));  // keys 8-15
            }
            // rescale what was accumulated so far only when a row's max moved
            if (__any_sync(0xffffffffu, mn0 != m[0] || mn1 != m[1])) {
                const float al0 = fast_exp2(m[0] - base0), al1 = fast_exp2(m[1] - base1);
                l[0] *= al0;
                l[1] *= al1;
    #pragma unroll
                for (int t = 0; t < DV / 16; ++t) {
                    acc[t][0] *= al0;
                    acc[t][1] *= al1;
                    acc[t][2] *= al0;
                    acc[t][3] *= al1;
                }
            }
            l[0] += ps0;
            l[1] += ps1;
            m[0] = mn0;
            m[1] = mn1;

            // ---- cache slots at or beyond this batch's length may hold anything
            // (NaN included): zero those V rows so 0 * V stays 0.
            if ((p.seqlens || p.cu_q) && jbase + C::KEYS_PER_WARP > n) {
                for (int idx = lane; idx < C::KEYS_PER_WARP * C::VBOX * 8; idx += 32) {
                    const int key = idx / (C::VBOX * 8);
                    const int rem = idx % (C::VBOX * 8);
                    if (jbase + key >= n) {
                        const uint32_t a = ILV ? vst + vblk[key >> 4] + (rem >> 3) * chs + (key & 15) * 128 + (rem & 7) * 16
                                               : vbase + (rem >> 3) * C::BOX_BYTES + key * 128 + (rem & 7) * 16;
                        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
            }
            // ---- O^T (DV x 8 rows) += V^T P^T
    #pragma unroll
            for (int t = 0; t < DV / 16; ++t) {
    #pragma unroll
                for (int kb = 0; kb < KB; ++kb) {
                    uint32_t a0, a1, a2, a3;
                    ldmatrix_x4_trans((ILV ? vst + vblk[kb] : vbase + kb * 16 * 128) + voff[t], a0, a1, a2, a3);
                    Mma<T>::run(acc[t], a0, a1, a2, a3, pb[kb][0], pb[kb][1]);
                }
            }
            __syncwarp();
            if (lane == 0 && !warm) mbar_arrive(empty_bar(s));  // the stage (K, V, Q) is free again
            if (!(md.flags & kMetaLast)) continue;

            // ------------------------------------------------------------ epilogue
            // full l of this warp's rows (sum over the 8 lanes sharing lane & 3)
    #pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                l[0] += __shfl_xor_sync(0xffffffffu, l[0], off);
                l[1] += __shfl_xor_sync(0xffffffffu, l[1], off);
            }
            if (lane < 4) {
                sm_m[warp * kRowsPerCta + r_lo] = m[0];
                sm_m[warp * kRowsPerCta + r_lo + 1] = m[1];
                sm_l[warp * kRowsPerCta + r_lo] = l[0];
                sm_l[warp * kRowsPerCta + r_lo + 1] = l[1];
            }
            {
                float *buf = red + warp * kRowsPerCta * C::RED_STRIDE;
    #pragma unroll
                for (int t = 0; t < DV / 16; ++t) {
                    const int d = t * 16 + (lane >> 2);
                    buf[r_lo * C::RED_STRIDE + d] = acc[t][0];
                    buf[(r_lo + 1) * C::RED_STRIDE + d] = acc[t][1];
                    buf[r_lo * C::RED_STRIDE + d + 8] = acc[t][2];
                    buf[(r_lo + 1) * C::RED_STRIDE + d + 8] = acc[t][3];
                }
            }
            if (!consumer_sync_bounded(ep_bar, ep_phase, abort_flag, p.status, p.wait_limit_ns)) break;
            merge_store(md, warm, cg);
            // red / sm_m / sm_l are reused by the next segment, if there is one
            if (md.flags & kMetaFinal) break;
            if (!consumer_sync_bounded(ep_bar, ep_phase, abort_flag, p.status, p.wait_limit_ns)) break;
        }
    }
}

}  // namespace fa
