// fa_common.cuh -- shared pieces of the sm_100a decode-attention kernels:
// kernel parameters, the device-side work partition, and thin wrappers over
// the PTX instructions the kernels issue (mbarrier, TMA, ldmatrix, mma.sync,
// movmatrix, ex2, griddepcontrol).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace fa {

// Query rows packed into one CTA: the g*Lq rows of a GQA group that share a
// kv head are laid out as r = h_local * Lq + i and cut into row blocks of
// Params::rpc rows.  The mma.sync kernel takes blocks of 8 (the N extent of
// one m16n8k16 MMA when keys are the M operand); the tcgen05 split-KV kernel
// takes 16, 32 or 64 (the N extent of its products).
constexpr int kRowsPerCta = 8;
constexpr int kMaxRowsPerCta = 64;
constexpr int kConsumerWarps = 4;
constexpr int kThreads = 32 * (kConsumerWarps + 1);  // + one TMA producer warp
constexpr int kMaxPrefixEntries = 8192;              // B * row-blocks bound
constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned kStatusLayout = 2u;  // a kernel found its shared-memory base misaligned and did nothing

struct Params {
    const void *q;  // [B, Lq, Hq, Dqk]
    int64_t q_sb, q_sl, q_sh;
    void *o;  // [B, Lq, Hq, Dv]
    int64_t o_sb, o_sl, o_sh;
    float *lse;            // [B, Hq, Lq] or null
    float *ws_o;           // partial outputs [pieces][2][8][Dv]
    float *ws_lse;         // partial log2-sum-exp [pieces][2][8]
    const int *seqlens;    // [B] or null (then every batch has Lk keys)
    unsigned *status;      // device status word (timeouts)
    int B, Lq, Hq, Hkv, g, R, RB, Lk;
    int rpc;               // packed rows per row block (unit), RB = ceil(R / rpc)
    int dqk, dv;           // the call's head dims (the kernel's DQK / DV may be larger: columns past them are zero)
    unsigned long long wait_limit_ns;  // bound of every wait on a pipeline barrier
    int stall;             // test hook: the first CTA leaves its first stage empty
    int causal;
    float scale_log2;      // scale * log2(e)
    int P;                 // CTAs launched
    int min_share;         // least tiles per CTA
    int W_host;            // total tiles when known on the host (dense inputs), else -1
    int tile_keys;         // keys per tile (TK), a power of two
    int tile_shift;        // log2(tile_keys)
    int seg_cost;          // positions a unit occupies in the partition beyond its tiles (see below)
    // Paged K/V (block_table non-null): K and V are [num_blocks, page, Hkv, D]
    // and key j of batch b lives in block block_table[b * bt_stride + j / page]
    // at row j % page.
    const int *block_table;
    int64_t bt_stride;
    int max_pages;         // block-table entries per batch
    int page_shift;        // log2(page)
    int num_blocks;
    // Paged pages smaller than a tile, mma.sync kernel: each page's K (and V)
    // rows come in one 5-D box holding all of its 64-column chunks, so in a
    // stage slot page `sub` of the tile starts at sub * page * 128 * chunks
    // bytes and its chunk c at + c * page * 128 (else chunk c of the whole
    // tile starts at c * TK * 128, as for dense K / V).
    int kv_ilv;
    int seqlen_add;        // tokens appended to every cache by this call (added to seqlens[b])
    // Packed variable-length inputs (cu_q non-null): q / o are [1, total_q, H, D]
    // and k / v [1, total_k, Hkv, D]; sequence b owns query tokens
    // [cu_q[b], cu_q[b+1]) and key tokens [cu_k[b], cu_k[b+1]); Lq and Lk hold
    // the largest lengths.  lse element (b, hq, i) is at
    // b * lse_sb + hq * lse_sh + (query token offset) + i.
    const int *cu_q;
    const int *cu_k;
    int64_t lse_sb, lse_sh;
    int total_q;           // packed query tokens (the combine's row count is Hq * total_q)
};


// ------------------------------------------------------------------ schedule
// Work is counted in key tiles.  A unit is (batch b, row block rb, kv head
// hkv); unit u = (b * RB + rb) * Hkv + hkv owns t = ceil(kmax / TK) tiles,
// kmax being the number of leading keys any of its rows can see.  In the
// partition a unit with tiles occupies t + seg_cost positions: its tiles, then
// seg_cost positions that stand for the fixed cost of starting and finishing a
// unit (1 for the mma.sync kernel, 4 for the tcgen05 one).  The
// units' positions are laid end to end (W in total) and cut into P_eff equal
// contiguous ranges, one per CTA, so every CTA gets the same work however
// ragged the per-batch lengths are.  A range starting inside a unit's trailing
// positions begins with the next unit.  A unit whose tiles fall inside one
// range is finished by that CTA; a unit whose tiles are cut by range
// boundaries leaves one partial (normalised O and log2-sum-exp) per CTA
// touching them, in slot 0 if it is the CTA's first segment and slot 1
// otherwise, and the combine kernel merges them.

__host__ __device__ inline int keys_visible_to_block(int n, int rb, int R, int Lq, int causal, int rpc) {
    if (n <= 0 || rb * rpc >= R) return 0;  // no keys, or a row block past the batch's rows
    if (!causal) return n;
    // rows r0 .. r0 + cnt - 1 hold query positions i = r % Lq; the largest one
    // is r0 % Lq + cnt - 1 unless the run wraps past Lq - 1.
    const int r0 = rb * rpc;
    const int cnt = R - r0 < rpc ? R - r0 : rpc;
    const int a = r0 % Lq;
    const int maxi = (a + cnt - 1 >= Lq) ? Lq - 1 : a + cnt - 1;
    int k = maxi + n - Lq + 1;  // bottom-right: row i sees keys j <= i + n - Lq
    if (k > n) k = n;
    return k > 0 ? k : 0;
}

// Keys present for batch b: Lk for dense inputs, else cache_seqlens[b] plus
// the tokens appended by this call, clamped to [0, Lk].
__host__ __device__ inline int batch_keys(const int *seqlens, int b, int Lk, int add = 0) {
    if (!seqlens) return Lk;
    const long long n = (long long)seqlens[b] + add;
    return n < 0 ? 0 : (n > Lk ? Lk : (int)n);
}

#if defined(__CUDACC__)
// Row geometry of batch b: its query rows Lq, packed rows R = g * Lq, keys n
// and the token offsets of its first query / key row (0 unless packed).
struct BatchGeom {
    int Lq, R, n, q0, k0;
};

__device__ __forceinline__ BatchGeom batch_geom(const Params &p, int b) {
    BatchGeom G;
    if (p.cu_q) {
        const int q0 = p.cu_q[b], q1 = p.cu_q[b + 1], k0 = p.cu_k[b], k1 = p.cu_k[b + 1];
        int lq = q1 - q0, n = k1 - k0;
        lq = lq < 0 ? 0 : (lq > p.Lq ? p.Lq : lq);
        n = n < 0 ? 0 : (n > p.Lk ? p.Lk : n);
        G.Lq = lq;
        G.R = p.g * lq;
        G.n = n;
        G.q0 = q0;
        G.k0 = k0;
    } else {
        G.Lq = p.Lq;
        G.R = p.R;
        G.n = batch_keys(p.seqlens, b, p.Lk, p.seqlen_add);
        G.q0 = 0;
        G.k0 = 0;
    }
    return G;
}
#endif

// Tiles of tile_keys = 1 << tile_shift keys covering the visible keys.
__host__ __device__ inline int unit_tiles(int n, int rb, int R, int Lq, int causal, int tile_shift, int rpc) {
    const int k = keys_visible_to_block(n, rb, R, Lq, causal, rpc);
    return (k + (1 << tile_shift) - 1) >> tile_shift;
}

// Tile positions fit in 32 bits (the host rejects larger problems).
__host__ __device__ inline int eff_parts(int W, int P, int min_share) {
    const int need = (W + min_share - 1) / min_share;
    const int p = P < need ? P : need;
    return p < 1 ? 1 : p;
}

// Balanced contiguous partition of W tiles over P CTAs: the first W % P CTAs
// take one tile more than the others.
__host__ __device__ inline int part_start(int c, int W, int P) {
    const int share = W / P, rem = W % P;
    return c * share + (c < rem ? c : rem);
}

// The CTA whose range contains tile position t (0 <= t < W).
__host__ __device__ inline int part_of(int t, int W, int P) {
    const int share = W / P, rem = W % P;
    const int big = (share + 1) * rem;
    return t < big ? t / (share + 1) : rem + (t - big) / share;
}

// The work partition: W tiles over P = eff_parts(...) CTAs, CTA c taking the
// contiguous piece [part_start(c), part_start(c + 1)).  A piece leaves up to
// two partial results (slot 0: the unit it starts in, slot 1: the unit it ends
// in) for units it shares with other pieces; a unit inside one piece is
// finished directly.  (A dynamic tail -- CTAs claiming the last quarter of the
// tiles from a counter -- evened out when CTAs finish but did not move the
// last one, since the kernel is bound by the total DRAM bandwidth, and cost
// more than it saved.)
struct Partition {
    int W, P;
};

__host__ __device__ inline Partition make_partition(int W, int P_param, int min_share) {
    Partition q;
    q.W = W;
    q.P = eff_parts(W, P_param, min_share);
    return q;
}

__host__ __device__ inline int piece_of(const Partition &q, int t) { return part_of(t, q.W, q.P); }
__host__ __device__ inline int piece_start(const Partition &q, int id) { return part_start(id, q.W, q.P); }
__host__ __device__ inline int piece_end(const Partition &q, int id) { return part_start(id + 1, q.W, q.P); }
__host__ __device__ inline int num_pieces(const Partition &q) { return q.P; }

// ------------------------------------------------------------------ PTX wrappers
#if defined(__CUDACC__)

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait on an mbarrier phase.  Gives up when *abort is raised by
// another warp of the CTA, or after ~limit_ns of wall time (then it records
// a timeout in the device status word and raises *abort itself).  Returns
// true when the phase completed.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort,
                                          unsigned *status, uint64_t limit_ns) {
    for (int i = 0; i < 128; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0; it < (1u << 28); ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0) {
            if (*abort) return false;
            if (global_timer_ns() - t0 > limit_ns) break;
        }
    }
    if (status) atomicOr(status, kStatusTimeout);
    *abort = 1;
    return false;
}

// 4-D tiled TMA load into shared memory, completion counted on `bar`
// (no multicast).
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int c0, int c1, int c2, int c3, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
        "l"(policy)
        : "memory");
}

// The same for a 5-D tile (one page of a paged cache with all its 64-column
// chunks: coordinates {0, row, 0, head, block}).
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int c0, int c1, int c2, int c3, int c4, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2], %8;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4),
        "l"(policy)
        : "memory");
}

// L2 prefetch of one 4-D tile (no shared-memory destination, no completion
// to wait for; out-of-range coordinates fetch nothing).
__device__ __forceinline__ void tma_prefetch_4d(const CUtensorMap *map, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                            uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                                  uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

template <typename T>
struct Mma;

template <>
struct Mma<__half> {
    __device__ __forceinline__ static void run(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
            "{%8, %9}, {%0, %1, %2, %3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
    __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
        __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&h);
    }
};

template <>
struct Mma<__nv_bfloat16> {
    __device__ __forceinline__ static void run(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
            "{%8, %9}, {%0, %1, %2, %3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
    __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&h);
    }
};

// 16-bit element(s) to fp32 (exact), and fp32 to 16-bit (round to nearest even).
template <typename T>
struct Cvt;

template <>
struct Cvt<__half> {
    __device__ __forceinline__ static float f1(__half x) { return __half2float(x); }
    __device__ __forceinline__ static __half from(float x) { return __float2half_rn(x); }
    __device__ __forceinline__ static float2 f2(uint32_t x) {
        return __half22float2(*reinterpret_cast<const __half2 *>(&x));
    }
};

template <>
struct Cvt<__nv_bfloat16> {
    __device__ __forceinline__ static float f1(__nv_bfloat16 x) { return __bfloat162float(x); }
    __device__ __forceinline__ static __nv_bfloat16 from(float x) { return __float2bfloat16_rn(x); }
    __device__ __forceinline__ static float2 f2(uint32_t x) {
        return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&x));
    }
};

// 2^x on the special-function unit (PTX ex2.approx.ftz.f32): 2^-inf = +0.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait_primary() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Sync of the consumer warps through an mbarrier (one arrival per warp), with
// the same bounded wait as the pipeline: a warp that gave up never leaves the
// others blocked.  `phase` is the caller's running parity.
__device__ __forceinline__ bool consumer_sync_bounded(uint32_t bar, uint32_t &phase, volatile int *abort,
                                                      unsigned *status, uint64_t limit_ns) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
    const bool ok = mbar_wait(bar, phase, abort, status, limit_ns);
    phase ^= 1u;
    return __all_sync(0xffffffffu, ok);
}

// 16-byte global -> shared copy on the LSU async path (cp.async); src_bytes = 0
// fills the 16 bytes with zeros without reading global memory.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}

// The mbarrier's current phase also waits for this thread's earlier cp.async
// copies (the pending count is raised now and lowered when they land).
__device__ __forceinline__ void cp_async_mbar_arrive(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumerWarps) : "memory");
}

template <typename T>
__device__ __forceinline__ void store_row8(T *dst, const float *v);

template <>
__device__ __forceinline__ void store_row8<__half>(__half *dst, const float *v) {
    uint4 u;
    __half2 h0 = __floats2half2_rn(v[0], v[1]), h1 = __floats2half2_rn(v[2], v[3]);
    __half2 h2 = __floats2half2_rn(v[4], v[5]), h3 = __floats2half2_rn(v[6], v[7]);
    u.x = *reinterpret_cast<uint32_t *>(&h0);
    u.y = *reinterpret_cast<uint32_t *>(&h1);
    u.z = *reinterpret_cast<uint32_t *>(&h2);
    u.w = *reinterpret_cast<uint32_t *>(&h3);
    *reinterpret_cast<uint4 *>(dst) = u;
}

template <>
__device__ __forceinline__ void store_row8<__nv_bfloat16>(__nv_bfloat16 *dst, const float *v) {
    uint4 u;
    __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]), h1 = __floats2bfloat162_rn(v[2], v[3]);
    __nv_bfloat162 h2 = __floats2bfloat162_rn(v[4], v[5]), h3 = __floats2bfloat162_rn(v[6], v[7]);
    u.x = *reinterpret_cast<uint32_t *>(&h0);
    u.y = *reinterpret_cast<uint32_t *>(&h1);
    u.z = *reinterpret_cast<uint32_t *>(&h2);
    u.w = *reinterpret_cast<uint32_t *>(&h3);
    *reinterpret_cast<uint4 *>(dst) = u;
}

// ------------------------------------------------------------------ warp-level schedule
// Every warp of a CTA derives the same schedule on its own, in registers, so
// the copy pipeline can start without a block-wide prefix in shared memory.
// Entries x = b * RB + rb are visited in chunks of 32 (one per lane).

__device__ __forceinline__ int entry_tiles(const Params &p, int x) {
    const int b = x / p.RB, rb = x - b * p.RB;
    const BatchGeom G = batch_geom(p, b);
    return unit_tiles(G.n, rb, G.R, G.Lq, p.causal, p.tile_shift, p.rpc);
}

// Partition positions of one unit with t tiles.
__host__ __device__ __forceinline__ int unit_weight(int t, int seg_cost) { return t > 0 ? t + seg_cost : 0; }

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// Positions of all units of entries [x0, x1), counted Hkv times (one per kv head).
__device__ __forceinline__ int warp_entry_tiles(const Params &p, int x0, int x1) {
    const int lane = threadIdx.x & 31;
    int acc = 0;
    for (int x = x0 + lane; x < x1; x += 32) acc += unit_weight(entry_tiles(p, x), p.seg_cost);
    return warp_sum(acc) * p.Hkv;
}

// Dense inputs (no cache lengths, not packed): every batch has the same units,
// and the schedule needs no memory reads.
__device__ __forceinline__ bool uniform_batches(const Params &p) { return !p.seqlens && !p.cu_q; }

// Total positions W.
__device__ __forceinline__ int warp_total_tiles(const Params &p) {
    if (p.W_host >= 0) return p.W_host;
    if (uniform_batches(p)) return warp_entry_tiles(p, 0, p.RB) * p.B;
    return warp_entry_tiles(p, 0, p.B * p.RB);
}

// First position of entry x's units.
__device__ __forceinline__ int warp_entry_begin(const Params &p, int x) {
    if (uniform_batches(p)) {
        const int b = x / p.RB;
        return warp_entry_tiles(p, 0, p.RB) * b + warp_entry_tiles(p, b * p.RB, x);
    }
    return warp_entry_tiles(p, 0, x);
}

// Entry x holding position t (0 <= t < W); *x_begin receives the first
// position of x's units.
__device__ __forceinline__ int warp_locate(const Params &p, int t, int *x_begin) {
    const int lane = threadIdx.x & 31;
    int x_lo = 0, x_hi = p.B * p.RB, run = 0;
    if (uniform_batches(p)) {  // jump straight to the batch: all batches weigh the same
        const int per_batch = warp_entry_tiles(p, 0, p.RB);
        const int b = t / per_batch;
        x_lo = b * p.RB;
        x_hi = x_lo + p.RB;
        run = per_batch * b;
    }
    for (int c0 = x_lo; c0 < x_hi; c0 += 32) {
        const int x = c0 + lane;
        const int tt = x < x_hi ? unit_weight(entry_tiles(p, x), p.seg_cost) * p.Hkv : 0;
        int incl = tt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        const int excl = run + incl - tt;
        const unsigned hit = __ballot_sync(0xffffffffu, tt > 0 && excl <= t && t < excl + tt);
        if (hit) {
            const int src = __ffs(hit) - 1;
            *x_begin = __shfl_sync(0xffffffffu, excl, src);
            return c0 + src;
        }
        run += __shfl_sync(0xffffffffu, incl, 31);
    }
    *x_begin = run;  // not reached for t < W
    return x_hi - 1;
}

// Walks the segments of one CTA's range [start, end) of positions: each
// segment is a run of tiles of one unit.  Producer and consumers step
// identical copies.
struct SegmentWalker {
    int x, hkv;   // current (b*RB + rb) entry and kv head
    int u0;       // first position of the current unit (its first tile)
    int t, w;     // tiles and positions of the current unit
    int pos, start, end;

    // Must be called by all 32 lanes of a warp (uses warp collectives).
    __device__ __forceinline__ void init(const Params &p, int s, int e) {
        start = s;
        end = e;
        pos = s;
        int xb = 0;
        x = warp_locate(p, s, &xb);
        t = entry_tiles(p, x);
        w = unit_weight(t, p.seg_cost);
        hkv = (s - xb) / w;
        u0 = xb + hkv * w;
        // a range starting in a unit's trailing positions begins with the next unit
        if (pos >= u0 + t) advance(p);
    }
    __device__ __forceinline__ bool done() const { return pos >= end; }
    __device__ __forceinline__ int b(const Params &p) const { return x / p.RB; }
    __device__ __forceinline__ int rb(const Params &p) const { return x % p.RB; }
    // end (position) of the current segment's tiles
    __device__ __forceinline__ int seg_end() const {
        const int ue = u0 + t;
        return ue < end ? ue : end;
    }
    // whether the current segment is the range's last (the next unit starts at
    // or past the range's end)
    __device__ __forceinline__ bool last_segment() const { return u0 + w >= end; }
    // Move past the current unit.
    __device__ __forceinline__ void advance(const Params &p) {
        pos = u0 + w;
        if (pos >= end) return;
        u0 += w;
        if (++hkv < p.Hkv) return;
        hkv = 0;
        const int BR = p.B * p.RB;
        for (;;) {
            ++x;
            if (x >= BR) { t = 1; w = 1; return; }  // unreachable while pos < end
            t = entry_tiles(p, x);
            w = unit_weight(t, p.seg_cost);
            if (t > 0) return;
        }
    }
};

#endif  // __CUDACC__

}  // namespace fa
