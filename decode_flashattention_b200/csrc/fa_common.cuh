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
// kv head are laid out as r = h_local * Lq + i and cut into blocks of 8
// (the N extent of one m16n8k16 MMA when keys are the M operand).
constexpr int kRowsPerCta = 8;
constexpr int kConsumerWarps = 4;
constexpr int kThreads = 32 * (kConsumerWarps + 1);  // + one TMA producer warp
constexpr int kMaxPrefixEntries = 8192;              // B * row-blocks bound
constexpr unsigned kStatusTimeout = 1u;

struct Params {
    const void *q;  // [B, Lq, Hq, Dqk]
    int64_t q_sb, q_sl, q_sh;
    void *o;  // [B, Lq, Hq, Dv]
    int64_t o_sb, o_sl, o_sh;
    float *lse;            // [B, Hq, Lq] or null
    float *ws_o;           // partial outputs [P][2][8][Dv]
    float *ws_lse;         // partial log2-sum-exp [P][2][8]
    const int *seqlens;    // [B] or null (then every batch has Lk keys)
    unsigned *status;      // device status word (timeouts)
    int B, Lq, Hq, Hkv, g, R, RB, Lk;
    int causal;
    float scale_log2;      // scale * log2(e)
    int P;                 // CTAs launched
    int min_share;         // least tiles per CTA
    int tile_keys;         // keys per tile (TK)
};

// ------------------------------------------------------------------ schedule
// Work is counted in key tiles.  A unit is (batch b, row block rb, kv head
// hkv); unit u = (b * RB + rb) * Hkv + hkv owns ceil(kmax / TK) tiles, kmax
// being the number of leading keys any of its rows can see.  The units' tiles
// are laid end to end (W tiles in total) and cut into P_eff equal contiguous
// ranges, one per CTA, so every CTA streams the same number of tiles however
// ragged the per-batch lengths are.  A unit that falls inside one range is
// finished by that CTA; a unit cut by range boundaries leaves one partial
// (normalised O and log2-sum-exp) per CTA touching it, in slot 0 if it is the
// CTA's first segment and slot 1 otherwise, and the combine kernel merges them.

__host__ __device__ inline int keys_visible_to_block(int n, int rb, int R, int Lq, int causal) {
    if (n <= 0) return 0;
    if (!causal) return n;
    int r0 = rb * kRowsPerCta;
    int r1 = r0 + kRowsPerCta < R ? r0 + kRowsPerCta : R;
    int maxi = -1;
    for (int r = r0; r < r1; ++r) {
        int i = r % Lq;
        maxi = i > maxi ? i : maxi;
    }
    int k = maxi + n - Lq + 1;  // bottom-right: row i sees keys j <= i + n - Lq
    if (k > n) k = n;
    return k > 0 ? k : 0;
}

// Keys present for batch b: cache_seqlens[b] clamped to [0, Lk], or Lk.
__host__ __device__ inline int batch_keys(const int *seqlens, int b, int Lk) {
    if (!seqlens) return Lk;
    int n = seqlens[b];
    return n < 0 ? 0 : (n > Lk ? Lk : n);
}

__host__ __device__ inline int unit_tiles(int n, int rb, int R, int Lq, int causal, int TK) {
    int k = keys_visible_to_block(n, rb, R, Lq, causal);
    return (k + TK - 1) / TK;
}

__host__ __device__ inline int64_t eff_parts(int64_t W, int64_t P, int64_t min_share) {
    int64_t need = (W + min_share - 1) / min_share;
    int64_t p = P < need ? P : need;
    return p < 1 ? 1 : p;
}

__host__ __device__ inline int64_t part_start(int64_t c, int64_t W, int64_t P) { return (c * W) / P; }

// The CTA whose range contains tile position t (0 <= t < W).
__host__ __device__ inline int64_t part_of(int64_t t, int64_t W, int64_t P) {
    int64_t c = (t * P) / W;
    if (c >= P) c = P - 1;
    while (c + 1 < P && part_start(c + 1, W, P) <= t) ++c;
    while (c > 0 && part_start(c, W, P) > t) --c;
    return c;
}

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

// Exclusive prefix over the (batch, row-block) entries: pre[x] = Hkv * (tiles
// of entries before x), pre[BR] = W.  Runs on the whole CTA (NT
// threads); pre must hold BR + 1 int64 in shared memory, warp_tot NT / 32.
template <int NT>
__device__ __forceinline__ void build_prefix(const Params &p, long long *pre, long long *warp_tot) {
    const int BR = p.B * p.RB;
    const int tid = threadIdx.x;
    const int per = (BR + NT - 1) / NT;
    const int lo = tid * per;
    const int hi = lo + per < BR ? lo + per : BR;
    long long local = 0;
    for (int x = lo; x < hi; ++x) {
        int b = x / p.RB, rb = x % p.RB;
        int n = batch_keys(p.seqlens, b, p.Lk);
        local += unit_tiles(n, rb, p.R, p.Lq, p.causal, p.tile_keys);
    }
    // inclusive warp scan
    const int lane = tid & 31, warp = tid >> 5;
    long long incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        long long y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    long long base = 0;
    for (int w = 0; w < warp; ++w) base += warp_tot[w];
    long long run = base + incl - local;  // exclusive prefix of this thread's chunk
    for (int x = lo; x < hi; ++x) {
        int b = x / p.RB, rb = x % p.RB;
        int n = batch_keys(p.seqlens, b, p.Lk);
        pre[x] = run * p.Hkv;
        run += unit_tiles(n, rb, p.R, p.Lq, p.causal, p.tile_keys);
    }
    if (tid == NT - 1) pre[BR] = run * p.Hkv;
    __syncthreads();
}

// Largest x in [0, BR) with pre[x] <= t (t < pre[BR]); that entry has tiles.
__device__ __forceinline__ int find_entry(const long long *pre, int BR, long long t) {
    int lo = 0, hi = BR - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (pre[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Walks the segments of one CTA's tile range [start, end): each segment is a
// run of tiles of one unit.  Producer and consumers step identical copies.
struct SegmentWalker {
    int x, hkv;        // current (b*RB + rb) entry and kv head
    long long u0;      // first tile position of the current unit
    int t;             // tiles of the current unit
    long long pos, start, end;

    __device__ __forceinline__ void init(const Params &p, const long long *pre, long long s,
                                         long long e) {
        start = s;
        end = e;
        pos = s;
        const int BR = p.B * p.RB;
        x = find_entry(pre, BR, s);
        t = (int)((pre[x + 1] - pre[x]) / p.Hkv);
        hkv = (int)((s - pre[x]) / t);
        u0 = pre[x] + (long long)hkv * t;
    }
    __device__ __forceinline__ bool done() const { return pos >= end; }
    __device__ __forceinline__ int b(const Params &p) const { return x / p.RB; }
    __device__ __forceinline__ int rb(const Params &p) const { return x % p.RB; }
    __device__ __forceinline__ long long seg_end() const {
        long long ue = u0 + t;
        return ue < end ? ue : end;
    }
    // Move past the current segment.
    __device__ __forceinline__ void advance(const Params &p) {
        pos = seg_end();
        if (pos >= end) return;
        // pos is now the end of the current unit: step to the next unit with tiles
        u0 += t;
        if (++hkv < p.Hkv) return;
        hkv = 0;
        const int BR = p.B * p.RB;
        for (;;) {
            ++x;
            if (x >= BR) { t = 1; return; }  // unreachable while pos < end
            int n = batch_keys(p.seqlens, x / p.RB, p.Lk);
            t = unit_tiles(n, x % p.RB, p.R, p.Lq, p.causal, p.tile_keys);
            if (t > 0) return;
        }
    }
};

#endif  // __CUDACC__

}  // namespace fa
