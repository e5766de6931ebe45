// fa_combine.cu -- log-sum-exp weighted merge of split-KV partials.
//
// For an output row whose unit was cut across pieces s = first..last of the
// work partition, each piece left a normalised partial O_s and its
// log2-sum-exp lse2_s.  The row's
// result is
//     L2 = M + log2 sum_s 2^(lse2_s - M),     M = max_s lse2_s
//     O  = sum_s 2^(lse2_s - L2) O_s,         lse = L2 * ln 2
// (the log-sum-exp recurrence of the online softmax applied once more across
// splits: CSDN "FlashAttention on Ascend CANN" post, "在线 Softmax" section;
// split-KV partials as in the M1 split-KV decode kernel of the MXFlashAttn
// README).  Rows whose unit has no visible key get O = 0, lse = -inf; rows
// finished inside one piece were already written by the main kernel and are
// skipped.  One warp per row (or, for the wide row blocks of the tcgen05
// kernel, one to four warps per unit); lanes cover the head dim with vector
// loads.  Each warp re-derives the work partition from the sizes (and cache
// lengths) exactly as the split-KV kernel did: a partial lives at a fixed slot
// of the piece that produced it, whichever CTA ran that piece.
#include "fa_common.cuh"
#include "fa_internal.h"

namespace fa {

constexpr int kCombineThreads = 128;
constexpr int kCombineWarps = kCombineThreads / 32;

constexpr int kPartsPerPass = 8;  // partials one warp handles per pass (one per lane)

// Warps given to a unit by the per-unit form: one per row of it, up to four (a
// unit holds min(rpc, R) rows: R = g * Lq packed rows per kv head).
__host__ __device__ inline int combine_warps_per_unit(int rpc, int R) {
    const int rows = rpc < R ? rpc : R;
    return rows >= 4 ? 4 : (rows >= 2 ? 2 : 1);
}

// Lane `lane`'s partial of a pass: the partial of piece c = cf + j0 + lane for
// row rl of the unit whose tiles start at u0 (slot 0 when the piece starts
// inside the unit, else slot 1).
__device__ __forceinline__ long long partial_base(const Params &p, const Partition &pt, int c, int u0, int rl) {
    return ((long long)c * 2 + (piece_start(pt, c) >= u0 - p.seg_cost ? 0 : 1)) * p.rpc + rl;
}

// Merges the np partials (pieces cf .. cf + np - 1) of one output row -- row
// rl of a unit with tu > 0 tiles starting at u0 -- into O (dims below dmax)
// at op and the natural-log lse at lse_out (when not null); tu == 0 writes
// O = 0, lse = -inf.  b0: this lane's partial of the first pass (computed
// ahead by the caller).  The warm-up form reads and writes the sink.
template <typename T, int DV>
__device__ __forceinline__ void merge_row(const Params &p, const Partition &pt, bool warm, const float *sink, int tu,
                                          int np, int cf, int u0, int rl, long long b0, T *op, float *lse_out,
                                          int lane_off) {
    constexpr int EPL = DV / 32;  // elements per lane
    constexpr int PPP = DV >= 256 ? 4 : kPartsPerPass;  // partials per pass (fewer for wide rows: registers)
    const int lane = threadIdx.x & 31;
    const float *ws_o = warm ? sink : p.ws_o;
    const float *ws_lse = warm ? sink : p.ws_lse;
    float acc[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
    float lse2 = -INFINITY;
    if (tu > 0) {
        float M = -INFINITY, L = 0.f;
        for (int j0 = 0; j0 < np; j0 += PPP) {
            // lane j < PPP owns partial cf + j0 + j; its lse and every lane's
            // O slices of the pass are loaded together
            const int c = cf + j0 + lane;
            const bool has = lane < PPP && j0 + lane < np;
            const long long base = j0 == 0 ? b0 : (has && !warm ? partial_base(p, pt, c, u0, rl) : 0);
            const int cnt = np - j0 < PPP ? np - j0 : PPP;
            const float ls = has ? ws_lse[base] : -INFINITY;
            float v[PPP][EPL];
#pragma unroll
            for (int q = 0; q < PPP; ++q) {
                const long long bq = __shfl_sync(0xffffffffu, base, q);
                if (q < cnt) {
                    const float *src = ws_o + bq * DV + lane_off;
                    if constexpr (EPL % 4 == 0) {
#pragma unroll
                        for (int e = 0; e < EPL; e += 4) {
                            const float4 x4 = *reinterpret_cast<const float4 *>(src + e);
                            v[q][e] = x4.x; v[q][e + 1] = x4.y; v[q][e + 2] = x4.z; v[q][e + 3] = x4.w;
                        }
                    } else {
                        const float2 x2 = *reinterpret_cast<const float2 *>(src);
                        v[q][0] = x2.x; v[q][1] = x2.y;
                    }
                }
            }
            float mx = ls;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float Mn = fmaxf(M, mx);
            if (Mn == -INFINITY) continue;
            const float w = ls == -INFINITY ? 0.f : fast_exp2(ls - Mn);  // unnormalised weight
            float sum = w;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            const float scale_old = M == -INFINITY ? 0.f : fast_exp2(M - Mn);
            L = L * scale_old + sum;
            M = Mn;
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] *= scale_old;
#pragma unroll
            for (int q = 0; q < PPP; ++q) {
                const float wq = __shfl_sync(0xffffffffu, w, q);
                if (q < cnt) {
#pragma unroll
                    for (int e = 0; e < EPL; ++e) acc[e] += wq * v[q][e];
                }
            }
        }
        if (M != -INFINITY) {
            const float inv = 1.f / L;
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] *= inv;
            lse2 = M + log2f(L);
        }
    }
    const int dmax = warm ? DV : p.dv;  // only the call's Dv dims (a multiple of 8) are written
#pragma unroll
    for (int e = 0; e < EPL; e += 2)
        if (lane_off + e < dmax) *reinterpret_cast<uint32_t *>(op + e) = Mma<T>::pack(acc[e], acc[e + 1]);
    if (lse_out && lane == 0) *lse_out = lse2 == -INFINITY ? -INFINITY : lse2 * 0.69314718055994531f;
    __syncwarp();
}

// Per-row form (row blocks of up to 8 rows, the mma.sync kernel's): one warp
// per output row; a CTA's four warps take four consecutive rows.  Everything
// that needs no memory -- the row's unit, the partition, this lane's first
// partial -- is worked out before the wait for dense inputs.  (Its merge is
// written out here rather than through merge_row: the shared routine cost the
// single-row decode 0.7 us per call, measured.)
template <typename T, int DV>
__global__ void __launch_bounds__(kCombineThreads)
    combine_rows_kernel(const Params p) {
    // The next kernel in the stream may start its prologue now; it still waits
    // for this grid to finish before touching memory.
    pdl_launch_dependents();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * (kCombineThreads / 32) + warp;
    // This warp's output row (b, hq, i), the token offset q0 of its batch's
    // first query row, and its unit.  Dense rows are numbered (b, hq, i);
    // packed variable-length rows (hq, token), the batch found in cu_q -- so
    // only after the wait for them.
    bool live = false;
    int b = 0, hq = 0, i = 0, q0 = 0, rr = 0, hkv = 0, x = 0;
    auto locate = [&]() {
        int r = 0;
        if (p.cu_q) {
            live = row < (long long)p.Hq * p.total_q;
            if (!live) return;
            hq = (int)(row / p.total_q);
            const int tok = (int)(row % p.total_q);
            int lo = 0, hi = p.B;  // the batch b with cu_q[b] <= tok < cu_q[b + 1]
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (p.cu_q[mid] <= tok) lo = mid;
                else hi = mid;
            }
            b = lo;
            q0 = p.cu_q[b];
            i = tok - q0;
            const BatchGeom G = batch_geom(p, b);
            if (i >= G.Lq) {  // past the longest query length: not computed
                live = false;
                return;
            }
            r = (hq % p.g) * G.Lq + i;
        } else {
            live = row < (long long)p.B * p.Hq * p.Lq;
            if (!live) return;
            i = (int)(row % p.Lq);
            hq = (int)((row / p.Lq) % p.Hq);
            b = (int)(row / ((long long)p.Lq * p.Hq));
            r = (hq % p.g) * p.Lq + i;
        }
        rr = r % p.rpc;
        hkv = hq / p.g;
        x = b * p.RB + r / p.rpc;
    };
    if (!p.cu_q) locate();

    // The partition and the partials' addresses are worked out before the
    // wait (dense inputs need no memory for it); cache lengths only after it.
    constexpr int EPL = DV / 32;  // elements per lane
    constexpr int PPP = DV >= 256 ? 4 : kPartsPerPass;  // partials per pass (fewer for wide rows: registers)
    int t = 0, u0 = 0, cf = 0, nparts = 0;
    long long base0 = 0;  // this lane's partial in the first pass
    Partition pt = {0, 1};
    auto plan = [&]() {
        pt = make_partition(warp_total_tiles(p), p.P, p.min_share);
        t = entry_tiles(p, x);
        u0 = warp_entry_begin(p, x) + hkv * unit_weight(t, p.seg_cost);
        nparts = 0;
        base0 = 0;
        if (t > 0) {
            cf = piece_of(pt, u0);
            nparts = piece_of(pt, u0 + t - 1) - cf + 1;
            const int c = cf + lane;
            if (lane < PPP && lane < nparts)
                base0 = ((long long)c * 2 + (piece_start(pt, c) >= u0 - p.seg_cost ? 0 : 1)) * p.rpc + rr;
        }
    };
    if (uniform_batches(p) && live) plan();

    // Two passes over the same code: a warm-up pass before the wait for the
    // split-KV kernel, which merges eight copies of a shared-memory row into a
    // shared-memory sink (its result is discarded), so that the instructions
    // are cached when the real pass runs; then the real pass.
    __shared__ __align__(16) float sink[DV + 4];
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        const bool warm = pass == 0;
        if (!warm) {
            // Every CTA waits for the split-KV kernel before it exits, so this
            // grid completing implies that one completed too.
            pdl_wait_primary();
            if (p.cu_q) locate();
            if (!live) return;
            if (!uniform_batches(p)) plan();
            if (t > 0 && nparts == 1) return;  // finished inside one piece by the split-KV kernel
        }
        const int tu = warm ? 1 : t, np = warm ? PPP : nparts;
        const long long b0 = warm ? 0 : base0;
        const float *ws_o = warm ? sink : p.ws_o;
        const float *ws_lse = warm ? sink : p.ws_lse;
        T *op = warm ? reinterpret_cast<T *>(sink)
                     : reinterpret_cast<T *>(p.o) + b * p.o_sb + (long long)(q0 + i) * p.o_sl +
                           (long long)hq * p.o_sh + lane * EPL;
        float *lse_out = warm ? sink : (p.lse ? p.lse + b * p.lse_sb + hq * p.lse_sh + q0 + i : nullptr);
        const int lane_off = warm ? 0 : lane * EPL;
        float acc[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
        float lse2 = -INFINITY;

        if (tu > 0) {
            float M = -INFINITY, L = 0.f;
            for (int j0 = 0; j0 < np; j0 += PPP) {
                // lane j < PPP owns partial cf + j0 + j; its lse and every
                // lane's O slices of the pass are loaded together
                const int c = cf + j0 + lane;
                const bool has = lane < PPP && j0 + lane < np;
                const long long base =
                    j0 == 0 ? b0
                            : (has ? ((long long)c * 2 + (piece_start(pt, c) >= u0 - p.seg_cost ? 0 : 1)) * p.rpc + rr : 0);
                const int cnt = np - j0 < PPP ? np - j0 : PPP;
                const float ls = has ? ws_lse[base] : -INFINITY;
                float v[PPP][EPL];
#pragma unroll
                for (int q = 0; q < PPP; ++q) {
                    const long long bq = __shfl_sync(0xffffffffu, base, q);
                    if (q < cnt) {
                        const float *src = ws_o + bq * DV + lane_off;
                        if constexpr (EPL % 4 == 0) {
#pragma unroll
                            for (int e = 0; e < EPL; e += 4) {
                                const float4 x4 = *reinterpret_cast<const float4 *>(src + e);
                                v[q][e] = x4.x; v[q][e + 1] = x4.y; v[q][e + 2] = x4.z; v[q][e + 3] = x4.w;
                            }
                        } else {
                            const float2 x2 = *reinterpret_cast<const float2 *>(src);
                            v[q][0] = x2.x; v[q][1] = x2.y;
                        }
                    }
                }
                float mx = ls;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                const float Mn = fmaxf(M, mx);
                if (Mn == -INFINITY) continue;
                const float w = ls == -INFINITY ? 0.f : fast_exp2(ls - Mn);  // unnormalised weight
                float sum = w;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
                const float scale_old = M == -INFINITY ? 0.f : fast_exp2(M - Mn);
                L = L * scale_old + sum;
                M = Mn;
#pragma unroll
                for (int e = 0; e < EPL; ++e) acc[e] *= scale_old;
#pragma unroll
                for (int q = 0; q < PPP; ++q) {
                    const float wq = __shfl_sync(0xffffffffu, w, q);
                    if (q < cnt) {
#pragma unroll
                        for (int e = 0; e < EPL; ++e) acc[e] += wq * v[q][e];
                    }
                }
            }
            if (M != -INFINITY) {
                const float inv = 1.f / L;
#pragma unroll
                for (int e = 0; e < EPL; ++e) acc[e] *= inv;
                lse2 = M + log2f(L);
            }
        }
        const int dmax = warm ? DV : p.dv;  // only the call's Dv dims (a multiple of 8) are written
#pragma unroll
        for (int e = 0; e < EPL; e += 2)
            if (lane_off + e < dmax) *reinterpret_cast<uint32_t *>(op + e) = Mma<T>::pack(acc[e], acc[e + 1]);
        if (lse_out && lane == 0) *lse_out = lse2 == -INFINITY ? -INFINITY : lse2 * 0.69314718055994531f;
        __syncwarp();
    }
}

// Per-unit form (row blocks of 16 to 64 rows, the tcgen05 split-KV
// kernel's): a unit u = (b * RB + rb) * Hkv + hkv is taken by one to four
// warps of a CTA (combine_warps_per_unit).  Each warp works out the unit's
// place in the partition once for all its rows; a unit finished inside one
// piece was written by the split-KV kernel and its warps exit at once, a unit
// with no visible key gets O = 0 and lse = -inf, and a unit cut between
// pieces has its rows merged, the unit's warps taking every wpu-th row.  (One
// warp per row of such blocks made every row's warp repeat the partition
// arithmetic: 41 us against 22.5 us on a batched GQA-8 speculative decode.)
template <typename T, int DV>
__global__ void __launch_bounds__(kCombineThreads)
    combine_units_kernel(const Params p) {
    pdl_launch_dependents();

    constexpr int EPL = DV / 32;
    constexpr int PPP = DV >= 256 ? 4 : kPartsPerPass;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wpu = combine_warps_per_unit(p.rpc, p.R);
    const int u = blockIdx.x * (kCombineWarps / wpu) + warp / wpu, wu = warp % wpu;
    if (u >= p.B * p.RB * p.Hkv) return;
    const int x = u / p.Hkv, hkv = u - x * p.Hkv;
    const int b = x / p.RB, rb = x - b * p.RB;

    int t = 0, u0 = 0, cf = 0, nparts = 0;
    Partition pt = {0, 1};
    auto plan = [&]() {
        pt = make_partition(warp_total_tiles(p), p.P, p.min_share);
        t = entry_tiles(p, x);
        u0 = warp_entry_begin(p, x) + hkv * unit_weight(t, p.seg_cost);
        nparts = 0;
        if (t > 0) {
            cf = piece_of(pt, u0);
            nparts = piece_of(pt, u0 + t - 1) - cf + 1;
        }
    };
    if (uniform_batches(p)) plan();

    __shared__ __align__(16) float sink[DV + 4];
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        const bool warm = pass == 0;
        BatchGeom G = {1, 1, 1, 0, 0};
        int nrows = warm && wu == 0 ? 1 : 0;
        if (!warm) {
            pdl_wait_primary();
            if (!uniform_batches(p)) plan();
            if (t > 0 && nparts == 1) return;  // finished inside one piece by the split-KV kernel
            G = batch_geom(p, b);
            nrows = G.R - rb * p.rpc < p.rpc ? G.R - rb * p.rpc : p.rpc;
        }
#pragma unroll 1
        for (int rl = wu; rl < nrows; rl += wpu) {
            const int r = rb * p.rpc + rl;
            const int hq = hkv * p.g + r / G.Lq, i = r % G.Lq;
            T *op = warm ? reinterpret_cast<T *>(sink)
                         : reinterpret_cast<T *>(p.o) + b * p.o_sb + (long long)(G.q0 + i) * p.o_sl +
                               (long long)hq * p.o_sh + lane * EPL;
            float *lse_out = warm ? sink : (p.lse ? p.lse + b * p.lse_sb + hq * p.lse_sh + G.q0 + i : nullptr);
            const long long b0 =
                !warm && t > 0 && lane < PPP && lane < nparts ? partial_base(p, pt, cf + lane, u0, rl) : 0;
            merge_row<T, DV>(p, pt, warm, sink, warm ? 1 : t, warm ? PPP : nparts, cf, u0, rl, b0, op, lse_out,
                             warm ? 0 : lane * EPL);
        }
    }
}

// Which form: per unit for wide row blocks when the units are many (the
// per-row form would repeat the partition arithmetic for every row), per row
// otherwise (few units: their rows merge in parallel).
bool combine_per_unit(long long units, int rpc, int sms) { return rpc > kRowsPerCta && units >= 2LL * sms; }

// CTAs of the combine kernel: rows / 4 for the per-row form, units / (units
// per CTA) for the per-unit form.
int combine_grid(long long rows, long long units, int rpc, int R, bool per_unit) {
    if (!per_unit) return (int)((rows + kCombineWarps - 1) / kCombineWarps);
    const int per_cta = kCombineWarps / combine_warps_per_unit(rpc, R);
    return (int)((units + per_cta - 1) / per_cta);
}

template <typename T, int DV>
static void fill(KernelInfo *out, bool per_unit) {
    out->fn = per_unit ? reinterpret_cast<const void *>(&combine_units_kernel<T, DV>)
                       : reinterpret_cast<const void *>(&combine_rows_kernel<T, DV>);
    out->threads = kCombineThreads;
    out->smem = 0;
    out->tile_keys = 0;
    out->stages = 0;
    out->variant = 0;
}

bool get_combine_kernel(int dtype, int dv, bool per_unit, KernelInfo *out) {
    if (dtype == 0) {
        if (dv == 64) { fill<__half, 64>(out, per_unit); return true; }
        if (dv == 128) { fill<__half, 128>(out, per_unit); return true; }
        if (dv == 256) { fill<__half, 256>(out, per_unit); return true; }
    } else if (dtype == 1) {
        if (dv == 64) { fill<__nv_bfloat16, 64>(out, per_unit); return true; }
        if (dv == 128) { fill<__nv_bfloat16, 128>(out, per_unit); return true; }
        if (dv == 256) { fill<__nv_bfloat16, 256>(out, per_unit); return true; }
    }
    return false;
}

}  // namespace fa
