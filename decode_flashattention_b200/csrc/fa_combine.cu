// fa_combine.cu -- log-sum-exp weighted merge of split-KV partials.
//
// For an output row whose unit was cut across CTAs s = first..last, each CTA
// left a normalised partial O_s and its log2-sum-exp lse2_s.  The row's
// result is
//     L2 = M + log2 sum_s 2^(lse2_s - M),     M = max_s lse2_s
//     O  = sum_s 2^(lse2_s - L2) O_s,         lse = L2 * ln 2
// (the log-sum-exp recurrence of the online softmax applied once more across
// splits: CSDN "FlashAttention on Ascend CANN" post, "在线 Softmax" section;
// split-KV partials as in the M1 split-KV decode kernel of the MXFlashAttn
// README).  Rows whose unit has no visible key get O = 0, lse = -inf; rows
// finished inside one CTA were already written by the main kernel and are
// skipped.  One warp per row; lanes cover the head dim with vector loads.
#include "fa_common.cuh"
#include "fa_internal.h"

namespace fa {

constexpr int kCombineThreads = 128;

template <typename T, int DV>
__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const Params p) {
    extern __shared__ long long pre[];  // BR + 1 entries
    __shared__ long long warp_tot[kCombineThreads / 32];
    // seqlens is an input of the whole call: it was complete before the main
    // kernel started, so the schedule can be rebuilt before waiting on it.
    build_prefix<kCombineThreads>(p, pre, warp_tot);
    const long long W = pre[p.B * p.RB];
    const long long P = eff_parts(W, p.P, p.min_share);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * (kCombineThreads / 32) + warp;
    const long long rows = (long long)p.B * p.Hq * p.Lq;
    if (row >= rows) return;
    const int i = (int)(row % p.Lq);
    const int hq = (int)((row / p.Lq) % p.Hq);
    const int b = (int)(row / ((long long)p.Lq * p.Hq));
    const int r = (hq % p.g) * p.Lq + i;
    const int rb = r / kRowsPerCta, rr = r % kRowsPerCta, hkv = hq / p.g;
    const int n = batch_keys(p.seqlens, b, p.Lk);
    const int t = unit_tiles(n, rb, p.R, p.Lq, p.causal, p.tile_keys);

    constexpr int EPL = DV / 32;  // elements per lane
    T *op = reinterpret_cast<T *>(p.o) + b * p.o_sb + (long long)i * p.o_sl + (long long)hq * p.o_sh +
            lane * EPL;
    float acc[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
    float lse2 = -INFINITY;

    if (t > 0) {
        const long long u0 = pre[b * p.RB + rb] + (long long)hkv * t;
        const long long u1 = u0 + t;
        const long long cf = part_of(u0, W, P), cl = part_of(u1 - 1, W, P);
        if (cf == cl) return;  // finished by one CTA
        pdl_wait_primary();    // partials come from the main kernel
        auto slot_of = [&](long long c) { return part_start(c, W, P) >= u0 ? 0 : 1; };
        float M = -INFINITY;
        for (long long c = cf + lane; c <= cl; c += 32)
            M = fmaxf(M, p.ws_lse[(c * 2 + slot_of(c)) * kRowsPerCta + rr]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        if (M != -INFINITY) {
            float L = 0.f;
            for (long long c = cf + lane; c <= cl; c += 32) {
                const float ls = p.ws_lse[(c * 2 + slot_of(c)) * kRowsPerCta + rr];
                L += fast_exp2(ls - M);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
            lse2 = M + log2f(L);
            for (long long c = cf; c <= cl; ++c) {
                const long long base = (c * 2 + slot_of(c)) * kRowsPerCta + rr;
                const float w = fast_exp2(p.ws_lse[base] - lse2);
                const float *src = p.ws_o + base * DV + lane * EPL;
                if constexpr (EPL == 4) {
                    const float4 x = *reinterpret_cast<const float4 *>(src);
                    acc[0] += w * x.x;
                    acc[1] += w * x.y;
                    acc[2] += w * x.z;
                    acc[3] += w * x.w;
                } else {
#pragma unroll
                    for (int e = 0; e < EPL; ++e) acc[e] += w * src[e];
                }
            }
        }
    }
#pragma unroll
    for (int e = 0; e < EPL; e += 2)
        *reinterpret_cast<uint32_t *>(op + e) = Mma<T>::pack(acc[e], acc[e + 1]);
    if (p.lse && lane == 0)
        p.lse[((long long)b * p.Hq + hq) * p.Lq + i] = lse2 == -INFINITY ? -INFINITY : lse2 * 0.69314718055994531f;
}

template <typename T, int DV>
static void fill(KernelInfo *out) {
    out->fn = reinterpret_cast<const void *>(&combine_kernel<T, DV>);
    out->threads = kCombineThreads;
    out->smem = 0;  // the host adds (BR + 1) * 8 bytes
    out->tile_keys = 0;
    out->stages = 0;
    out->variant = 0;
}

bool get_combine_kernel(int dtype, int dv, KernelInfo *out) {
    if (dtype == 0) {
        if (dv == 64) { fill<__half, 64>(out); return true; }
        if (dv == 128) { fill<__half, 128>(out); return true; }
    } else if (dtype == 1) {
        if (dv == 64) { fill<__nv_bfloat16, 64>(out); return true; }
        if (dv == 128) { fill<__nv_bfloat16, 128>(out); return true; }
    }
    return false;
}

}  // namespace fa
