// fa_splitkv_mma.cu -- split-KV decode / small-Q attention, tensor-core variant.
//
// One CTA streams a contiguous range of key tiles (see the schedule in
// fa_common.cuh) for one or more (batch, kv-head, 8-row block) units:
//
//   warp 4 (producer): one lane issues TMA tile loads of K and V (64 keys x
//       64 elements per box, 128-byte swizzle, no multicast) into a ring of
//       STAGES shared-memory stages, each guarded by a full/empty mbarrier pair
//       (K-outer blocking with prefetch of the next tiles while the current one
//       is consumed: "SmallQ FlashAttention for Ascend 910B", section "算法要点",
//       and the CSDN "FlashAttention on Ascend CANN" post, section on
//       pipelining HBM prefetch with compute);
//   warps 0-3 (consumers): each takes 16 of the 64 keys of a tile and computes
//       S^T = K Q^T with mma.sync m16n8k16 (keys are the M operand, the 8
//       packed query rows are N, fp32 accumulation), masks, runs the online
//       softmax in base 2 (running max m and sum l in fp32, previous
//       accumulator rescaled by 2^(m_old - m_new) whenever the max grows:
//       "昇腾CANN上的FlashAttention工程实战", tiling + online softmax section),
//       turns P into the B operand with movmatrix, and accumulates
//       O^T += V^T P^T with a second m16n8k16 (head dim as M).
//   At the end of a unit's segment the four warps merge their (m, l, O) in
//   shared memory and write either the final O / lse (unit finished by this
//   CTA) or a normalised partial O and its log2-sum-exp (unit shared with
//   other CTAs; merged by the combine kernel).
#include "fa_common.cuh"
#include "fa_internal.h"

namespace fa {

template <int DQK, int DV, int STAGES>
struct MmaCfg {
    static constexpr int TK = 64;  // keys per tile: 4 consumer warps x 16
    static constexpr int KBOX = DQK / 64;
    static constexpr int VBOX = DV / 64;
    static constexpr int BOX_BYTES = TK * 128;  // 64 keys x 64 elements x 2 bytes
    static constexpr int STAGE_BYTES = (KBOX + VBOX) * BOX_BYTES;
    static constexpr int RED_STRIDE = DV + 4;  // padded row: conflict-free scatter
    static constexpr int RED_BYTES = 2 * kRowsPerCta * RED_STRIDE * 4;
    static constexpr int OFF_RED = STAGES * STAGE_BYTES;
    static constexpr int OFF_M = OFF_RED + RED_BYTES;
    static constexpr int OFF_L = OFF_M + kConsumerWarps * kRowsPerCta * 4;
    static constexpr int OFF_BAR = OFF_L + kConsumerWarps * kRowsPerCta * 4;
    static constexpr int OFF_MISC = OFF_BAR + 2 * STAGES * 8;
    static constexpr int SMEM_USED = OFF_MISC + 16 + 8 * 8;
    static constexpr int SMEM = SMEM_USED + 1024;  // slack to align the base to 1024 B
    static_assert(DQK % 64 == 0 && DV % 64 == 0, "head dims are multiples of 64");
    static_assert(STAGES * STAGE_BYTES >= (kMaxPrefixEntries + 1) * 8,
                  "the stage area also holds the schedule prefix");
};

constexpr uint64_t kWaitLimitNs = 4000000000ull;  // 4 s

template <typename T, int DQK, int DV, int STAGES>
__global__ void __launch_bounds__(kThreads, 2)
    splitkv_mma_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const Params p) {
    using C = MmaCfg<DQK, DV, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    // Let the combine kernel's CTAs be scheduled as soon as every CTA of this
    // grid is running; the combine waits for this grid's memory before reading.
    pdl_launch_dependents();

    float *red = reinterpret_cast<float *>(smem + C::OFF_RED);
    float *sm_m = reinterpret_cast<float *>(smem + C::OFF_M);
    float *sm_l = reinterpret_cast<float *>(smem + C::OFF_L);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC);
    long long *warp_tot = reinterpret_cast<long long *>(smem + C::OFF_MISC + 16);
    long long *pre = reinterpret_cast<long long *>(smem);  // stage area, before any TMA

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t smem_base = smem_u32(smem);
    auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
    auto empty_bar = [&](int s) { return smem_u32(&bars[STAGES + s]); };

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), kConsumerWarps);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kConsumerWarps && lane == 0) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    build_prefix<kThreads>(p, pre, warp_tot);  // ends with __syncthreads
    const long long W = pre[p.B * p.RB];
    const long long P = eff_parts(W, p.P, p.min_share);
    if (W == 0 || (long long)blockIdx.x >= P) return;  // uniform across the CTA
    const long long r_start = part_start(blockIdx.x, W, P);
    const long long r_end = part_start(blockIdx.x + 1, W, P);
    SegmentWalker wk;
    wk.init(p, pre, r_start, r_end);
    __syncthreads();  // the prefix is dead from here on: the stages may be filled

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer
        if (lane != 0) return;
        const uint64_t policy = l2_policy_evict_first();
        int it = 0;
        bool stop = false;
        for (; !wk.done() && !stop; wk.advance(p)) {
            const int b = wk.b(p), hkv = wk.hkv;
            const long long t0 = wk.pos - wk.u0, t1 = wk.seg_end() - wk.u0;
            for (long long tt = t0; tt < t1; ++tt, ++it) {
                const int s = it % STAGES, use = it / STAGES;
                if (use > 0 && !mbar_wait(empty_bar(s), (use - 1) & 1, abort_flag, p.status, kWaitLimitNs)) {
                    stop = true;
                    break;
                }
                const uint32_t kdst = smem_base + s * C::STAGE_BYTES;
                const uint32_t vdst = kdst + C::KBOX * C::BOX_BYTES;
                const int j = (int)(tt * C::TK);
                mbar_arrive_expect_tx(full_bar(s), C::STAGE_BYTES);
#pragma unroll
                for (int c = 0; c < C::KBOX; ++c)
                    tma_load_4d(kdst + c * C::BOX_BYTES, &tmK, full_bar(s), c * 64, j, hkv, b, policy);
#pragma unroll
                for (int c = 0; c < C::VBOX; ++c)
                    tma_load_4d(vdst + c * C::BOX_BYTES, &tmV, full_bar(s), c * 64, j, hkv, b, policy);
            }
        }
        // Never leave the CTA with copies in flight: wait (bounded, whatever
        // the abort state) for the last load issued into each stage.
        const int issued = it;
        for (int s = 0; s < STAGES && s < issued; ++s) {
            const int last_use = (issued - 1 - s) / STAGES;
            volatile int no_abort = 0;
            mbar_wait(full_bar(s), last_use & 1, &no_abort, p.status, kWaitLimitNs / 8);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const T *__restrict__ qg = reinterpret_cast<const T *>(p.q);
    T *__restrict__ og = reinterpret_cast<T *>(p.o);
    const int kw = warp * 16;             // this warp's keys within a tile
    const int r_lo = 2 * (lane & 3);      // accumulator rows of this lane: r_lo, r_lo + 1
    const int ct = tid;                   // 0..127 epilogue thread index
    constexpr int EPT = DV / 16;          // epilogue elements per thread
    int it = 0;

    for (; !wk.done(); wk.advance(p)) {
        const int b = wk.b(p), rb = wk.rb(p), hkv = wk.hkv;
        const int n = batch_keys(p.seqlens, b, p.Lk);
        const long long t0 = wk.pos - wk.u0, t1 = wk.seg_end() - wk.u0;
        const bool whole = (wk.pos == wk.u0) && (wk.seg_end() == wk.u0 + wk.t);
        const int slot = (wk.pos == wk.start) ? 0 : 1;

        // Q as the B operand: lane holds row (lane >> 2), dims 2*(lane & 3) + {0, 1} (+8).
        uint32_t qf[DQK / 16][2];
        {
            const int rq = rb * kRowsPerCta + (lane >> 2);
            if (rq < p.R) {
                const int hq = hkv * p.g + rq / p.Lq, i = rq % p.Lq;
                const T *qp = qg + b * p.q_sb + (long long)i * p.q_sl + (long long)hq * p.q_sh + 2 * (lane & 3);
#pragma unroll
                for (int kk = 0; kk < DQK / 16; ++kk) {
                    qf[kk][0] = *reinterpret_cast<const uint32_t *>(qp + kk * 16);
                    qf[kk][1] = *reinterpret_cast<const uint32_t *>(qp + kk * 16 + 8);
                }
            } else {
#pragma unroll
                for (int kk = 0; kk < DQK / 16; ++kk) qf[kk][0] = qf[kk][1] = 0u;
            }
        }
        // Last visible key of this lane's two accumulator rows (bottom-right causal).
        int lim[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int r = rb * kRowsPerCta + r_lo + e;
            int l = n - 1;
            if (p.causal && r < p.R) {
                const int c = r % p.Lq + n - p.Lq;
                l = c < l ? c : l;
            }
            lim[e] = l;
        }

        float m[2] = {-INFINITY, -INFINITY};
        float l[2] = {0.f, 0.f};
        float acc[DV / 16][4];
#pragma unroll
        for (int t = 0; t < DV / 16; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

        for (long long tt = t0; tt < t1; ++tt, ++it) {
            const int s = it % STAGES, use = it / STAGES;
            mbar_wait(full_bar(s), use & 1, abort_flag, p.status, kWaitLimitNs);
            const uint32_t kbase = smem_base + s * C::STAGE_BYTES;
            const uint32_t vbase = kbase + C::KBOX * C::BOX_BYTES;
            const int jtile = (int)(tt * C::TK);

            // ---- S^T (16 keys x 8 rows) = K Q^T
            float sc[4] = {0.f, 0.f, 0.f, 0.f};
            {
                const int key = kw + (lane & 7) + ((lane >> 3) & 1) * 8;
                const uint32_t row = kbase + key * 128;
                const int sw = key & 7;
#pragma unroll
                for (int kk = 0; kk < DQK / 16; ++kk) {
                    const int d = kk * 16 + ((lane >> 4) & 1) * 8;
                    const uint32_t addr = row + (d >> 6) * C::BOX_BYTES + ((((d & 63) >> 3) ^ sw) << 4);
                    uint32_t a0, a1, a2, a3;
                    ldmatrix_x4(addr, a0, a1, a2, a3);
                    Mma<T>::run(sc, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
                }
            }
            // ---- mask + online softmax (base 2)
            const int j0 = jtile + kw + (lane >> 2), j1 = j0 + 8;
            float s0 = j0 <= lim[0] ? sc[0] * p.scale_log2 : -INFINITY;
            float s1 = j0 <= lim[1] ? sc[1] * p.scale_log2 : -INFINITY;
            float s2 = j1 <= lim[0] ? sc[2] * p.scale_log2 : -INFINITY;
            float s3 = j1 <= lim[1] ? sc[3] * p.scale_log2 : -INFINITY;
            float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
            }
            const float mn0 = fmaxf(m[0], mx0), mn1 = fmaxf(m[1], mx1);
            const float base0 = mn0 == -INFINITY ? 0.f : mn0;
            const float base1 = mn1 == -INFINITY ? 0.f : mn1;
            const float al0 = fast_exp2(m[0] - base0), al1 = fast_exp2(m[1] - base1);
            const float p0 = fast_exp2(s0 - base0), p2 = fast_exp2(s2 - base0);
            const float p1 = fast_exp2(s1 - base1), p3 = fast_exp2(s3 - base1);
            l[0] = l[0] * al0 + (p0 + p2);
            l[1] = l[1] * al1 + (p1 + p3);
            m[0] = mn0;
            m[1] = mn1;
#pragma unroll
            for (int t = 0; t < DV / 16; ++t) {
                acc[t][0] *= al0;
                acc[t][1] *= al1;
                acc[t][2] *= al0;
                acc[t][3] *= al1;
            }
            const uint32_t pb0 = movmatrix_trans(Mma<T>::pack(p0, p1));  // keys 0-7
            const uint32_t pb1 = movmatrix_trans(Mma<T>::pack(p2, p3));  // keys 8-15

            // ---- cache slots at or beyond this batch's length may hold
            // anything (NaN included): zero those V rows so 0 * V stays 0.
            if (p.seqlens && jtile + C::TK > n) {
                for (int idx = lane; idx < 16 * C::VBOX * 8; idx += 32) {
                    const int key = kw + idx / (C::VBOX * 8);
                    const int rem = idx % (C::VBOX * 8);
                    if (jtile + key >= n) {
                        const uint32_t a = vbase + (rem >> 3) * C::BOX_BYTES + key * 128 + (rem & 7) * 16;
                        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
            }
            // ---- O^T (DV x 8 rows) += V^T P^T
            {
                const int key = kw + (lane & 7) + ((lane >> 4) & 1) * 8;
                const uint32_t row = vbase + key * 128;
                const int sw = key & 7;
#pragma unroll
                for (int t = 0; t < DV / 16; ++t) {
                    const int d = t * 16 + ((lane >> 3) & 1) * 8;
                    const uint32_t addr = row + (d >> 6) * C::BOX_BYTES + ((((d & 63) >> 3) ^ sw) << 4);
                    uint32_t a0, a1, a2, a3;
                    ldmatrix_x4_trans(addr, a0, a1, a2, a3);
                    Mma<T>::run(acc[t], a0, a1, a2, a3, pb0, pb1);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_bar(s));
        }

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
        consumer_sync();
        // per-warp weight 2^(m_w - M) / L for this lane's two rows
        float f[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int r = r_lo + e;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm_m[w * kRowsPerCta + r]);
            float L = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) {
                    const float mw = sm_m[w * kRowsPerCta + r];
                    if (mw != -INFINITY) L += sm_l[w * kRowsPerCta + r] * fast_exp2(mw - M);
                }
            }
            f[e] = (L > 0.f && m[e] != -INFINITY) ? fast_exp2(m[e] - M) / L : 0.f;
        }
        // tree merge of the four warps' scaled accumulators through 2 buffers
        auto scatter = [&](float *buf) {
#pragma unroll
            for (int t = 0; t < DV / 16; ++t) {
                const int d = t * 16 + (lane >> 2);
                buf[r_lo * C::RED_STRIDE + d] = acc[t][0] * f[0];
                buf[(r_lo + 1) * C::RED_STRIDE + d] = acc[t][1] * f[1];
                buf[r_lo * C::RED_STRIDE + d + 8] = acc[t][2] * f[0];
                buf[(r_lo + 1) * C::RED_STRIDE + d + 8] = acc[t][3] * f[1];
            }
        };
        float *buf_w = red + (warp & 1) * kRowsPerCta * C::RED_STRIDE;
        if (warp >= 2) scatter(buf_w);
        consumer_sync();
        if (warp < 2) {
#pragma unroll
            for (int t = 0; t < DV / 16; ++t) {
                const int d = t * 16 + (lane >> 2);
                acc[t][0] = acc[t][0] * f[0] + buf_w[r_lo * C::RED_STRIDE + d];
                acc[t][1] = acc[t][1] * f[1] + buf_w[(r_lo + 1) * C::RED_STRIDE + d];
                acc[t][2] = acc[t][2] * f[0] + buf_w[r_lo * C::RED_STRIDE + d + 8];
                acc[t][3] = acc[t][3] * f[1] + buf_w[(r_lo + 1) * C::RED_STRIDE + d + 8];
            }
        }
        consumer_sync();
        if (warp < 2) {
            f[0] = f[1] = 1.f;
            scatter(buf_w);
        }
        consumer_sync();
        {
            const int r = ct / 16;
            const int d0 = (ct % 16) * EPT;
            float v[EPT];
#pragma unroll
            for (int e = 0; e < EPT; ++e)
                v[e] = red[r * C::RED_STRIDE + d0 + e] + red[(kRowsPerCta + r) * C::RED_STRIDE + d0 + e];
            float M = -INFINITY, L = 0.f;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm_m[w * kRowsPerCta + r]);
            if (M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) {
                    const float mw = sm_m[w * kRowsPerCta + r];
                    if (mw != -INFINITY) L += sm_l[w * kRowsPerCta + r] * fast_exp2(mw - M);
                }
            }
            const float lse2 = L > 0.f ? M + log2f(L) : -INFINITY;
            const int rr = rb * kRowsPerCta + r;
            if (whole) {
                if (rr < p.R) {
                    const int hq = hkv * p.g + rr / p.Lq, i = rr % p.Lq;
                    T *op = og + b * p.o_sb + (long long)i * p.o_sl + (long long)hq * p.o_sh + d0;
#pragma unroll
                    for (int e = 0; e < EPT; e += 2) {
                        const uint32_t w2 = Mma<T>::pack(v[e], v[e + 1]);
                        *reinterpret_cast<uint32_t *>(op + e) = w2;
                    }
                    if (p.lse && (ct % 16) == 0)
                        p.lse[((long long)b * p.Hq + hq) * p.Lq + i] = lse2 * 0.69314718055994531f;
                }
            } else {
                float *wo = p.ws_o + (((long long)blockIdx.x * 2 + slot) * kRowsPerCta + r) * DV + d0;
#pragma unroll
                for (int e = 0; e < EPT; e += 4)
                    *reinterpret_cast<float4 *>(wo + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                if ((ct % 16) == 0)
                    p.ws_lse[((long long)blockIdx.x * 2 + slot) * kRowsPerCta + r] = lse2;
            }
        }
        consumer_sync();  // red / sm_m / sm_l are reused by the next segment
    }
}

// ---------------------------------------------------------------------- registry
template <typename T, int DQK, int DV, int STAGES>
static void fill(KernelInfo *out, int variant) {
    using C = MmaCfg<DQK, DV, STAGES>;
    out->fn = reinterpret_cast<const void *>(&splitkv_mma_kernel<T, DQK, DV, STAGES>);
    out->threads = kThreads;
    out->smem = C::SMEM;
    out->tile_keys = C::TK;
    out->stages = STAGES;
    out->variant = variant;
}

bool get_mma_kernel(int dtype, int dqk, int dv, KernelInfo *out) {
    constexpr int kMma = 1;
    if (dtype == 0) {
        if (dqk == 64 && dv == 64) { fill<__half, 64, 64, 5>(out, kMma); return true; }
        if (dqk == 128 && dv == 128) { fill<__half, 128, 128, 3>(out, kMma); return true; }
        if (dqk == 192 && dv == 128) { fill<__half, 192, 128, 2>(out, kMma); return true; }
    } else if (dtype == 1) {
        if (dqk == 64 && dv == 64) { fill<__nv_bfloat16, 64, 64, 5>(out, kMma); return true; }
        if (dqk == 128 && dv == 128) { fill<__nv_bfloat16, 128, 128, 3>(out, kMma); return true; }
        if (dqk == 192 && dv == 128) { fill<__nv_bfloat16, 192, 128, 2>(out, kMma); return true; }
    }
    return false;
}

}  // namespace fa
