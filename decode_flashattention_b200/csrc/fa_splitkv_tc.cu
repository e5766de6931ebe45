// fa_splitkv_tc.cu -- the split-KV kernel on the 5th-generation tensor cores,
// for 9 to 64 packed query rows per kv head (GQA groups times speculative
// query positions: g * Lq rows that all read the same K / V).
//
// Same work partition, producer and combine as the mma.sync kernel
// (fa_splitkv.cuh, fa_combine.cu): one CTA per SM walks a contiguous piece of
// the key-tile space; a unit is (batch, block of NR packed rows, kv head), so
// the g * Lq rows of a GQA group are one unit and K / V are streamed once for
// all of them.  Per 128-key tile, with the keys on the 128-row M side of the
// products (the packed rows are too few to fill it):
//
//   S^T = K Q^T      tcgen05.mma, M = 128 keys, N = NR rows, K = head dim;
//                    A = K and B = Q, both K-major in shared memory (128-byte
//                    swizzle); fp32 accumulator in TMEM (lane = key),
//                    double-buffered so the next tile's product runs during
//                    this tile's softmax
//   softmax          four warps, one thread per key (TMEM lane): mask, then
//                    the base-2 online softmax with one running max m per row
//                    shared by all 128 threads; m moves only when some score
//                    exceeds it by more than 2^8 (a flag exchanged once per
//                    tile), and then O and the sums are rescaled
//   P^T -> smem      each thread writes its key's row of P^T (16-bit, N-major,
//                    128-byte swizzle)
//   O^T += V^T P^T   tcgen05.mma, M = 128 head dims, N = 64 (rows, zero
//                    padded), K = 16 keys per product; A = V (MN-major from
//                    the TMA stage), B = P^T (MN-major); O^T stays in TMEM
//                    (lane = head dim) for the whole segment
//
// (the tiled online softmax with its running max and sum and the split-KV
// partials merged by log-sum-exp: "昇腾CANN上的FlashAttention工程实战" and the
// MXFlashAttn README's split-KV decode kernel; the Cube / Vector split of the
// ops-transformer walkthrough mapped onto the tensor core and the CUDA cores.)
// At the end of a segment the row sums are reduced across the 128 threads and
// the epilogue reads O^T (thread = head dim) and writes the final O / lse of a
// unit finished here, or the normalised partial and its log2-sum-exp.
//
// Warps: 0-3 softmax / epilogue (TMEM lanes 0-127), 4 the TMA producer, 5 the
// MMA issuer (one thread).  Every wait is bounded; on a timeout the CTA records
// it, waits (bounded) for its last tensor-core work and copies, and frees its
// TMEM before returning.
#include <type_traits>

#include "fa.h"
#include "fa_splitkv.cuh"
#include "fa_tcgen05.cuh"

namespace fa {

namespace tcd {
constexpr int kSoftmaxWarps = 4;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreads = 192;
constexpr float kLazyMax = 8.f;      // log2 of the largest p before a row's max moves
constexpr float kPadMax = 1e30f;     // running max of a padding row: its p is 0 and it never moves
constexpr uint32_t kTmemCols = 256;  // S^T buffers at columns 0 and 64, O^T at 128
constexpr int kPvN = 64;             // N of the PV products (rows, zero padded)
}  // namespace tcd

template <int DQK, int DV, int NR, int KS, int VS>
struct TcCfg {
    static constexpr bool ILV = false;  // paged K / V in the plain per-chunk layout
    static constexpr int TK = 128;
    static constexpr int TK_SHIFT = 7;
    static constexpr int KBOX = DQK / 64;
    static constexpr int VBOX = DV / 64;
    static constexpr int BOX_BYTES = TK * 128;                      // 128 keys x 64 elements
    static constexpr int K_BYTES = KBOX * BOX_BYTES;                // K of one tile
    static constexpr int V_BYTES = VBOX * BOX_BYTES;                // V of one tile
    static constexpr int Q_BOX = NR * 128;                          // NR rows x 64 elements
    static constexpr int Q_BYTES = KBOX * Q_BOX;
    static constexpr int P_BYTES = TK * 128;                        // P^T: 128 keys x 64 rows
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + KS * K_BYTES;
    static constexpr int OFF_Q = OFF_V + VS * V_BYTES;
    static constexpr int OFF_P = OFF_Q + Q_BYTES;
    static constexpr int OFF_META = OFF_P + P_BYTES;
    static constexpr int NBARS = 2 * KS + 2 * VS + 10;
    static constexpr int OFF_BAR = OFF_META + kMetaRing * (int)sizeof(StageMeta);
    static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;            // tmem base, abort flag, tile flags [2][4]
    static constexpr int OFF_M = (OFF_MISC + 48 + 15) & ~15;        // running max per row [NR]
    static constexpr int OFF_A = OFF_M + NR * 4;                    // rescale factors / row sums [NR]
    static constexpr int OFF_LIM = OFF_A + NR * 4;                  // last visible key per row [NR]
    static constexpr int OFF_RED = OFF_LIM + NR * 4;                // per-warp row maxima / sums [4][NR]
    static constexpr int OFF_OOFF = OFF_RED + 4 * NR * 4;           // output row offsets [NR] (elements)
    static constexpr int OFF_LOFF = OFF_OOFF + NR * 8;              // lse offsets [NR] (-1: none)
    static constexpr int SMEM_USED = OFF_LOFF + NR * 8;
    // the dynamic shared memory base is at least 16-byte aligned, so 1008
    // bytes of slack always reach the next 1024-byte boundary
    static constexpr int SMEM = SMEM_USED + 1008;
    static_assert(DQK % 64 == 0 && DV == 128, "instances: head dims (128 | 192, 128)");
    static_assert(NR % 16 == 0 && NR >= 16 && NR <= tcd::kPvN, "16 to 64 packed rows (N of the S products)");
    static_assert(Q_BOX % 1024 == 0 && OFF_V % 1024 == 0 && OFF_Q % 1024 == 0 && OFF_P % 1024 == 0,
                  "swizzle atoms on 1024-byte boundaries");
    static_assert(SMEM <= 232448, "fits the 227 KB per-CTA shared memory limit");
};

// Maximum over the warp's 32 lanes (sm_100 warp reduction on fp32; NaN inputs
// are ignored, -inf is the identity).
__device__ __forceinline__ float warp_max_f32(float v) {
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
}

// Row sums of 32 rows over the warp's 32 lanes (v[r]: this lane's part of row
// r; v is consumed): a reduce-scatter butterfly -- at each step a lane keeps
// one half of its rows and adds its partner's copy of that half -- after
// which lane r holds the warp's sum of row r.  31 shuffles for 32 rows.
__device__ __forceinline__ float warp_row_sums32(float (&v)[32]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int half = 16; half >= 1; half >>= 1) {
        const bool up = (lane & half) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = up ? v[i] : v[i + half];
            const float keep = up ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, half);
        }
    }
    return v[0];
}

template <typename T, int DQK, int DV, int NR, int KS, int VS>
__global__ void __launch_bounds__(tcd::kThreads, 1)
    splitkv_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const Params p) {
    using namespace pf;
    using C = TcCfg<DQK, DV, NR, KS, VS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    // K slots: kfull (TMA bytes + the producer's arrival), kempty (the S
    // products' commit); V slots: vfull, vempty (the PV products' commit); the
    // tile headers are in their own ring, meta[it % kMetaRing]
    const uint32_t kfull0 = bar(0), kempty0 = bar(KS), vfull0 = bar(2 * KS), vempty0 = bar(2 * KS + VS);
    auto kfull = [&](int s) { return kfull0 + 8u * s; };
    auto kempty = [&](int s) { return kempty0 + 8u * s; };
    auto vfull = [&](int s) { return vfull0 + 8u * s; };
    auto vempty = [&](int s) { return vempty0 + 8u * s; };
    constexpr int B0 = 2 * KS + 2 * VS;
    const uint32_t sfull0 = bar(B0), sfree0 = bar(B0 + 2);
    const uint32_t pready = bar(B0 + 4), pdone = bar(B0 + 5), ofree = bar(B0 + 6);
    const uint32_t qfree = bar(B0 + 7), drain = bar(B0 + 8), syncb = bar(B0 + 9);
    StageMeta *meta = reinterpret_cast<StageMeta *>(smem + C::OFF_META);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    volatile int *flag_sh = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 16);  // [2][4]
    float *m_sh = reinterpret_cast<float *>(smem + C::OFF_M);
    float *a_sh = reinterpret_cast<float *>(smem + C::OFF_A);
    int *lim_sh = reinterpret_cast<int *>(smem + C::OFF_LIM);
    float *red_sh = reinterpret_cast<float *>(smem + C::OFF_RED);
    long long *ooff_sh = reinterpret_cast<long long *>(smem + C::OFF_OOFF);
    long long *loff_sh = reinterpret_cast<long long *>(smem + C::OFF_LOFF);

    if (tid == 0) {
        for (int s = 0; s < KS; ++s) {
            mbar_init(kfull(s), 1);
            mbar_init(kempty(s), 1);
        }
        for (int s = 0; s < VS; ++s) {
            mbar_init(vfull(s), 1);
            mbar_init(vempty(s), 1);  // one tcgen05.commit after the tile's PV products
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(sfull0 + 8u * b, 1);
            mbar_init(sfree0 + 8u * b, tcd::kSoftmaxWarps);
        }
        mbar_init(pready, tcd::kSoftmaxWarps);
        mbar_init(pdone, 1);
        mbar_init(ofree, tcd::kSoftmaxWarps);
        mbar_init(qfree, 1);
        mbar_init(drain, 1);
        mbar_init(syncb, tcd::kSoftmaxWarps);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == tcd::kProducerWarp && lane == 0) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(tcd::kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if constexpr (NR < tcd::kPvN) {
        // P^T's padding rows (columns NR..63 of every key's 128-byte row) stay
        // zero for the whole kernel: the PV products read them as N columns
        if (warp < tcd::kSoftmaxWarps) {
            for (int c = NR / 8; c < 8; ++c) {
                const uint32_t a = sb + C::OFF_P + tid * 128 + ((c ^ (tid & 7)) << 4);
                asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
            }
            fence_proxy_async_smem();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    constexpr bool bf16 = std::is_same<T, __nv_bfloat16>::value;

    if (warp == tcd::kProducerWarp) {
        // ============================================================ producer warp
        // The unit's NR packed query rows go into the single Q slot in the
        // K-major 128-byte-swizzle layout (rows past g * Lq and dims past the
        // call's head dim are zero), once the previous segment's S products,
        // which read the slot, are done.
        const T *__restrict__ qg = reinterpret_cast<const T *>(p.q);
        auto q_write = [&](int s, int seg, int b, int rb, int hkv, const BatchGeom &G) {
            (void)s;
            bool ok = seg == 0 || mbar_wait(qfree, (seg - 1) & 1, abort_flag, p.status, p.wait_limit_ns);
            if (!__all_sync(0xffffffffu, ok)) return false;
            const uint32_t qs = sb + C::OFF_Q;
            for (int idx = lane; idx < NR * (DQK / 8); idx += 32) {
                const int r = idx / (DQK / 8), c = idx % (DQK / 8);
                const int rq = rb * NR + r;
                const T *src = qg;
                uint32_t nbytes = 0;
                if (rq < G.R && c * 8 < p.dqk) {
                    const int hq = hkv * p.g + rq / G.Lq, i = rq % G.Lq;
                    src = qg + b * p.q_sb + (long long)(G.q0 + i) * p.q_sl + (long long)hq * p.q_sh + c * 8;
                    nbytes = 16;
                }
                cp_async_16(qs + (c >> 3) * C::Q_BOX + r * 128 + (((c & 7) ^ (r & 7)) << 4), src, nbytes);
            }
            asm volatile("cp.async.wait_all;" ::: "memory");
            fence_proxy_async_smem();  // the tensor core reads the slot through the async proxy
            return true;
        };
        const RingLayout ring = {sb + C::OFF_K, (uint32_t)C::K_BYTES, sb + C::OFF_V, (uint32_t)C::V_BYTES,
                                 kfull0, kempty0, vfull0, vempty0};
        splitkv_produce<C, KS, VS>(&tmK, &tmV, p, ring, meta, abort_flag, q_write);
    } else if (warp == tcd::kMmaWarp) {
        // ============================================================ MMA issue (one thread)
        if (lane == 0) {
            const uint32_t idesc_s = instr_desc(bf16, 128, NR, false, false);        // S^T: K-major K and Q
            const uint32_t idesc_o = instr_desc(bf16, 128, tcd::kPvN, true, true);    // O^T: MN-major V and P^T
            const uint64_t dq0 = smem_desc(sb + C::OFF_Q, 16, 1024);
            const uint64_t dk0 = smem_desc(sb + C::OFF_K, 16, 1024);                // K slot 0
            const uint64_t dv0 = smem_desc(sb + C::OFF_V, C::BOX_BYTES, 1024);      // V slot 0
            const uint64_t dp0 = smem_desc(sb + C::OFF_P, C::BOX_BYTES, 1024);
            auto wait = [&](uint32_t b, uint32_t parity) {
                return mbar_wait(b, parity, abort_flag, p.status, p.wait_limit_ns);
            };
            // tile j's PV products (P^T(j) written, the O^T of its segment free)
            int pv_seg = 0;
            bool pv_first = false, pending = false;
            auto issue_pv = [&](int j) {
                const int vs = j % VS;
                if (!wait(pready, j & 1) || !wait(vfull(vs), (j / VS) & 1)) return false;
                if (pv_first && pv_seg > 0 && !wait(ofree, (pv_seg - 1) & 1)) return false;
                tc_fence_after();
                const uint64_t dv = dv0 + (uint64_t)((vs * C::V_BYTES) >> 4);
#pragma unroll
                for (int ks = 0; ks < C::TK / 16; ++ks)
                    umma(tmem + 128, dv + (uint64_t)((ks * 2048) >> 4), dp0 + (uint64_t)((ks * 2048) >> 4), idesc_o,
                         (pv_first && ks == 0) ? 0u : 1u);
                umma_commit(pdone);
                umma_commit(vempty(vs));  // the tile's V is read
                return true;
            };
            int it = 0, seg = -1;
            bool ok = true;
            for (;; ++it) {
                const int s = it % KS, use = it / KS;
                // while this tile's K is still landing, the previous tile's PV
                // can go first (it frees a V slot sooner)
                if (pending && !mbar_try_wait(kfull(s), use & 1)) {
                    if (!(ok = issue_pv(it - 1))) break;
                    pending = false;
                }
                if (!(ok = wait(kfull(s), use & 1))) break;
                const StageMeta md = meta[it % kMetaRing];
                if (md.flags & kMetaDone) break;
                if (md.flags & kMetaFirst) ++seg;
                // S^T(it) into buffer it & 1, last read by the softmax of tile it - 2
                if (it >= 2 && !(ok = wait(sfree0 + 8u * (it & 1), ((it >> 1) - 1) & 1))) break;
                tc_fence_after();
                const uint64_t dk = dk0 + (uint64_t)((s * C::K_BYTES) >> 4);
#pragma unroll
                for (int kk = 0; kk < DQK / 16; ++kk) {
                    const uint32_t ok_ = (uint32_t)(((kk >> 2) * C::BOX_BYTES + (kk & 3) * 32) >> 4);
                    const uint32_t oq = (uint32_t)(((kk >> 2) * C::Q_BOX + (kk & 3) * 32) >> 4);
                    umma(tmem + (uint32_t)((it & 1) * 64), dk + ok_, dq0 + oq, idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(sfull0 + 8u * (it & 1));
                umma_commit(kempty(s));  // the tile's K is read once its S products are done
                if (md.flags & kMetaLast) umma_commit(qfree);  // the segment's last read of the Q slot
                if (pending && !(ok = issue_pv(it - 1))) break;
                pending = true;
                pv_seg = seg;
                pv_first = (md.flags & kMetaFirst) != 0;
            }
            if (ok && pending) issue_pv(it - 1);
            // every product this thread issued is done before TMEM can be freed
            umma_commit(drain);
            volatile int no_abort = 0;
            mbar_wait(drain, 0, &no_abort, p.status, p.wait_limit_ns);
        }
        __syncwarp();
    } else {
        // ============================================================ softmax / epilogue warps
        pdl_wait_primary();  // outputs and workspace are written below
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const uint32_t prow = sb + C::OFF_P + tid * 128;  // this key's row of P^T
        uint32_t sync_phase = 0;
        auto csync = [&]() { return consumer_sync_bounded(syncb, sync_phase, abort_flag, p.status, p.wait_limit_ns); };
        T *__restrict__ og = reinterpret_cast<T *>(p.o);
        float l[NR];
        int minlim = 0, rreal = 0;
        BatchGeom G = {0, 0, 0, 0, 0};
        for (int it = 0;; ++it) {
            // The tile header (and V) through the V slot's barrier: a V slot is
            // refilled only after this tile's PV, which needs this group's P, so
            // the wait can never fall a whole phase behind -- unlike a K slot,
            // which the S products free two tiles ahead of the softmax.
            bool ok = mbar_wait(vfull(it % VS), (it / VS) & 1, abort_flag, p.status, p.wait_limit_ns);
            if (!__all_sync(0xffffffffu, ok)) break;
            const StageMeta md = meta[it % kMetaRing];
            if (md.flags & kMetaDone) break;
            const bool first = (md.flags & kMetaFirst) != 0;
            if (first) {
                // the unit's rows: last visible key (bottom-right causal corner),
                // running max; padding rows get lim -1 and a max nothing exceeds
                G = batch_geom(p, md.b);
                rreal = G.R - md.rb * NR < NR ? G.R - md.rb * NR : NR;
                if (tid < NR) {
                    int lim = -1;
                    float m0 = tcd::kPadMax;
                    long long oo = 0, lo = -1;
                    if (tid < rreal) {
                        const int rg = md.rb * NR + tid;
                        const int i = rg % G.Lq, hq = md.hkv * p.g + rg / G.Lq;
                        lim = G.n - 1;
                        if (p.causal && i + G.n - G.Lq < lim) lim = i + G.n - G.Lq;
                        m0 = -INFINITY;
                        oo = md.b * p.o_sb + (long long)(G.q0 + i) * p.o_sl + (long long)hq * p.o_sh;
                        if (p.lse) lo = md.b * p.lse_sb + (long long)hq * p.lse_sh + G.q0 + i;
                    }
                    lim_sh[tid] = lim;
                    m_sh[tid] = m0;
                    ooff_sh[tid] = oo;
                    loff_sh[tid] = lo;
                }
#pragma unroll
                for (int r = 0; r < NR; ++r) l[r] = 0.f;
                if (!csync()) break;
                minlim = 1 << 30;
                for (int r = 0; r < rreal; ++r) minlim = min(minlim, lim_sh[r]);
            }
            // ---- S^T(it): this thread's key against the NR rows
            ok = mbar_wait(sfull0 + 8u * (it & 1), (it >> 1) & 1, abort_flag, p.status, p.wait_limit_ns);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            float x[NR];
            {
                uint32_t v[NR / 16][16];
#pragma unroll
                for (int c = 0; c < NR / 16; ++c) tmem_ld16(tmem + (uint32_t)((it & 1) * 64 + c * 16) + lane_off, v[c]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < NR / 16; ++c)
#pragma unroll
                    for (int e = 0; e < 16; ++e) x[c * 16 + e] = __uint_as_float(v[c][e]) * p.scale_log2;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(sfree0 + 8u * (it & 1));
            const int key = md.tile * C::TK + tid;
            if (key > minlim) {  // past some row's last visible key (or past the keys)
#pragma unroll
                for (int r = 0; r < NR; ++r) x[r] = key <= lim_sh[r] ? x[r] : -INFINITY;
            }
            // ---- does any row's max move?  One flag per warp, exchanged once
            bool need = false;
#pragma unroll
            for (int r = 0; r < NR; r += 4) {
                const float4 m4 = *reinterpret_cast<const float4 *>(m_sh + r);
                need |= (x[r] > m4.x + tcd::kLazyMax) | (x[r + 1] > m4.y + tcd::kLazyMax) |
                        (x[r + 2] > m4.z + tcd::kLazyMax) | (x[r + 3] > m4.w + tcd::kLazyMax);
            }
            need = __any_sync(0xffffffffu, need);
            if (lane == 0) flag_sh[(it & 1) * 4 + warp] = need ? 1 : 0;
            if (!csync()) break;
            const int fb = (it & 1) * 4;
            if (flag_sh[fb] | flag_sh[fb + 1] | flag_sh[fb + 2] | flag_sh[fb + 3]) {
                // per-row max over this warp's 32 keys (one warp reduction per
                // row), then over the 4 warps
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    const float v = warp_max_f32(x[r]);
                    if (lane == (r & 31)) red_sh[warp * NR + r] = v;
                }
                if (!csync()) break;
                if (tid < NR) {
                    const float mo = m_sh[tid];
                    const float mx = fmaxf(fmaxf(red_sh[tid], red_sh[NR + tid]),
                                           fmaxf(red_sh[2 * NR + tid], red_sh[3 * NR + tid]));
                    const float mn = mx > mo + tcd::kLazyMax ? mx : mo;
                    a_sh[tid] = mo == -INFINITY ? 0.f : fast_exp2(mo - mn);
                    m_sh[tid] = mn;
                }
                if (!csync()) break;
                bool moved = false;
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    const float a = a_sh[r];
                    l[r] *= a;
                    moved |= a != 1.f;
                }
                if (!first && moved) {  // uniform: every thread reads the same factors
                    // O^T holds PV(it - 1)'s sums once that product is done
                    ok = mbar_wait(pdone, (it - 1) & 1, abort_flag, p.status, p.wait_limit_ns);
                    if (!__all_sync(0xffffffffu, ok)) break;
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < NR / 16; ++c) {
                        uint32_t v[16];
                        tmem_ld16(tmem + 128u + (uint32_t)(c * 16) + lane_off, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * a_sh[c * 16 + e]);
                        tmem_st16(tmem + 128u + (uint32_t)(c * 16) + lane_off, v);
                    }
                    tmem_wait_st();
                }
            }
            // ---- cache slots at or beyond the batch's length may hold anything
            // (NaN included): zero this key's V row so 0 * V stays 0
            if ((p.seqlens || p.cu_q) && key >= G.n) {  // (this tile's V has landed: vfull above)
                const uint32_t vrow = sb + C::OFF_V + (it % VS) * C::V_BYTES + tid * 128;
#pragma unroll
                for (int c = 0; c < C::VBOX * 8; ++c) {
                    const uint32_t a = vrow + (c >> 3) * C::BOX_BYTES + (c & 7) * 16;
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
                }
            }
            // ---- P^T row of this key; the buffer is free once PV(it - 1) is done
            if (it > 0) {
                ok = mbar_wait(pdone, (it - 1) & 1, abort_flag, p.status, p.wait_limit_ns);
                if (!__all_sync(0xffffffffu, ok)) break;
            }
#pragma unroll
            for (int c = 0; c < NR / 8; ++c) {
                const float4 ma = *reinterpret_cast<const float4 *>(m_sh + c * 8);
                const float4 mb = *reinterpret_cast<const float4 *>(m_sh + c * 8 + 4);
                const float mm[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
                float pv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float base = mm[e] == -INFINITY ? 0.f : mm[e];
                    pv[e] = fast_exp2(x[c * 8 + e] - base);
                    l[c * 8 + e] += pv[e];
                }
                const uint32_t a = prow + ((c ^ (tid & 7)) << 4);
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(Mma<T>::pack(pv[0], pv[1])),
                             "r"(Mma<T>::pack(pv[2], pv[3])), "r"(Mma<T>::pack(pv[4], pv[5])),
                             "r"(Mma<T>::pack(pv[6], pv[7]))
                             : "memory");
            }
            fence_proxy_async_smem();  // P^T and zeroed V rows are read by the tensor core
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(pready);
            if (!(md.flags & kMetaLast)) continue;

            // ================================================ segment epilogue
            // Row sums over the 128 keys (a reduce-scatter butterfly per warp,
            // then the four warps' sums), then O^T read from TMEM -- this
            // thread's lane is head dim tid, so each row of O is written by
            // 128 consecutive threads -- scaled by 1 / sum; row offsets were
            // worked out at the segment's start.
            ok = mbar_wait(pdone, it & 1, abort_flag, p.status, p.wait_limit_ns);  // the last PV
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < NR; h += 32) {
                float v[32];
#pragma unroll
                for (int r = 0; r < 32; ++r) v[r] = h + r < NR ? l[h + r] : 0.f;
                const float rs = warp_row_sums32(v);
                if (h + lane < NR) red_sh[warp * NR + h + lane] = rs;
            }
            if (!csync()) break;
            const bool whole = (md.flags & kMetaWhole) != 0;
            const long long wbase = ((long long)md.piece * 2 + md.slot) * NR;
            if (tid < rreal) {
                const float L = (red_sh[tid] + red_sh[NR + tid]) + (red_sh[2 * NR + tid] + red_sh[3 * NR + tid]);
                a_sh[tid] = L > 0.f ? 1.f / L : 0.f;
                const float lse2 = L > 0.f ? m_sh[tid] + log2f(L) : -INFINITY;
                if (whole) {
                    if (loff_sh[tid] >= 0) p.lse[loff_sh[tid]] = L > 0.f ? lse2 * 0.69314718055994531f : -INFINITY;
                } else {
                    p.ws_lse[wbase + tid] = lse2;
                }
            }
            if (!csync()) break;
#pragma unroll
            for (int c = 0; c < NR / 16; ++c) {  // 16 rows (TMEM columns) at a time
                uint32_t ov[16];
                tmem_ld16(tmem + 128u + (uint32_t)(c * 16) + lane_off, ov);
                tmem_wait_ld();
                if (whole) {
                    if (tid < p.dv) {
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            if (c * 16 + e < rreal)
                                og[ooff_sh[c * 16 + e] + tid] = Cvt<T>::from(__uint_as_float(ov[e]) * a_sh[c * 16 + e]);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        if (c * 16 + e < rreal)
                            p.ws_o[(wbase + c * 16 + e) * DV + tid] = __uint_as_float(ov[e]) * a_sh[c * 16 + e];
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ofree);  // O^T may be overwritten by the next segment's products
            if (md.flags & kMetaFinal) break;
            if (!csync()) break;  // m_sh / lim_sh / a_sh are rewritten by the next segment
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tcd::kTmemCols)
                     : "memory");
    }
}

template <typename T, int DQK, int DV, int NR, int KS, int VS>
static void fill_tc(KernelInfo *out) {
    using C = TcCfg<DQK, DV, NR, KS, VS>;
    out->fn = reinterpret_cast<const void *>(&splitkv_tc_kernel<T, DQK, DV, NR, KS, VS>);
    out->threads = tcd::kThreads;
    out->smem = C::SMEM;
    out->tile_keys = C::TK;
    out->stages = VS;
    out->variant = FA_VARIANT_TCGEN05_SPLIT;
    out->rows = NR;
    out->form = 0;
}

// K slots are released as soon as their S products are done, V slots only
// after the PV products: two K slots, and as many V slots as fit beside the Q
// slot and P^T.
template <typename T>
static bool fill_tc_dims(int dqk, int nr, KernelInfo *out) {
    if (dqk == 128) {
        if (nr == 16) { fill_tc<T, 128, 128, 16, 2, 4>(out); return true; }
        if (nr == 32) { fill_tc<T, 128, 128, 32, 2, 4>(out); return true; }
        if (nr == 64) { fill_tc<T, 128, 128, 64, 2, 3>(out); return true; }
    } else if (dqk == 192) {
        if (nr == 16) { fill_tc<T, 192, 128, 16, 2, 3>(out); return true; }
        if (nr == 32) { fill_tc<T, 192, 128, 32, 2, 3>(out); return true; }
        if (nr == 64) { fill_tc<T, 192, 128, 64, 2, 2>(out); return true; }
    }
    return false;
}

bool get_tc_split_kernel(int dtype, int dqk, int dv, int nr, KernelInfo *out) {
    if (dv != 128) return false;
    if (dtype == 0) return fill_tc_dims<__half>(dqk, nr, out);
    if (dtype == 1) return fill_tc_dims<__nv_bfloat16>(dqk, nr, out);
    return false;
}

}  // namespace fa
