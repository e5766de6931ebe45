// fa_prefill.cu -- dense attention for many packed query rows on the 5th-gen
// tensor cores (tcgen05 + TMEM): the prefill-shaped calls of fa_fwd.
//
// Packed row r of kv head hkv is query head hkv * g + r / Lq at position
// r % Lq (the same packing as the split-KV kernel), so the g heads of a GQA
// group share every K / V tile; a CTA walks all 128-key tiles its rows can
// see (no split, no combine).  Per tile, for a 128-row query tile:
//
//   S  = Q K^T        tcgen05.mma (M 128 rows, N 128 keys, K = head dim),
//                     fp32 accumulator in TMEM
//   softmax           one thread per row reads its S row from TMEM
//                     (tcgen05.ld), masks, and runs the base-2 online
//                     softmax (running max m, sum l in fp32); O in TMEM is
//                     rescaled by 2^(m_old - m_new) (tcgen05.ld / st)
//   O += P V          tcgen05.mma (M 128 rows, N = head dim, K 128 keys),
//                     fp32 accumulator in TMEM
//
// (the tiled online softmax of "昇腾CANN上的FlashAttention工程实战", with the
// Cube / Vector split of the ops-transformer walkthrough mapped onto the
// tensor core and the CUDA cores).  K and V arrive by TMA (128-byte swizzle,
// the canonical K-major layout for K and the MN-major one for V), and
// tcgen05.commit releases a stage once its products are done.  Two kernels:
//
//   prefill3_kernel   one or two query tiles per CTA, a dedicated MMA warp
//                     and a TMA warp; with two tiles one tile's products run
//                     during the other's softmax, with one tile S is
//                     double-buffered; P stays in TMEM (the library's choice)
//   prefill_kernel    an earlier design kept for comparison (reached only by
//                     forcing its form): one query tile per CTA whose four
//                     softmax warps issue the products themselves, S
//                     double-buffered in TMEM, P through shared memory
//
// Every wait is bounded; on a timeout the CTA records the error, waits
// (bounded) for its last tensor-core work and copies, and frees its TMEM
// before returning.
#include <type_traits>

#include "fa.h"
#include "fa_common.cuh"
#include "fa_internal.h"
#include "fa_tcgen05.cuh"

namespace fa {

namespace pf {

constexpr int kRows = 128;       // packed query rows per CTA (MMA M)
constexpr int kD = 128;          // head dim (both products)
constexpr int kStages = 2;
constexpr int kBoxQ = kRows * 128;                  // one 64-column box of 128 rows (bytes): Q and P
constexpr int kTileQ = 2 * kBoxQ;                   // Q: 128 rows x 128 elements
constexpr int NBAR = 2 * kStages + 4;               // full[2], empty[2], s_done[2], o_done, compute sync
constexpr int kThreads = 160;                       // 4 compute warps (TMEM lanes 0-127) + 1 producer
constexpr uint64_t kWaitLimitNs = 4000000000ull;

// Shared-memory layout for KEYS keys per tile.  KEYS = 128: one CTA per SM,
// a 2-stage ring of 64 KB K + V stages, S double-buffered in TMEM (512 columns).
// KEYS = 64: half the stage and P sizes, so two CTAs share an SM (their
// softmax warps interleave on each sub-partition), 256 TMEM columns each; the
// base must then already be 1024-byte aligned (checked at run time) since
// there is no room for alignment slack.
template <int KEYS>
struct Cfg {
    static constexpr int kKeys = KEYS;
    static constexpr int kBoxKV = KEYS * 128;         // one 64-column box of K or V (bytes)
    static constexpr int kTileKV = 2 * kBoxKV;        // K or V tile: KEYS rows x 128 elements
    static constexpr int kStageBytes = 2 * kTileKV;   // K + V
    static constexpr int kPBytes = kRows * KEYS * 2;  // P: 128 rows x KEYS keys
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_P = OFF_Q + kTileQ;
    static constexpr int OFF_KV = OFF_P + kPBytes;
    static constexpr int OFF_BAR = OFF_KV + kStages * kStageBytes;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort flag, 4 warp maxima
    static constexpr int SLACK = KEYS == 128 ? 1024 : 0;
    static constexpr int SMEM = OFF_MISC + 64 + SLACK;
    static constexpr uint32_t kTmemCols = KEYS == 128 ? 512 : 256;  // S x 2 [0, 2 KEYS), O [2 KEYS, 2 KEYS + 128)
    static constexpr int kMinBlocks = KEYS == 128 ? 1 : 2;
    static_assert(SMEM <= 232448, "fits the per-CTA shared memory");
    static_assert(KEYS == 128 || 2 * (SMEM + 1024) <= 233472, "two CTAs fit an SM");
};


}  // namespace pf

template <typename T, int KEYS>
__global__ void __launch_bounds__(pf::kThreads, pf::Cfg<KEYS>::kMinBlocks)
    prefill_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const Params p) {
    using namespace pf;
    using C = Cfg<KEYS>;
    constexpr int kKeys = KEYS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (C::SLACK == 0 && smem != smem_raw) {  // no room to align: the base must already be aligned
        if (tid == 0) atomicOr(p.status, kStatusLayout);
        return;
    }
    const int rb = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
    auto empty_bar = [&](int s) { return smem_u32(&bars[kStages + s]); };
    auto s_bar = [&](int buf) { return smem_u32(&bars[2 * kStages + buf]); };
    const uint32_t o_bar = smem_u32(&bars[2 * kStages + 2]);
    const uint32_t cs_bar = smem_u32(&bars[2 * kStages + 3]);  // bounded sync of the 4 compute warps
    uint32_t cs_phase = 0;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    int *warp_keys = reinterpret_cast<int *>(smem + C::OFF_MISC + 16);

    // ---- this thread's row (compute warps): head, query position, last visible key
    const int r = rb * kRows + tid;  // packed row
    const bool row_live = tid < kRows && r < p.R;
    const int hq = row_live ? hkv * p.g + r / p.Lq : 0;
    const int qi = row_live ? r % p.Lq : 0;
    const int n = p.Lk;
    int lim = -1;  // last visible key of the row
    if (row_live) {
        lim = n - 1;
        if (p.causal) {
            const int c = qi + n - p.Lq;
            lim = c < lim ? c : lim;
        }
    }

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(s_bar(0), 1);
        mbar_init(s_bar(1), 1);
        mbar_init(o_bar, 1);
        mbar_init(cs_bar, 4);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {  // TMEM: S double buffer in columns [0, 256), O in [256, 384)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(C::kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // keys the block's rows can see (tiles to walk)
    {
        int kv = lim + 1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kv = max(kv, __shfl_xor_sync(0xffffffffu, kv, off));
        if (lane == 0 && warp < 4) warp_keys[warp] = kv;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int kmax = max(max(warp_keys[0], warp_keys[1]), max(warp_keys[2], warp_keys[3]));
    const int ntiles = (kmax + kKeys - 1) / kKeys;

    pdl_wait_primary();

    if (warp == 4) {
        // ================================================= producer: K / V tiles by TMA
        if (lane == 0) {
            for (int j = 0; j < ntiles; ++j) {
                const int s = j % kStages, use = j / kStages;
                if (use > 0 && !mbar_wait(empty_bar(s), (use - 1) & 1, abort_flag, p.status, kWaitLimitNs)) break;
                const uint32_t kd = sb + C::OFF_KV + s * C::kStageBytes, vd = kd + C::kTileKV;
                mbar_expect_tx(full_bar(s), C::kStageBytes);
                for (int c = 0; c < 2; ++c) {
                    tma_load_4d_plain(kd + c * C::kBoxKV, &tmK, full_bar(s), c * 64, j * kKeys, hkv, b);
                    tma_load_4d_plain(vd + c * C::kBoxKV, &tmV, full_bar(s), c * 64, j * kKeys, hkv, b);
                }
                mbar_arrive(full_bar(s));
            }
        }
        __syncwarp();
    } else {
        // ================================================= compute warps: one row per thread
        // Q rows into the operand layout (K-major, 128-byte swizzle): row tid,
        // 16-byte chunk c of the head dim at box c / 8, swizzled chunk (c % 8) ^ (tid % 8)
        {
            const T *qg = reinterpret_cast<const T *>(p.q);
            const T *src = qg + b * p.q_sb + (long long)qi * p.q_sl + (long long)hq * p.q_sh;
            for (int c = 0; c < kD / 8; ++c) {
                const uint32_t dst =
                    sb + C::OFF_Q + (c >> 3) * kBoxQ + tid * 128 + ((((c & 7) ^ (tid & 7))) << 4);
                cp_async_16(dst, src + c * 8, row_live ? 16u : 0u);
            }
            asm volatile("cp.async.wait_all;" ::: "memory");
            fence_proxy_async_smem();
        }
        constexpr bool bf16 = std::is_same<T, __nv_bfloat16>::value;
        const uint32_t idesc_s = instr_desc(bf16, kRows, kKeys, false);
        const uint32_t idesc_o = instr_desc(bf16, kRows, kD, true);
        const uint32_t t_o = tmem + 2 * kKeys;  // S buffers at tmem, tmem + kKeys
        // S_jj = Q K_jj^T into S buffer jj % 2, issued by one thread once tile jj
        // has landed (issue_s_ready: the caller knows it has).
        auto issue_s_ready = [&](int jj) -> bool {
            const int st = jj % kStages;
            const uint32_t kbase = sb + C::OFF_KV + st * C::kStageBytes;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
                const uint32_t aoff = (kk >> 2) * kBoxQ + (kk & 3) * 32, boff = (kk >> 2) * C::kBoxKV + (kk & 3) * 32;
                umma(tmem + (jj & 1) * kKeys, smem_desc(sb + C::OFF_Q + aoff, 16, 1024),
                     smem_desc(kbase + boff, 16, 1024), idesc_s, kk > 0);
            }
            umma_commit(s_bar(jj & 1));
            return true;
        };
        auto issue_s = [&](int jj) -> bool {
            const int st = jj % kStages;
            if (!mbar_wait(full_bar(st), (jj / kStages) & 1, abort_flag, p.status, kWaitLimitNs)) return false;
            return issue_s_ready(jj);
        };
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;  // this warp's TMEM lanes
        float m = -INFINITY, l = 0.f;
        // every Q row is in shared memory
        bool ok = consumer_sync_bounded(cs_bar, cs_phase, abort_flag, p.status, kWaitLimitNs);
        if (ok && tid == 0 && ntiles > 0) ok = issue_s(0);

        for (int j = 0; j < ntiles && ok; ++j) {
            const int s = j % kStages;
            const uint32_t vb = sb + C::OFF_KV + s * C::kStageBytes + C::kTileKV;
            // the next tile's S now if its K has landed, else just before this tile's PV
            bool next_issued = false;
            if (tid == 0 && j + 1 < ntiles &&
                mbar_try_wait(full_bar((j + 1) % kStages), ((j + 1) / kStages) & 1)) {
                ok = issue_s_ready(j + 1);
                next_issued = true;
            }
            __syncwarp();
            ok = mbar_wait(s_bar(j & 1), (j >> 1) & 1, abort_flag, p.status, kWaitLimitNs) && ok;
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            tc_fence_after();

            // ---- this row's scores (raw fp32): the four TMEM loads in flight at once
            uint32_t v0[32], v1[32], v2[32], v3[32];
            {
                const uint32_t ts = tmem + (j & 1) * kKeys + lane_off;
                tmem_ld32(ts, v0);
                tmem_ld32(ts + 32, v1);
                if constexpr (kKeys == 128) {
                    tmem_ld32(ts + 64, v2);
                    tmem_ld32(ts + 96, v3);
                }
                tmem_wait_ld();
            }
            float x[kKeys];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                x[e] = __uint_as_float(v0[e]);
                x[32 + e] = __uint_as_float(v1[e]);
                if constexpr (kKeys == 128) {
                    x[64 + e] = __uint_as_float(v2[e]);
                    x[96 + e] = __uint_as_float(v3[e]);
                }
            }
            // mask only where some row of the warp has keys of this tile hidden
            const int key0 = j * kKeys;
            if (!__all_sync(0xffffffffu, key0 + kKeys - 1 <= lim)) {
#pragma unroll
                for (int e = 0; e < kKeys; ++e) x[e] = key0 + e <= lim ? x[e] : -INFINITY;
            }
            // row max with independent chains, in base-2 units (scale > 0)
            // row max: eight independent chains of three-input max
            float mxa[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) mxa[e] = fmaxf(x[2 * e], x[2 * e + 1]);
#pragma unroll
            for (int e = 16; e < kKeys; e += 16)
#pragma unroll
                for (int c = 0; c < 8; ++c) mxa[c] = max3f(mxa[c], x[e + 2 * c], x[e + 2 * c + 1]);
            const float mx = max3f(max3f(mxa[0], mxa[1], mxa[2]), max3f(mxa[3], mxa[4], mxa[5]),
                                   fmaxf(mxa[6], mxa[7])) *
                             p.scale_log2;
            const float mn = fmaxf(m, mx);
            const float base = mn == -INFINITY ? 0.f : mn;
            const float alpha = fast_exp2(m - base);  // 0 while nothing was seen
            // p = 2^(x * scale_log2 - base): one packed FMA per key pair and one
            // ex2 per score; sums in four packed accumulators
            const uint64_t sc2 = pack2f(p.scale_log2, p.scale_log2), nb2 = pack2f(-base, -base);
            uint64_t sum2[4] = {pack2f(0.f, 0.f), pack2f(0.f, 0.f), pack2f(0.f, 0.f), pack2f(0.f, 0.f)};
            uint32_t pk[kKeys / 2];
#pragma unroll
            for (int e = 0; e < kKeys; e += 2) {
                float y0, y1;
                unpack2f(ffma2(pack2f(x[e], x[e + 1]), sc2, nb2), y0, y1);
                const float p0 = fast_exp2(y0), p1 = fast_exp2(y1);
                sum2[(e >> 1) & 3] = fadd2(sum2[(e >> 1) & 3], pack2f(p0, p1));
                pk[e / 2] = Mma<T>::pack(p0, p1);
            }
            float suma[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) unpack2f(sum2[q], suma[2 * q], suma[2 * q + 1]);
            const float sum = ((suma[0] + suma[1]) + (suma[2] + suma[3])) + ((suma[4] + suma[5]) + (suma[6] + suma[7]));
            l = l * alpha + sum;
            m = mn;

            if (j > 0) {
                // the previous PV product is done: O may be rescaled and P rewritten
                ok = mbar_wait(o_bar, (j - 1) & 1, abort_flag, p.status, kWaitLimitNs);
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
                    // O row in 64-column halves (fewer live registers with two CTAs per SM)
#pragma unroll
                    for (int h = 0; h < kD / 64; ++h) {
                        const uint32_t to = t_o + lane_off + h * 64;
                        tmem_ld32(to, v0);
                        tmem_ld32(to + 32, v1);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            v0[e] = __float_as_uint(__uint_as_float(v0[e]) * alpha);
                            v1[e] = __float_as_uint(__uint_as_float(v1[e]) * alpha);
                        }
                        tmem_st32(to, v0);
                        tmem_st32(to + 32, v1);
                    }
                    tmem_wait_st();
                }
            }
            // ---- P row into the operand layout (keys as K, K-major, swizzled)
#pragma unroll
            for (int c = 0; c < kKeys / 8; ++c) {
                const uint32_t dst = sb + C::OFF_P + (c >> 3) * kBoxQ + tid * 128 + ((((c & 7) ^ (tid & 7))) << 4);
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(pk[c * 4]),
                             "r"(pk[c * 4 + 1]), "r"(pk[c * 4 + 2]), "r"(pk[c * 4 + 3])
                             : "memory");
            }
            fence_proxy_async_smem();
            tc_fence_before();
            if (!consumer_sync_bounded(cs_bar, cs_phase, abort_flag, p.status, kWaitLimitNs)) {
                ok = false;
                break;
            }
            if (tid == 0 && j + 1 < ntiles && !next_issued) ok = issue_s(j + 1) && ok;
            if (tid == 0) {  // O += P V
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kKeys / 16; ++kk) {
                    const uint32_t aoff = (kk >> 2) * kBoxQ + (kk & 3) * 32;
                    umma(t_o, smem_desc(sb + C::OFF_P + aoff, 16, 1024), smem_desc(vb + kk * 2048, C::kBoxKV, 1024),
                         idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(o_bar);
                umma_commit(empty_bar(s));
            }
            __syncwarp();
        }

        // ---- epilogue: O / l, lse
        if (ok && ntiles > 0) {
            ok = mbar_wait(o_bar, (ntiles - 1) & 1, abort_flag, p.status, kWaitLimitNs);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
        }
        if (ok) {
            const float inv = l > 0.f ? 1.f / l : 0.f;
            T *og = reinterpret_cast<T *>(p.o) + b * p.o_sb + (long long)qi * p.o_sl + (long long)hq * p.o_sh;
#pragma unroll
            for (int c = 0; c < kD / 32; ++c) {
                uint32_t v[32];
                if (ntiles > 0) {
                    tmem_ld32(t_o + lane_off + c * 32, v);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = 0u;
                }
                if (row_live) {
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        float f[8];
#pragma unroll
                        for (int z = 0; z < 8; ++z) f[z] = __uint_as_float(v[e + z]) * inv;
                        store_row8<T>(og + c * 32 + e, f);
                    }
                }
            }
            if (row_live && p.lse)
                p.lse[b * p.lse_sb + hq * p.lse_sh + qi] = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
        } else if (tid == 0) {
            // timed out: wait (bounded) for the tensor core's last work before TMEM is freed
            volatile int no_abort = 0;
            mbar_wait(o_bar, 0, &no_abort, nullptr, kWaitLimitNs / 8);
            mbar_wait(o_bar, 1, &no_abort, nullptr, kWaitLimitNs / 8);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::kTmemCols) : "memory");
    }
}

// ---------------------------------------------------------------------------
// Two query tiles per CTA with 128-key K / V tiles (the kernel also runs
// with one tile): every QK^T product is M 128 x N 128 x K 16, every PV product
// M 128 x N D x K 16, and per 128 keys the MMA warp issues 32 products (16
// for D = 64) with four commits and two waits.  K and V tiles stream
// separately through a ring of three slots (K(j), V(j), K(j + 1), ...; 128
// keys x D each).  S is single-buffered per group; per tile j the MMA warp
// issues, for group A then group B,
//   PV_g(j) once the group has written P_g(j) (so it has read S_g(j)),
//   S_g(j + 1) right behind it (the tensor core runs one thread's products
//   in order),
// so one group's products run while the other group's softmax does.  P stays
// in TMEM: the softmax writes it (two 16-bit values per 32-bit column) over
// the S columns it has just read, and PV_g(j) takes its A operand from there,
// so P never goes through shared memory.  The softmax keeps a running max m
// that only moves when a tile's max exceeds it by more than 2^8 (p = 2^(s - m)
// then stays below 256, exact in fp32 and representable in the 16-bit P), so
// O is rescaled only on those tiles.
namespace pf3 {
constexpr int kKeys = 128;
constexpr int kSlots = 3;
constexpr int kBox = kKeys * 128;                // one 64-column box of 128 rows (bytes)
// full[kSlots], empty[kSlots], s_done[2], p_ready[2], o_done[2], q_ready, drain
constexpr int NBAR = 2 * kSlots + 2 + 2 + 2 + 2;
constexpr int kThreads = 320;                    // an MMA warp, a producer warp, 8 softmax warps
constexpr int kMmaWarp = 0, kProducerWarp = 1, kFirstSoftmaxWarp = 2;
constexpr uint32_t kTmemCols = 512;              // S_A, S_B (128 columns each), O_A, O_B (D each)
constexpr float kLazyMax = 8.f;                  // log2 of the largest p before the max moves
// Shared-memory layout for head dim D (64 or 128): rows of Q, K and V are
// D / 64 boxes of 64 columns.
template <int D>
struct Cfg3 {
    static constexpr int kBoxes = D / 64;
    static constexpr int kTileQ = kBoxes * kBox;     // one 128-row query tile
    static constexpr int kSlotBytes = kBoxes * kBox; // a K or V tile: 128 keys x D
    static constexpr int OFF_Q = 0;                  // Q_A, Q_B
    static constexpr int OFF_KV = OFF_Q + 2 * kTileQ;
    static constexpr int OFF_BAR = OFF_KV + kSlots * kSlotBytes;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort flag, 8 warp maxima
    static constexpr int SMEM = OFF_MISC + 64 + 1024;    // + alignment slack
    static_assert(D == 64 || D == 128, "head dims 64 and 128");
    static_assert(SMEM <= 232448, "fits the per-CTA shared memory");
    static_assert(2 * kKeys + 2 * D <= (int)kTmemCols, "S_A, S_B, O_A, O_B fit TMEM");
};
}  // namespace pf3

// TILES: query tiles per CTA (2; or 1 when two-tile CTAs would leave SMs idle);
// D: head dim (64 or 128, Dqk = Dv).
template <typename T, int TILES, int D>
__global__ void __launch_bounds__(pf3::kThreads, 1)
    prefill3_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const Params p) {
    using namespace pf;
    using namespace pf3;
    using L = Cfg3<D>;
    constexpr int kCtaRows = TILES * kRows;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // row blocks in reverse order: under a causal mask the late rows see the
    // most keys, so the longest CTAs start first
    const int rb = gridDim.x - 1 - blockIdx.x, hkv = blockIdx.y, b = blockIdx.z;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::OFF_BAR);
    auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
    auto empty_bar = [&](int s) { return smem_u32(&bars[kSlots + s]); };
    auto s_bar = [&](int g) { return smem_u32(&bars[2 * kSlots + g]); };
    auto p_bar = [&](int g) { return smem_u32(&bars[2 * kSlots + 2 + g]); };
    auto o_bar = [&](int g) { return smem_u32(&bars[2 * kSlots + 4 + g]); };
    const uint32_t q_bar = smem_u32(&bars[2 * kSlots + 6]);
    const uint32_t drain_bar = smem_u32(&bars[2 * kSlots + 7]);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::OFF_MISC + 4);
    int *warp_keys = reinterpret_cast<int *>(smem + L::OFF_MISC + 16);

    // ---- softmax threads: group, row, head, query position, last visible key
    const bool softmax = warp >= kFirstSoftmaxWarp;
    const int grp = ((warp - kFirstSoftmaxWarp) >> 2) & 1, quarter = warp & 3;  // TMEM lanes 32 (warp % 4) ..
    const int trow = quarter * 32 + lane;  // row within the group's tile = TMEM lane
    const int r = rb * kCtaRows + grp * kRows + trow;
    const bool row_live = softmax && grp < TILES && r < p.R;
    const int hq = row_live ? hkv * p.g + r / p.Lq : 0;
    const int qi = row_live ? r % p.Lq : 0;
    const int n = p.Lk;
    int lim = -1;
    if (row_live) {
        lim = n - 1;
        if (p.causal) {
            const int c = qi + n - p.Lq;
            lim = c < lim ? c : lim;
        }
    }
    if (tid == 0) {
        for (int s = 0; s < kSlots; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int g = 0; g < 2; ++g) {
            mbar_init(s_bar(g), 1);
            mbar_init(p_bar(g), 4);  // one arrival per softmax warp of the group
            mbar_init(o_bar(g), 1);
        }
        mbar_init(q_bar, 8);  // one arrival per softmax warp
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    {
        int kv = lim + 1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kv = max(kv, __shfl_xor_sync(0xffffffffu, kv, off));
        if (lane == 0 && softmax) warp_keys[warp - kFirstSoftmaxWarp] = kv;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int kmax = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) kmax = max(kmax, warp_keys[w]);
    const int ntiles = (kmax + kKeys - 1) / kKeys;
    // a last row block of at most 128 rows leaves group B without rows: its
    // products and softmax are skipped
    const int ngroups = TILES == 2 && rb * kCtaRows + kRows < p.R ? 2 : 1;
    constexpr bool bf16 = std::is_same<T, __nv_bfloat16>::value;

    pdl_wait_primary();

    if (warp == kProducerWarp) {
        // ================================================= producer: K(0), V(0), K(1), ... by TMA
        if (lane == 0) {
            int issued = 0;
            for (int q = 0; q < 2 * ntiles; ++q) {
                const int s = q % kSlots, use = q / kSlots;
                if (use > 0 && !mbar_wait(empty_bar(s), (use - 1) & 1, abort_flag, p.status, kWaitLimitNs)) break;
                const uint32_t dst = sb + L::OFF_KV + s * L::kSlotBytes;
                const CUtensorMap *map = (q & 1) ? &tmV : &tmK;
                mbar_expect_tx(full_bar(s), L::kSlotBytes);
                for (int c = 0; c < L::kBoxes; ++c)
                    tma_load_4d_plain(dst + c * kBox, map, full_bar(s), c * 64, (q >> 1) * kKeys, hkv, b);
                mbar_arrive(full_bar(s));
                issued = q + 1;
            }
            if (*abort_flag) {
                // let the copies still in flight land before the CTA's shared memory is released
                volatile int no_abort = 0;
                for (int q = issued - kSlots < 0 ? 0 : issued - kSlots; q < issued; ++q)
                    mbar_wait(full_bar(q % kSlots), (q / kSlots) & 1, &no_abort, nullptr, kWaitLimitNs / 16);
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ================================================= MMA issue (one thread)
        if (lane == 0) {
            const uint32_t idesc = instr_desc(bf16, kRows, kKeys, false);   // S: N = 128 keys, K-major K
            const uint32_t idesc_o = instr_desc(bf16, kRows, D, true);     // PV: N = 128 dims, MN-major V
            // Operand descriptors: a base descriptor plus a constant offset in
            // 16-byte units (every shared address stays below 256 KB, so the sum
            // never carries out of the address field).
            const uint64_t dq0 = smem_desc(sb + L::OFF_Q, 16, 1024);
            const uint64_t dk0 = smem_desc(sb + L::OFF_KV, 16, 1024);        // a slot holding K
            const uint64_t dv0 = smem_desc(sb + L::OFF_KV, kBox, 1024);      // a slot holding V
            auto wait = [&](uint32_t bar, uint32_t parity) {
                return mbar_wait(bar, parity, abort_flag, p.status, kWaitLimitNs);
            };
            // S_g(j) = Q_g K(j)^T; K(j) is ring entry 2j
            auto issue_s = [&](int g, int j) {
                const uint64_t dk = dk0 + (uint64_t)((((2 * j) % kSlots) * L::kSlotBytes) >> 4);
                const uint64_t dq = dq0 + (uint64_t)((g * L::kTileQ) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (uint32_t)(((kk >> 2) * kBox + (kk & 3) * 32) >> 4);
                    umma(tmem + g * kKeys, dq + off, dk + off, idesc, kk > 0);
                }
                umma_commit(s_bar(g));
            };
            bool ok = ntiles > 0 && wait(q_bar, 0) && wait(full_bar(0), 0);
            if constexpr (TILES == 1) {
                // One tile: S double-buffered in TMEM columns [0, 128) and
                // [128, 256) (the second tile's, unused), so S(j + 1) is issued as
                // soon as K(j + 1) has landed and its softmax can start while PV(j)
                // runs.  S(j + 1)'s buffer last held P(j - 1), read by PV(j - 1),
                // which was issued before it.
                auto issue_s1 = [&](int j) {
                    const uint64_t dk = dk0 + (uint64_t)((((2 * j) % kSlots) * L::kSlotBytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (uint32_t)(((kk >> 2) * kBox + (kk & 3) * 32) >> 4);
                        umma(tmem + (j & 1) * kKeys, dq0 + off, dk + off, idesc, kk > 0);
                    }
                    umma_commit(s_bar(j & 1));
                };
                if (ok) {
                    tc_fence_after();
                    issue_s1(0);
                    umma_commit(empty_bar(0));
                }
                for (int j = 0; j < ntiles && ok; ++j) {
                    const int qv = 2 * j + 1, qk = 2 * j + 2;  // ring entries of V(j), K(j + 1)
                    bool next = j + 1 >= ntiles;
                    if (!next && mbar_try_wait(full_bar(qk % kSlots), (qk / kSlots) & 1)) {
                        tc_fence_after();
                        issue_s1(j + 1);
                        umma_commit(empty_bar(qk % kSlots));
                        next = true;
                    }
                    ok = wait(p_bar(0), j & 1) && wait(full_bar(qv % kSlots), (qv / kSlots) & 1);
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t dv = dv0 + (uint64_t)(((qv % kSlots) * L::kSlotBytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < kKeys / 16; ++kk)
                        umma_ts(tmem + 2 * kKeys, tmem + (j & 1) * kKeys + kk * 8, dv + (uint64_t)((kk * 2048) >> 4),
                                idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(o_bar(0));  // every tile: the softmax's rescale and the epilogue wait on it
                    umma_commit(empty_bar(qv % kSlots));
                    if (!next) {
                        ok = wait(full_bar(qk % kSlots), (qk / kSlots) & 1);
                        if (!ok) break;
                        tc_fence_after();
                        issue_s1(j + 1);
                        umma_commit(empty_bar(qk % kSlots));
                    }
                }
            } else {
            if (ok) {
                tc_fence_after();
                for (int g = 0; g < ngroups; ++g) issue_s(g, 0);
                umma_commit(empty_bar(0));  // K(0) read once its products are done
            }
            for (int j = 0; j < ntiles && ok; ++j) {
                const int qv = 2 * j + 1, qk = 2 * j + 2;  // ring entries of V(j), K(j + 1)
                const bool more = j + 1 < ntiles;
                const uint64_t dv = dv0 + (uint64_t)(((qv % kSlots) * L::kSlotBytes) >> 4);
                for (int g = 0; g < ngroups && ok; ++g) {
                    // P_g(j) written (S_g(j) read, O_g rescaled); V(j) landed
                    ok = wait(p_bar(g), j & 1) && (g > 0 || wait(full_bar(qv % kSlots), (qv / kSlots) & 1));
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kKeys / 16; ++kk)  // P_g(j): 16 keys = 8 TMEM columns per step
                        umma_ts(tmem + 2 * kKeys + g * D, tmem + g * kKeys + kk * 8,
                                dv + (uint64_t)((kk * 2048) >> 4), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
                    // O_g is final after the last tile's PV; before that, the commit
                    // of S_g(j + 1) (issued after PV_g(j), and a commit covers all of
                    // this thread's earlier products) tells the softmax PV_g(j) is done
                    if (j + 1 == ntiles) umma_commit(o_bar(g));
                    if (g == ngroups - 1) umma_commit(empty_bar(qv % kSlots));  // V(j) read by its products
                    if (more) {
                        if (g == 0) {
                            ok = wait(full_bar(qk % kSlots), (qk / kSlots) & 1);
                            if (!ok) break;
                            tc_fence_after();
                        }
                        issue_s(g, j + 1);
                        if (g == ngroups - 1) umma_commit(empty_bar(qk % kSlots));  // K(j + 1) read by its products
                    }
                }
            }
            }
            // every product this thread issued is done before TMEM can be freed
            umma_commit(drain_bar);
            volatile int no_abort = 0;
            mbar_wait(drain_bar, 0, &no_abort, p.status, kWaitLimitNs);
        }
        __syncwarp();
    } else {
        // ================================================= softmax group grp: one row per thread
        {
            const T *qg = reinterpret_cast<const T *>(p.q);
            const T *src = qg + b * p.q_sb + (long long)qi * p.q_sl + (long long)hq * p.q_sh;
            for (int c = 0; c < D / 8; ++c) {
                const uint32_t dst =
                    sb + L::OFF_Q + grp * L::kTileQ + (c >> 3) * kBoxQ + trow * 128 + ((((c & 7) ^ (trow & 7))) << 4);
                cp_async_16(dst, src + c * 8, row_live ? 16u : 0u);
            }
            asm volatile("cp.async.wait_all;" ::: "memory");
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(q_bar);
        }
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t t_o = tmem + 2 * kKeys + grp * D + lane_off;
        float m = -INFINITY, l = 0.f;  // m in base-2 units of the scaled scores
        bool ok = grp < ngroups;  // a group without rows has nothing to do
        for (int j = 0; j < ntiles && ok; ++j) {
            // this tile's S: the group's buffer (two tiles), or buffer j % 2 (one tile)
            const uint32_t t_s = tmem + (TILES == 2 ? grp : (j & 1)) * kKeys + lane_off;
            ok = TILES == 2 ? mbar_wait(s_bar(grp), j & 1, abort_flag, p.status, kWaitLimitNs)
                            : mbar_wait(s_bar(j & 1), (j >> 1) & 1, abort_flag, p.status, kWaitLimitNs);
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float x[kKeys];
            {
                uint32_t v[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(t_s + c * 32, v[c]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[c * 32 + e] = __uint_as_float(v[c][e]);
            }
            const int key0 = j * kKeys;
            if (!__all_sync(0xffffffffu, key0 + kKeys - 1 <= lim)) {
#pragma unroll
                for (int e = 0; e < kKeys; ++e) x[e] = key0 + e <= lim ? x[e] : -INFINITY;
            }
            // row max: eight independent chains of three-input max
            float mxa[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) mxa[e] = fmaxf(x[2 * e], x[2 * e + 1]);
#pragma unroll
            for (int e = 16; e < kKeys; e += 16)
#pragma unroll
                for (int c = 0; c < 8; ++c) mxa[c] = max3f(mxa[c], x[e + 2 * c], x[e + 2 * c + 1]);
            const float mx = max3f(max3f(mxa[0], mxa[1], mxa[2]), max3f(mxa[3], mxa[4], mxa[5]),
                                   fmaxf(mxa[6], mxa[7])) *
                             p.scale_log2;
            // the running max moves only when this tile's max is more than 2^8 above it
            const float mn = mx > m + kLazyMax ? mx : m;
            const float base = mn == -INFINITY ? 0.f : mn;
            const float alpha = fast_exp2(m - base);  // 1 when m stays, 0 while nothing was seen
            m = mn;
            // p = 2^(x * scale_log2 - m), packed two keys per 32-bit column and
            // written over this row's S columns [0, 64) in TMEM: the A operand of
            // PV_g(j).  (The scores are all in registers by now; PV_g(j - 1),
            // which read the previous P there, finished before S_g(j) did.)
            // y = x * scale_log2 - base on key pairs (one packed FMA), p = 2^y,
            // sums in two packed accumulators
            const uint64_t sc2 = pack2f(p.scale_log2, p.scale_log2), nb2 = pack2f(-base, -base);
            uint64_t sum2[2] = {pack2f(0.f, 0.f), pack2f(0.f, 0.f)};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t pk[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    float y0, y1;
                    unpack2f(ffma2(pack2f(x[h * 64 + 2 * c], x[h * 64 + 2 * c + 1]), sc2, nb2), y0, y1);
                    const float p0 = fast_exp2(y0), p1 = fast_exp2(y1);
                    sum2[c & 1] = fadd2(sum2[c & 1], pack2f(p0, p1));
                    pk[c] = Mma<T>::pack(p0, p1);
                }
                tmem_st32(t_s + h * 32, pk);
            }
            float suma[4];
            unpack2f(sum2[0], suma[0], suma[1]);
            unpack2f(sum2[1], suma[2], suma[3]);
            // O_g *= alpha where the max moved.  With two tiles PV_g(j - 1) is
            // complete: S_g(j), whose barrier this warp waited on, was committed
            // after it; with one tile S(j) may have gone first, so wait for it.
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                if constexpr (TILES == 1) {
                    ok = mbar_wait(o_bar(0), (j - 1) & 1, abort_flag, p.status, kWaitLimitNs);
                    if (!__all_sync(0xffffffffu, ok)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
#pragma unroll
                for (int h = 0; h < D / 64; ++h) {
                    uint32_t v0[32], v1[32];
                    tmem_ld32(t_o + h * 64, v0);
                    tmem_ld32(t_o + h * 64 + 32, v1);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        v0[e] = __float_as_uint(__uint_as_float(v0[e]) * alpha);
                        v1[e] = __float_as_uint(__uint_as_float(v1[e]) * alpha);
                    }
                    tmem_st32(t_o + h * 64, v0);
                    tmem_st32(t_o + h * 64 + 32, v1);
                }
            }
            tmem_wait_st();
            l = l * alpha + ((suma[0] + suma[1]) + (suma[2] + suma[3]));
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_bar(grp));  // this warp's rows of P(j) are written
        }
        if (ok && ntiles > 0) {
            // the last PV: with two tiles o_bar's one commit; with one tile the
            // MMA thread's final (drain) commit -- up to two of o_bar's per-tile
            // phases can still be open here, which a parity wait cannot tell apart
            ok = TILES == 2 ? mbar_wait(o_bar(grp), 0, abort_flag, p.status, kWaitLimitNs)
                            : mbar_wait(drain_bar, 0, abort_flag, p.status, kWaitLimitNs);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
        }
        if (ok) {
            const float inv = l > 0.f ? 1.f / l : 0.f;
            T *og = reinterpret_cast<T *>(p.o) + b * p.o_sb + (long long)qi * p.o_sl + (long long)hq * p.o_sh;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                if (ntiles > 0) {
                    tmem_ld32(t_o + c * 32, v);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = 0u;
                }
                if (row_live) {
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        float f[8];
#pragma unroll
                        for (int z = 0; z < 8; ++z) f[z] = __uint_as_float(v[e + z]) * inv;
                        store_row8<T>(og + c * 32 + e, f);
                    }
                }
            }
            if (row_live && p.lse)
                p.lse[b * p.lse_sb + hq * p.lse_sh + qi] = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

template <typename T, int KEYS>
static void fill(KernelInfo *out) {
    out->fn = reinterpret_cast<const void *>(&prefill_kernel<T, KEYS>);
    out->threads = pf::kThreads;
    out->smem = pf::Cfg<KEYS>::SMEM;
    out->tile_keys = KEYS;
    out->stages = pf::kStages;
    out->variant = 3;  // FA_VARIANT_TCGEN05
    out->rows = pf::kRows;
    out->form = FA_TCGEN05_ONE_TILE;
}

// 128-key tiles, one CTA per SM.  (64-key tiles with two CTAs per SM measured
// the same on a 4K causal prefill -- 332 vs 334 us -- the doubled per-tile
// overhead cancelling the second CTA's interleaving.)
constexpr int kPrefillKeys = 128;

template <typename T, int TILES, int D>
static void fill3(KernelInfo *out) {
    out->fn = reinterpret_cast<const void *>(&prefill3_kernel<T, TILES, D>);
    out->threads = pf3::kThreads;
    out->smem = pf3::Cfg3<D>::SMEM;
    out->tile_keys = pf3::kKeys;
    out->stages = pf3::kSlots;
    out->variant = 3;  // FA_VARIANT_TCGEN05
    out->rows = TILES * pf::kRows;
    out->form = TILES == 2 ? FA_TCGEN05_TWO_TILES : FA_TCGEN05_ONE_TILE_MMA;
}

bool get_prefill_kernel(int dtype, int dqk, int dv, int form, KernelInfo *out) {
    if (dtype < 0 || dtype > 1 || dqk != dv || (dqk != 64 && dqk != 128)) return false;
    const bool h = dtype == 0;
    switch (form) {
    case FA_TCGEN05_ONE_TILE:  // head dim 128 only
        if (dqk != 128) return false;
        if (h) fill<__half, kPrefillKeys>(out);
        else fill<__nv_bfloat16, kPrefillKeys>(out);
        return true;
    case FA_TCGEN05_TWO_TILES:
        if (dqk == 64) {
            if (h) fill3<__half, 2, 64>(out);
            else fill3<__nv_bfloat16, 2, 64>(out);
        } else {
            if (h) fill3<__half, 2, 128>(out);
            else fill3<__nv_bfloat16, 2, 128>(out);
        }
        return true;
    case FA_TCGEN05_ONE_TILE_MMA:
        if (dqk == 64) {
            if (h) fill3<__half, 1, 64>(out);
            else fill3<__nv_bfloat16, 1, 64>(out);
        } else {
            if (h) fill3<__half, 1, 128>(out);
            else fill3<__nv_bfloat16, 1, 128>(out);
        }
        return true;
    default:
        return false;
    }
}

}  // namespace fa
