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
// tcgen05.commit releases a slot once its products are done.  The kernel,
// prefill3_kernel, takes one or two query tiles per CTA with a dedicated MMA
// warp and a TMA warp; with two tiles one tile's products run during the
// other's softmax, with one tile S is double-buffered; P stays in TMEM.
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
constexpr int kRows = 128;           // packed query rows per query tile (MMA M)
constexpr int kBoxQ = kRows * 128;   // one 64-column box of 128 rows (bytes)
}  // namespace pf

// ---------------------------------------------------------------------------
// Two query tiles per CTA with 128-key K / V tiles (the kernel also runs
// with one tile): every QK^T product is M 128 x N 128 x K 16, every PV product
// M 128 x N Dv x K 16, and per 128 keys the MMA warp issues 32 products (16
// for head dim 64, 40 for 192/128) with four commits and two waits.  K and V
// tiles stream separately through a ring of three slots (two for Dqk = 192;
// K(j), V(j), K(j + 1), ...; 128 keys each).  S is single-buffered per group; per tile j the MMA warp
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
constexpr int kBox = kKeys * 128;                // one 64-column box of 128 rows (bytes)
constexpr int kThreads = 320;                    // an MMA warp, a producer warp, 8 softmax warps
constexpr int kMmaWarp = 0, kProducerWarp = 1, kFirstSoftmaxWarp = 2;
constexpr uint32_t kTmemCols = 512;              // S_A, S_B (128 columns each), O_A, O_B (Dv each)
constexpr float kLazyMax = 8.f;                  // log2 of the largest p before the max moves
// Shared-memory layout for head dims (DQK, DV) = (64, 64), (128, 128) or
// (192, 128): rows of Q and K are DQK / 64 boxes of 64 columns, rows of V
// DV / 64.  K and V tiles take turns in a ring of equal slots (K(0), V(0),
// K(1), ...): three, or two for DQK = 192, whose two 48 KB query tiles leave
// room for two 48 KB slots only.
template <int DQK, int DV>
struct Cfg3 {
    static constexpr int kBoxesQK = DQK / 64, kBoxesV = DV / 64;
    static constexpr int kTileQ = kBoxesQK * kBox;   // one 128-row query tile
    static constexpr int kKBytes = kBoxesQK * kBox;  // a K tile: 128 keys x DQK
    static constexpr int kVBytes = kBoxesV * kBox;   // a V tile: 128 keys x DV
    static constexpr int kSlotBytes = kKBytes > kVBytes ? kKBytes : kVBytes;
    static constexpr int kSlots = DQK > 128 ? 2 : 3;
    // full[kSlots], empty[kSlots], s_done[2], p_ready[2], o_done[2], q_ready, drain
    static constexpr int NBAR = 2 * kSlots + 2 + 2 + 2 + 2;
    static constexpr int OFF_Q = 0;                  // Q_A, Q_B
    static constexpr int OFF_KV = OFF_Q + 2 * kTileQ;
    static constexpr int OFF_BAR = OFF_KV + kSlots * kSlotBytes;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort flag, 8 warp maxima
    static constexpr int SMEM = OFF_MISC + 64 + 1024;    // + alignment slack
    static_assert((DQK == 64 && DV == 64) || (DQK == 128 && DV == 128) || (DQK == 192 && DV == 128),
                  "head dims 64/64, 128/128 and 192/128");
    static_assert(SMEM <= 232448, "fits the per-CTA shared memory");
    static_assert(2 * kKeys + 2 * DV <= (int)kTmemCols, "S_A, S_B, O_A, O_B fit TMEM");
};
}  // namespace pf3

// TILES: query tiles per CTA (2; or 1 when two-tile CTAs would leave SMs idle);
// DQK, DV: head dims (64/64, 128/128 or 192/128).
template <typename T, int TILES, int DQK, int DV>
__global__ void __launch_bounds__(pf3::kThreads, 1)
    prefill3_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const Params p) {
    using namespace pf;
    using namespace pf3;
    using L = Cfg3<DQK, DV>;
    constexpr int kSlots = L::kSlots;
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
            // test hook: the first CTA leaves K(0)'s slot empty (no copy, no
            // arrival), so the MMA thread's wait on it runs out
            const int q_first = p.stall && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 ? 1 : 0;
            int issued = 0;
            for (int q = q_first; q < 2 * ntiles; ++q) {
                const int s = q % kSlots, use = q / kSlots;
                if (use > 0 && !mbar_wait(empty_bar(s), (use - 1) & 1, abort_flag, p.status, p.wait_limit_ns)) break;
                const uint32_t dst = sb + L::OFF_KV + s * L::kSlotBytes;
                const CUtensorMap *map = (q & 1) ? &tmV : &tmK;
                mbar_expect_tx(full_bar(s), (q & 1) ? L::kVBytes : L::kKBytes);
                for (int c = 0; c < ((q & 1) ? L::kBoxesV : L::kBoxesQK); ++c)
                    tma_load_4d_plain(dst + c * kBox, map, full_bar(s), c * 64, (q >> 1) * kKeys, hkv, b);
                mbar_arrive(full_bar(s));
                issued = q + 1;
            }
            if (*abort_flag) {
                // let the copies still in flight land before the CTA's shared memory is released
                volatile int no_abort = 0;
                for (int q = issued - kSlots < q_first ? q_first : issued - kSlots; q < issued; ++q)
                    mbar_wait(full_bar(q % kSlots), (q / kSlots) & 1, &no_abort, nullptr, p.wait_limit_ns / 16);
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ================================================= MMA issue (one thread)
        if (lane == 0) {
            const uint32_t idesc = instr_desc(bf16, kRows, kKeys, false);   // S: N = 128 keys, K-major K
            const uint32_t idesc_o = instr_desc(bf16, kRows, DV, true);    // PV: N = DV dims, MN-major V
            // Operand descriptors: a base descriptor plus a constant offset in
            // 16-byte units (every shared address stays below 256 KB, so the sum
            // never carries out of the address field).
            const uint64_t dq0 = smem_desc(sb + L::OFF_Q, 16, 1024);
            const uint64_t dk0 = smem_desc(sb + L::OFF_KV, 16, 1024);        // a slot holding K
            const uint64_t dv0 = smem_desc(sb + L::OFF_KV, kBox, 1024);      // a slot holding V
            auto wait = [&](uint32_t bar, uint32_t parity) {
                return mbar_wait(bar, parity, abort_flag, p.status, p.wait_limit_ns);
            };
            // S_g(j) = Q_g K(j)^T; K(j) is ring entry 2j
            auto issue_s = [&](int g, int j) {
                const uint64_t dk = dk0 + (uint64_t)((((2 * j) % kSlots) * L::kSlotBytes) >> 4);
                const uint64_t dq = dq0 + (uint64_t)((g * L::kTileQ) >> 4);
#pragma unroll
                for (int kk = 0; kk < DQK / 16; ++kk) {
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
                    for (int kk = 0; kk < DQK / 16; ++kk) {
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
                        umma_ts(tmem + 2 * kKeys + g * DV, tmem + g * kKeys + kk * 8,
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
            mbar_wait(drain_bar, 0, &no_abort, p.status, p.wait_limit_ns);
        }
        __syncwarp();
    } else {
        // ================================================= softmax group grp: one row per thread
        {
            const T *qg = reinterpret_cast<const T *>(p.q);
            const T *src = qg + b * p.q_sb + (long long)qi * p.q_sl + (long long)hq * p.q_sh;
            for (int c = 0; c < DQK / 8; ++c) {
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
        const uint32_t t_o = tmem + 2 * kKeys + grp * DV + lane_off;
        float m = -INFINITY, l = 0.f;  // m in base-2 units of the scaled scores
        bool ok = grp < ngroups;  // a group without rows has nothing to do
        for (int j = 0; j < ntiles && ok; ++j) {
            // this tile's S: the group's buffer (two tiles), or buffer j % 2 (one tile)
            const uint32_t t_s = tmem + (TILES == 2 ? grp : (j & 1)) * kKeys + lane_off;
            ok = TILES == 2 ? mbar_wait(s_bar(grp), j & 1, abort_flag, p.status, p.wait_limit_ns)
                            : mbar_wait(s_bar(j & 1), (j >> 1) & 1, abort_flag, p.status, p.wait_limit_ns);
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
                    ok = mbar_wait(o_bar(0), (j - 1) & 1, abort_flag, p.status, p.wait_limit_ns);
                    if (!__all_sync(0xffffffffu, ok)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
#pragma unroll
                for (int h = 0; h < DV / 64; ++h) {
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
            ok = TILES == 2 ? mbar_wait(o_bar(grp), 0, abort_flag, p.status, p.wait_limit_ns)
                            : mbar_wait(drain_bar, 0, abort_flag, p.status, p.wait_limit_ns);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
        }
        if (ok) {
            const float inv = l > 0.f ? 1.f / l : 0.f;
            T *og = reinterpret_cast<T *>(p.o) + b * p.o_sb + (long long)qi * p.o_sl + (long long)hq * p.o_sh;
#pragma unroll
            for (int c = 0; c < DV / 32; ++c) {
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

template <typename T, int TILES, int DQK, int DV>
static void fill3(KernelInfo *out) {
    out->fn = reinterpret_cast<const void *>(&prefill3_kernel<T, TILES, DQK, DV>);
    out->threads = pf3::kThreads;
    out->smem = pf3::Cfg3<DQK, DV>::SMEM;
    out->tile_keys = pf3::kKeys;
    out->stages = pf3::Cfg3<DQK, DV>::kSlots;
    out->variant = 3;  // FA_VARIANT_TCGEN05
    out->rows = TILES * pf::kRows;
    out->form = TILES == 2 ? FA_TCGEN05_TWO_TILES : FA_TCGEN05_ONE_TILE_MMA;
}

template <typename T, int TILES>
static bool fill3_dims(int dqk, int dv, KernelInfo *out) {
    if (dqk == 64 && dv == 64) { fill3<T, TILES, 64, 64>(out); return true; }
    if (dqk == 128 && dv == 128) { fill3<T, TILES, 128, 128>(out); return true; }
    if (dqk == 192 && dv == 128) { fill3<T, TILES, 192, 128>(out); return true; }
    return false;
}

bool get_prefill_kernel(int dtype, int dqk, int dv, int form, KernelInfo *out) {
    const bool h = dtype == 0;
    if (dtype < 0 || dtype > 1) return false;
    switch (form) {
    case FA_TCGEN05_TWO_TILES:
        return h ? fill3_dims<__half, 2>(dqk, dv, out) : fill3_dims<__nv_bfloat16, 2>(dqk, dv, out);
    case FA_TCGEN05_ONE_TILE_MMA:
        return h ? fill3_dims<__half, 1>(dqk, dv, out) : fill3_dims<__nv_bfloat16, 1>(dqk, dv, out);
    default:
        return false;
    }
}

}  // namespace fa
