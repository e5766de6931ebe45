// fa_api.cu -- host side of libfa_b200.so: the C ABI declared in include/fa.h.
//
// Each compute call validates its arguments on the host (nothing is launched
// for a bad call), plans the launch (variant, CTA count, work partition,
// workspace), encodes the K/V TMA tensor maps, then enqueues the split-KV
// kernel and, when some unit is shared between CTAs or has no visible key,
// the LSE combine kernel with programmatic dependent launch.  The caller
// owns every buffer; the library allocates no device memory and never
// synchronises a stream in the compute calls (the aclnn-style two-phase
// call of "SmallQ FlashAttention for Ascend 910B", section "aclnn API 调用":
// ask for the workspace size, let the caller allocate it, run on a stream).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "fa.h"
#include "fa_common.cuh"
#include "fa_internal.h"

// Device status word: bit 0 set when a kernel gave up waiting on its pipeline.
__device__ unsigned int g_fa_status = 0;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kDefaultMinShare = 2;
// Least tiles per CTA for the unit-aligned partition of uniform dense calls
// (make_plan).  Measured on one B200, µs per call, balanced over all SMs /
// aligned on 128 CTAs: GQA-4 decode at head dim 256 (32 units of 128 64-key
// tiles: 32 per CTA) 45.3 / 43.1; speculative decode, 64 heads x 4 queries
// over 3,000 keys (12 per CTA) 18.83 / 18.41; single-query decode, 32 heads
// over 4,096 keys (8 per CTA) 14.66 / 14.73.
constexpr int kAlignedMinTiles = 12;
// K / V bytes of re-reads (mma.sync kernel, blocks of 8 rows) the tcgen05
// split-KV kernel must save before the library chooses it.
constexpr int64_t kTcSplitMinSavedBytes = int64_t(128) << 20;
// Extra partition positions (in tiles) per unit for the tcgen05 split-KV
// kernel: its segment epilogue and the next segment's first tile take about
// this many tiles' worth of streaming time.
#ifndef FA_TC_SEG_COST
#define FA_TC_SEG_COST 4
#endif
constexpr int kTcSegCost = FA_TC_SEG_COST;
// The same for the mma.sync kernel: its epilogue at a unit boundary inside a
// piece (the merge of the four warps' partials and the partial's write) costs
// about one tile.  Measured on one B200 (µs per call, seg cost 0 / 1 / 2):
// single-row decode 14.83 / 14.70 / 14.72, speculative decode 19.18 / 18.80 /
// 18.99, batched kvcache 307.9 / 307.3 / 309.8.
#ifndef FA_MMA_SEG_COST
#define FA_MMA_SEG_COST 1
#endif
constexpr int kMmaSegCost = FA_MMA_SEG_COST;

thread_local std::string t_err;
thread_local fa_dispatch_info t_disp = {};
std::atomic<int64_t> g_launches{0};
std::atomic<int> g_force_variant{FA_VARIANT_AUTO};
std::atomic<int> g_force_tc_form{FA_TCGEN05_AUTO};
// Test hook (fa_test_stall_next_call): the next call's wait bound, 0 = none pending.
std::atomic<unsigned long long> g_stall_next{0};
constexpr unsigned long long kWaitLimitNs = 4000000000ull;  // 4 s

fa_status fail(fa_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    t_err = buf;
    return s;
}

fa_status cuda_fail(cudaError_t e, const char *what) {
    return fail(FA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ------------------------------------------------------------ per-device state
struct DeviceState {
    bool ready = false;
    int sms = 0;
    unsigned *status = nullptr;
};
std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

struct FnState {
    const void *fn;
    int device;
    int smem;
    int occupancy;
};
std::vector<FnState> g_fns;

fa_status device_state(DeviceState **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(FA_ERR_UNSUPPORTED, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState &d = g_dev[dev];
    if (!d.ready) {
        int major = 0, minor = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute");
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (major != 10 || minor != 0)
            return fail(FA_ERR_UNSUPPORTED, "compiled for sm_100a only; device %d is sm_%d%d", dev, major, minor);
        if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute(sm count)");
        void *ptr = nullptr;
        if ((e = cudaGetSymbolAddress(&ptr, g_fa_status)) != cudaSuccess)
            return cuda_fail(e, "cudaGetSymbolAddress(status)");
        d.status = static_cast<unsigned *>(ptr);
        d.ready = true;
    }
    *out = &d;
    return FA_OK;
}

// Sets the kernel's shared-memory limit once per device and returns its
// resident CTAs per SM.
fa_status prepare_fn(const void *fn, int threads, int smem, int *occupancy) {
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(g_mu);
    for (const FnState &f : g_fns)
        if (f.fn == fn && f.device == dev && f.smem >= smem) {
            *occupancy = f.occupancy;
            return FA_OK;
        }
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(max dynamic smem)");
    // Every kernel of the library asks for the same (largest) shared-memory
    // carve-out: an SM changes its L1 / shared split only when it is idle, so
    // kernels with different carve-outs could not share an SM, which is what
    // lets the combine kernel and the next call's split-KV kernel start while
    // the kernel before them is still finishing.
    e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(shared memory carve-out)");
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, threads, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    if (occ < 1) return fail(FA_ERR_UNSUPPORTED, "kernel does not fit on an SM (%d B shared memory)", smem);
    g_fns.push_back({fn, dev, smem, occ});
    *occupancy = occ;
    return FA_OK;
}

// ------------------------------------------------------------ validation
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fa_status check_tensor(const fa_tensor *t, const char *name) {
    if (!t) return fail(FA_ERR_INVALID_ARG, "%s: null descriptor", name);
    if (t->dtype != FA_F16 && t->dtype != FA_BF16)
        return fail(FA_ERR_UNSUPPORTED, "%s: element type %d is not fp16/bf16", name, t->dtype);
    int64_t numel = 1;
    for (int i = 0; i < 4; ++i) {
        if (t->shape[i] < 0 || t->shape[i] > INT32_MAX)
            return fail(FA_ERR_INVALID_ARG, "%s: shape[%d] = %lld out of range", name, i, (long long)t->shape[i]);
        numel *= t->shape[i];
    }
    if (t->stride[3] != 1) return fail(FA_ERR_UNSUPPORTED, "%s: last dimension must be contiguous", name);
    for (int i = 0; i < 3; ++i) {
        if (t->stride[i] < 0 || (t->stride[i] % 8) != 0 || t->stride[i] >= (int64_t(1) << 38))
            return fail(FA_ERR_UNSUPPORTED, "%s: stride[%d] = %lld must be a non-negative multiple of 8 elements",
                        name, i, (long long)t->stride[i]);
    }
    if (numel > 0) {
        if (!t->data) return fail(FA_ERR_INVALID_ARG, "%s: null data pointer", name);
        if (!aligned16(t->data)) return fail(FA_ERR_UNSUPPORTED, "%s: data must be 16-byte aligned", name);
    }
    return FA_OK;
}

struct Shapes {
    int dtype;
    int B, Lq, Hq, Lk, Hkv, Dqk, Dv, g, R, RB, BR;
    int rpc;        // packed rows per row block: RB = ceil(R / rpc) row blocks per (batch, kv head)
    int KDqk, KDv;  // head dims of the kernel instance that runs the call (>= Dqk, Dv)
    int page = 0;   // paged cache: keys per block (0: dense)
};

// Head dims: any multiple of 8 from 8 to 256 (a TMA row stride must be a
// multiple of 16 bytes).  A call runs on the compiled instance that covers
// both dims -- (192, 128) for MLA-shaped dims, else the square instance 64,
// 128 or 256 -- the dims past the call's read as zeros (TMA fills the columns
// past a row's end, the query rows are zero-filled) and are never written.
fa_status kernel_dims(Shapes *s) {
    auto ok_dim = [](int d) { return d >= 8 && d <= 256 && d % 8 == 0; };
    if (!ok_dim(s->Dqk) || !ok_dim(s->Dv))
        return fail(FA_ERR_UNSUPPORTED, "head dims (Dqk %d, Dv %d): each must be a multiple of 8 from 8 to 256",
                    s->Dqk, s->Dv);
    auto pad = [](int d) { return d <= 64 ? 64 : (d <= 128 ? 128 : 256); };
    if (s->Dqk > 128 && s->Dqk <= 192 && s->Dv <= 128) {
        s->KDqk = 192;
        s->KDv = 128;
    } else {
        s->KDqk = s->KDv = std::max(pad(s->Dqk), pad(s->Dv));
    }
    return FA_OK;
}

// Row blocks of rpc packed rows: RB per (batch, kv head), BR = B * RB entries.
fa_status set_row_blocks(Shapes *s, int rpc) {
    s->rpc = rpc;
    s->RB = (s->R + rpc - 1) / rpc;
    const int64_t BR = (int64_t)s->B * s->RB;
    if (BR > fa::kMaxPrefixEntries)
        return fail(FA_ERR_UNSUPPORTED, "B * ceil(g * Lq / %d) = %lld exceeds %d", rpc, (long long)BR,
                    fa::kMaxPrefixEntries);
    s->BR = (int)BR;
    return FA_OK;
}

// Paged K/V: K and V are [num_blocks, page, Hkv, D]; batch b's key j is row
// j % page of block block_table[b * bt_stride + j / page].
// Packed variable-length inputs: q / o [1, total_q, H, D], k / v
// [1, total_k, Hkv, D]; sequence b owns query tokens [cu_q[b], cu_q[b + 1])
// and key tokens [cu_k[b], cu_k[b + 1]).
struct Varlen {
    const int32_t *cu_q, *cu_k;
    int total_q;
};

struct Paging {
    const int32_t *block_table;
    int64_t bt_stride;
    int max_pages;
    int page;
    int num_blocks;
};

fa_status check_shapes(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v, const fa_tensor *o,
                       Shapes *s, const Paging *pg = nullptr) {
    fa_status st;
    if ((st = check_tensor(q, "q")) || (st = check_tensor(k, "k")) || (st = check_tensor(v, "v")))
        return st;
    if (o && (st = check_tensor(o, "o"))) return st;
    if (k->dtype != q->dtype || v->dtype != q->dtype || (o && o->dtype != q->dtype))
        return fail(FA_ERR_INVALID_ARG, "q, k, v and o must share one element type");
    s->dtype = q->dtype;
    s->B = (int)q->shape[0];
    s->Lq = (int)q->shape[1];
    s->Hq = (int)q->shape[2];
    s->Dqk = (int)q->shape[3];
    s->Lk = (int)k->shape[1];
    s->Hkv = (int)k->shape[2];
    s->Dv = (int)v->shape[3];
    if (pg) {
        // k, v: [num_blocks, page, Hkv, D]; the key capacity of a batch is
        // max_pages * page
        if (v->shape[0] != k->shape[0])
            return fail(FA_ERR_INVALID_ARG, "k_pages and v_pages must have the same number of blocks");
        if (k->shape[0] < 1 || k->shape[0] > INT32_MAX - 1)
            return fail(FA_ERR_INVALID_ARG, "num_blocks must be in [1, 2^31 - 2]");
        const int64_t page = k->shape[1];
        if (page < 16 || page > (1 << 20) || (page & (page - 1)))
            return fail(FA_ERR_UNSUPPORTED, "page size %lld: a power of two from 16 to 2^20 is required",
                        (long long)page);
        if (pg->max_pages < 1) return fail(FA_ERR_INVALID_ARG, "max_blocks_per_seq must be positive");
        if (pg->bt_stride < pg->max_pages)
            return fail(FA_ERR_INVALID_ARG, "block_table_stride (%lld) < max_blocks_per_seq (%d)",
                        (long long)pg->bt_stride, pg->max_pages);
        if ((int64_t)pg->max_pages * page > INT32_MAX / 2)
            return fail(FA_ERR_UNSUPPORTED, "max_blocks_per_seq * page too large");
        s->Lk = (int)((int64_t)pg->max_pages * page);
        s->page = (int)page;
    } else if (k->shape[0] != s->B || v->shape[0] != s->B) {
        return fail(FA_ERR_INVALID_ARG, "batch mismatch: q %d, k %lld, v %lld", s->B, (long long)k->shape[0],
                    (long long)v->shape[0]);
    }
    if (k->shape[3] != s->Dqk) return fail(FA_ERR_INVALID_ARG, "k head dim %lld != q head dim %d", (long long)k->shape[3], s->Dqk);
    if (v->shape[1] != k->shape[1] || v->shape[2] != s->Hkv)
        return fail(FA_ERR_INVALID_ARG, "v must be [B, Lk, Hkv, Dv] matching k");
    if (o && (o->shape[0] != s->B || o->shape[1] != s->Lq || o->shape[2] != s->Hq || o->shape[3] != s->Dv))
        return fail(FA_ERR_INVALID_ARG, "o must be [B, Lq, Hq, Dv]");
    if (s->Hkv <= 0 || s->Hq <= 0) return fail(FA_ERR_INVALID_ARG, "head counts must be positive");
    if (s->Hq % s->Hkv) return fail(FA_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", s->Hq, s->Hkv);
    if ((st = kernel_dims(s))) return st;
    s->g = s->Hq / s->Hkv;
    int64_t R = (int64_t)s->g * s->Lq;
    if (R > INT32_MAX / 2) return fail(FA_ERR_UNSUPPORTED, "g * Lq too large");
    s->R = (int)R;
    return set_row_blocks(s, fa::kRowsPerCta);
}

// ------------------------------------------------------------ planning
struct Plan {
    fa::KernelInfo main, comb;
    int occupancy;
    int P;           // CTAs launched for the main kernel
    int P_param;     // CTA count the partition is computed from
    int min_share;
    int64_t W;       // host-known total tiles (-1 for kvcache)
    bool need_combine;
    bool need_workspace;
    size_t pieces;   // partial-result slots reserved (pieces of the partition)
    size_t ws_o_off, ws_lse_off;
    size_t ws_bytes;
    int comb_smem;
    int comb_grid;
    bool prefill = false;  // the tcgen05 kernel: one CTA per (block of 128 rows, kv head, batch), no combine
    int seg_cost = 0;      // partition positions per unit beyond its tiles
    int row_blocks = 0;
};

// The tensor-core variant puts the keys on the MMA's 16-row side, so even one
// packed query row fills its operand tiles with keys; measured on B200 it is
// faster than the fp32 FMA variant at every packed-row count, one row
// included (decode fp16, 4096 keys, 32 heads: 15.7 vs 16.6 us per call), so
// the FMA variant runs only when forced.
int choose_variant(const Shapes &) {
    int forced = g_force_variant.load();
    if (forced != FA_VARIANT_AUTO) return forced;
    return FA_VARIANT_MMA;
}

// Host copy of the device partition for dense inputs (every batch has Lk keys):
// returns W and the partition, and whether some unit is cut between pieces
// or has no tiles (then the combine kernel has work).
void host_schedule(const Shapes &s, int causal, int tile_shift, int seg_cost, int P, int min_share, int *W_out,
                   fa::Partition *pt_out, bool *need_combine) {
    std::vector<int> pre(s.BR + 1, 0);
    bool empty_unit = false;
    for (int x = 0; x < s.BR; ++x) {
        int t = fa::unit_tiles(s.Lk, x % s.RB, s.R, s.Lq, causal, tile_shift, s.rpc);
        if (t == 0) empty_unit = true;
        pre[x + 1] = pre[x] + s.Hkv * fa::unit_weight(t, seg_cost);
    }
    const int W = pre[s.BR];
    const fa::Partition pt = fa::make_partition(W, P, min_share);
    bool split = false;
    for (int c = 1; c < fa::num_pieces(pt) && !split && W > 0; ++c) {
        const int pos = fa::piece_start(pt, c);
        int lo = 0, hi = s.BR - 1;  // entry containing pos
        while (lo < hi) {
            int mid = (lo + hi + 1) / 2;
            if (pre[mid] <= pos) lo = mid; else hi = mid - 1;
        }
        const int w = (pre[lo + 1] - pre[lo]) / s.Hkv;  // positions per unit of the entry
        if (w > 0) {
            const int off = (pos - pre[lo]) % w;  // a boundary strictly inside a unit's tiles splits it
            if (off > 0 && off < w - seg_cost) split = true;
        }
    }
    *W_out = W;
    *pt_out = pt;
    *need_combine = split || empty_unit;
}

int log2_exact(int v) {
    int k = 0;
    while ((1 << k) < v) ++k;
    return k;
}

// Plans the call; may change the row blocking of `s` (the tcgen05 split-KV
// kernel takes row blocks of 16 to 64 packed rows).
// rows_override: the number of output rows when it is not B * Hq * Lq (packed
// variable-length inputs: Hq * total_q).
fa_status make_plan(Shapes &s, int causal, int num_splits, bool kvcache, int64_t max_keys, Plan *pl,
                    int64_t rows_override = -1) {
    DeviceState *dev = nullptr;
    fa_status st = device_state(&dev);
    if (st) return st;
    int variant = choose_variant(s);
    // Calls with at least 128 packed rows (prefill-shaped) on dense K / V run on
    // the tcgen05 kernel: 128 rows fill its M side, and the whole key range is
    // one CTA's work (no split, no combine).  Its time is then one CTA's walk
    // over the keys, so it needs enough CTAs to beat the split-KV kernel, which
    // spreads the keys over every SM (measured with 64-dim heads: 2 CTAs lose at
    // every key length, 32 CTAs win from 128 keys on, 128 CTAs win 4-8x).
    const bool tc_dims = (s.Dqk == s.Dv && (s.Dqk == 128 || s.Dqk == 64)) || (s.Dqk == 192 && s.Dv == 128);
    const int64_t tc_ctas = (int64_t)((s.R + 127) / 128) * s.Hkv * s.B;
    const bool tc_shape = !kvcache && s.R >= 128 && tc_dims && tc_ctas >= 32;
    if (variant == FA_VARIANT_TCGEN05 || (g_force_variant.load() == FA_VARIANT_AUTO && tc_shape)) {
        if (kvcache || !tc_dims)
            return fail(FA_ERR_UNSUPPORTED,
                        "the tcgen05 variant handles dense fa_fwd calls with head dims 64/64, 128/128 or 192/128");
        // Two 128-row tiles per CTA while that still gives every SM a CTA (the
        // tiles' softmax and products overlap); with fewer CTAs than SMs one
        // tile per CTA, in the same MMA-warp pipeline with S double-buffered.
        int form = g_force_tc_form.load();
        if (form == FA_TCGEN05_AUTO) {
            const int64_t pairs = (int64_t)((s.R + 255) / 256) * s.Hkv * s.B;
            form = pairs >= dev->sms ? FA_TCGEN05_TWO_TILES : FA_TCGEN05_ONE_TILE_MMA;
        }
        if (!fa::get_prefill_kernel(s.dtype, s.Dqk, s.Dv, form, &pl->main))
            return fail(FA_ERR_UNSUPPORTED, "no tcgen05 kernel for dtype %d, head dim %d, form %d", s.dtype, s.Dqk, form);
        if ((st = prepare_fn(pl->main.fn, pl->main.threads, pl->main.smem, &pl->occupancy))) return st;
        pl->prefill = true;
        pl->row_blocks = (s.R + pl->main.rows - 1) / pl->main.rows;
        pl->P = (int)std::min<int64_t>((int64_t)pl->row_blocks * s.Hkv * s.B, INT32_MAX);
        pl->P_param = pl->P;
        pl->min_share = 0;
        pl->W = -1;
        pl->need_combine = pl->need_workspace = false;
        pl->pieces = 0;
        pl->ws_o_off = pl->ws_lse_off = pl->ws_bytes = 0;
        pl->comb_smem = pl->comb_grid = 0;
        if (pl->row_blocks > 65535 * 16 || s.Hkv > 65535 || s.B > 65535)
            return fail(FA_ERR_UNSUPPORTED, "grid too large for the tcgen05 variant");
        return FA_OK;
    }
    // More than 8 packed rows (a GQA group with several query positions): the
    // tcgen05 split-KV kernel takes them as one unit of up to 64 rows, so K / V
    // are streamed once for the whole group instead of once per 8 rows.  Its
    // fixed cost per call is higher (measured on GQA-8, qLen 4: 12.5 vs 4.0 us
    // at 128 keys, 28 vs 20 us at 8K keys, while at 32K keys or batch 4 x 8K
    // it wins 47 vs 59-67 us and at batch 16 x 8K 117 vs 303 us), so it is
    // chosen once the re-reads it saves reach kTcSplitMinSavedBytes.
    const bool tcs_dims = s.KDv <= 128 && s.KDqk <= 192;
    if (variant == FA_VARIANT_MMA && g_force_variant.load() == FA_VARIANT_AUTO && s.R > fa::kRowsPerCta && tcs_dims) {
        const int nr = s.R <= 16 ? 16 : (s.R <= 32 ? 32 : 64);
        const int64_t kv = (int64_t)s.B * s.Lk * s.Hkv * (s.Dqk + s.Dv) * 2;  // cache capacity for kvcache calls
        const int64_t saved = ((int64_t)(s.R + fa::kRowsPerCta - 1) / fa::kRowsPerCta - (s.R + nr - 1) / nr) * kv;
        if (saved >= kTcSplitMinSavedBytes) variant = FA_VARIANT_TCGEN05_SPLIT;
    }
    bool ok;
    if (variant == FA_VARIANT_TCGEN05_SPLIT) {
        const int nr = s.R <= 16 ? 16 : (s.R <= 32 ? 32 : 64);
        const int tdqk = s.KDqk <= 128 ? 128 : 192;
        ok = tcs_dims && fa::get_tc_split_kernel(s.dtype, tdqk, 128, nr, &pl->main);
        if (ok) {
            s.KDqk = tdqk;  // dims past the call's own read as zeros, as for the other instances
            s.KDv = 128;
            if ((st = set_row_blocks(&s, nr))) return st;
        }
    } else {
        ok = variant == FA_VARIANT_SCALAR ? fa::get_scalar_kernel(s.dtype, s.KDqk, s.KDv, &pl->main)
                                          : fa::get_mma_kernel(s.dtype, s.KDqk, s.KDv,
                                                               // pages in whole 64-column chunks of the call's dims
                                                               s.Dqk == s.KDqk && s.Dv == s.KDv ? s.page : 0,
                                                               &pl->main);
    }
    if (variant == FA_VARIANT_SCALAR && ok && s.R != 1)
        return fail(FA_ERR_UNSUPPORTED, "the scalar variant handles one packed row (g * Lq = 1), got %d", s.R);
    if (!ok) return fail(FA_ERR_UNSUPPORTED, "no kernel for variant %d, dtype %d, head dims (%d, %d)", variant,
                         s.dtype, s.Dqk, s.Dv);
    const bool comb_unit = fa::combine_per_unit((int64_t)s.B * s.RB * s.Hkv, s.rpc, dev->sms);
    if (!fa::get_combine_kernel(s.dtype, s.KDv, comb_unit, &pl->comb))
        return fail(FA_ERR_UNSUPPORTED, "no combine kernel for dtype %d, Dv %d", s.dtype, s.KDv);
    if ((st = prepare_fn(pl->main.fn, pl->main.threads, pl->main.smem, &pl->occupancy))) return st;
    pl->comb_smem = 0;
    int comb_occ = 0;
    if ((st = prepare_fn(pl->comb.fn, pl->comb.threads, pl->comb_smem, &comb_occ))) return st;

    const int TK = pl->main.tile_keys;
    const int tile_shift = log2_exact(TK);
    const int64_t units = (int64_t)s.B * s.RB * s.Hkv;
    // every tile position must fit in 32 bits
    // a segment epilogue and the next segment's start cost about seg_cost
    // tiles of streaming: every unit is weighted by that much more in the
    // partition
    pl->seg_cost = pl->main.variant == FA_VARIANT_TCGEN05_SPLIT ? kTcSegCost : kMmaSegCost;
    const int64_t max_tiles = units * (((int64_t)s.Lk + TK - 1) / TK + pl->seg_cost);
    if (max_tiles >= (int64_t(1) << 31) - 1)
        return fail(FA_ERR_UNSUPPORTED, "problem too large: %lld key tiles", (long long)max_tiles);
    int64_t P;
    if (num_splits > 0) {
        P = units * num_splits;
        pl->min_share = 1;
    } else {
        P = (int64_t)dev->sms * pl->occupancy;
        pl->min_share = kDefaultMinShare;
    }
    if (P > (1 << 20)) P = 1 << 20;
    if (P < 1) P = 1;
    pl->P_param = (int)P;
    if (!kvcache) {
        int W;
        fa::Partition pt;
        bool need;
        host_schedule(s, causal, tile_shift, pl->seg_cost, (int)P, pl->min_share, &W, &pt, &need);
        if (num_splits <= 0 && W <= P) {  // small problem: one tile per CTA, as many CTAs as tiles
            pl->min_share = 1;
            pl->seg_cost = 0;  // (no CTA holds two units: nothing to weigh)
            host_schedule(s, causal, tile_shift, pl->seg_cost, (int)P, pl->min_share, &W, &pt, &need);
        } else if (num_splits <= 0 && (s.RB == 1 || !causal)) {
            // Every unit holds the same t tiles.  With fewer units than CTAs,
            // k = P / units CTAs per unit each taking t / k tiles of one unit
            // -- no piece crosses a unit boundary, so no CTA runs a segment
            // epilogue mid-stream -- when t splits evenly, the pieces are long
            // enough and at most 15 % of the SMs stay idle.
            const int t = fa::unit_tiles(s.Lk, 0, s.R, s.Lq, causal, tile_shift, s.rpc);
            const int64_t k = units > 0 ? P / units : 0;
            if (t > 0 && k >= 2 && t % k == 0 && t / k >= kAlignedMinTiles && units * k * 20 >= P * 17) {
                P = units * k;
                pl->P_param = (int)P;
                pl->seg_cost = 0;
                host_schedule(s, causal, tile_shift, pl->seg_cost, (int)P, pl->min_share, &W, &pt, &need);
            }
        }
        pl->W = W;
        pl->P = W > 0 ? pt.P : 0;  // W == 0: nothing to stream, the combine writes every row
        pl->need_combine = need;
    } else {
        pl->W = -1;
        pl->P = max_keys > 0 ? (int)P : 0;  // an empty cache: the combine writes every row
        pl->need_combine = true;
    }
    pl->need_workspace = pl->need_combine;
    pl->pieces = (size_t)pl->P_param;  // one piece per CTA
    const size_t o_floats = pl->need_workspace ? pl->pieces * 2 * s.rpc * s.KDv : 0;
    const size_t lse_floats = pl->need_workspace ? pl->pieces * 2 * s.rpc : 0;
    pl->ws_o_off = 0;
    pl->ws_lse_off = pl->ws_o_off + ((o_floats * 4 + 255) & ~size_t(255));
    pl->ws_bytes = pl->need_workspace ? pl->ws_lse_off + ((lse_floats * 4 + 255) & ~size_t(255)) : 0;
    // the combine kernel: a warp per output row, or one to four per unit
    const int64_t nunits = (int64_t)s.B * s.RB * s.Hkv;
    const int64_t nrows = rows_override >= 0 ? rows_override : (int64_t)s.B * s.Hq * s.Lq;
    if (nunits > INT32_MAX || nrows > 4 * (int64_t)INT32_MAX)
        return fail(FA_ERR_UNSUPPORTED, "too many work units (%lld) or rows (%lld)", (long long)nunits,
                    (long long)nrows);
    pl->comb_grid = fa::combine_grid(nrows, nunits, s.rpc, s.R, comb_unit);
    return FA_OK;
}

// ------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// [B, L, H, D] tensor as a 4-D TMA map {D, L, H, B}; box = 64 elements x TK
// rows of one head of one batch, 128-byte swizzle, zero fill out of bounds.
fa_status encode_kv_map(const fa_tensor *t, int box_rows, CUtensorMap *map, const char *name) {
    auto fn = encode_fn();
    if (!fn) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const int64_t elt = 2;
    cuuint64_t dims[4] = {(cuuint64_t)t->shape[3], (cuuint64_t)t->shape[1], (cuuint64_t)t->shape[2],
                          (cuuint64_t)t->shape[0]};
    int64_t st[3] = {t->stride[1], t->stride[2], t->stride[0]};
    // A dimension of extent 1 is never stepped; give it a harmless legal stride.
    int64_t packed = t->shape[3];
    for (int i = 0; i < 3; ++i) {
        if (dims[i + 1] == 1 || st[i] == 0) st[i] = packed;
        packed = st[i] * (int64_t)dims[i + 1];
        if (st[i] % 8) st[i] = (st[i] + 7) / 8 * 8;
    }
    cuuint64_t strides[3] = {(cuuint64_t)(st[0] * elt), (cuuint64_t)(st[1] * elt), (cuuint64_t)(st[2] * elt)};
    cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUtensorMapDataType dt = t->dtype == FA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    // L2 promotion: fetch whole 256-byte (or 128-byte) lines only when every
    // head row starts on such a line and fills it, so a promoted fetch never
    // pulls in bytes of a neighbouring row (a 192-element row is 384 bytes).
    auto rows_fill = [&](uint64_t line) {
        if (reinterpret_cast<uintptr_t>(t->data) % line || (uint64_t)(t->shape[3] * elt) % line) return false;
        for (int i = 0; i < 3; ++i)
            if (dims[i + 1] > 1 && strides[i] % line) return false;
        return true;
    };
    const CUtensorMapL2promotion promo = rows_fill(256)   ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B
                                         : rows_fill(128) ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B
                                                          : CU_TENSOR_MAP_L2_PROMOTION_NONE;
    CUresult r = fn(map, dt, 4, t->data, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FA_ERR_UNSUPPORTED, "%s: cuTensorMapEncodeTiled failed (%d)", name, (int)r);
    return FA_OK;
}

// Paged cache [blocks, page, H, D] (page < tile, D a multiple of 64) as a 5-D
// TMA map {64, page, D / 64, H, blocks}: one box is one page of one head with
// all its 64-column chunks, chunk after chunk in shared memory (128-byte
// swizzle), so a tile takes one box per page for K and one for V instead of
// one per page and chunk.
fa_status encode_page_map(const fa_tensor *t, CUtensorMap *map, const char *name) {
    auto fn = encode_fn();
    if (!fn) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const int64_t elt = 2, D = t->shape[3];
    cuuint64_t dims[5] = {64, (cuuint64_t)t->shape[1], (cuuint64_t)(D / 64), (cuuint64_t)t->shape[2],
                          (cuuint64_t)t->shape[0]};
    // row within the page, chunk, head, block (elements); an extent-1
    // dimension is never stepped and gets a harmless legal stride
    int64_t st[4] = {t->stride[1], 64, t->stride[2], t->stride[0]};
    for (int i = 0; i < 4; ++i)
        if (dims[i + 1] == 1 || st[i] == 0) st[i] = 64;
    cuuint64_t strides[4];
    for (int i = 0; i < 4; ++i) strides[i] = (cuuint64_t)(st[i] * elt);
    cuuint32_t box[5] = {64, (cuuint32_t)t->shape[1], (cuuint32_t)(D / 64), 1, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUtensorMapDataType dt = t->dtype == FA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    // whole head rows are read, so a 256-byte promotion pulls in nothing else
    // when rows start on 256-byte lines and fill them
    const bool lines256 = reinterpret_cast<uintptr_t>(t->data) % 256 == 0 && (D * elt) % 256 == 0 &&
                          (t->shape[1] == 1 || (t->stride[1] * elt) % 256 == 0) &&
                          (t->shape[2] == 1 || (t->stride[2] * elt) % 256 == 0) &&
                          (t->shape[0] == 1 || (t->stride[0] * elt) % 256 == 0);
    CUresult r = fn(map, dt, 5, t->data, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B,
                    lines256 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FA_ERR_UNSUPPORTED, "%s: cuTensorMapEncodeTiled (pages) failed (%d)", name, (int)r);
    return FA_OK;
}

// ------------------------------------------------------------ profiling
struct ProfRec {
    cudaEvent_t e0, e1, e2;
    bool has_comb;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof;
size_t g_prof_used = 0;

// While the stream is being captured into a CUDA graph the events become
// event-record nodes of the graph, so every replay re-times the kernels.
fa_status prof_record(cudaEvent_t *ev, cudaStream_t stream) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(stream, &cs);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
    e = cs == cudaStreamCaptureStatusActive ? cudaEventRecordWithFlags(*ev, stream, cudaEventRecordExternal)
                                            : cudaEventRecord(*ev, stream);
    return e == cudaSuccess ? FA_OK : cuda_fail(e, "cudaEventRecord");
}

// ------------------------------------------------------------ the call
fa_status run(Shapes s, const fa_tensor *q, const fa_tensor *k, const fa_tensor *v, fa_tensor *o,
              const int32_t *seqlens, float *lse, int causal, float scale, int num_splits, void *workspace,
              size_t workspace_bytes, cudaStream_t stream, const Paging *pg = nullptr,
              const fa::AppendParams *ap = nullptr, const Varlen *vl = nullptr) {
    if (s.B == 0 || s.Lq == 0) {
        t_disp = {};
        return FA_OK;
    }
    Plan pl;
    fa_status st = make_plan(s, causal, num_splits, seqlens != nullptr || vl != nullptr, s.Lk, &pl,
                             vl ? (int64_t)s.Hq * vl->total_q : -1);
    if (st) return st;
    if (workspace_bytes < pl.ws_bytes)
        return fail(FA_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu required", workspace_bytes,
                    pl.ws_bytes);
    if (pl.ws_bytes && !workspace) return fail(FA_ERR_WORKSPACE, "workspace pointer is null");
    if (pl.ws_bytes && (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return fail(FA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return fail(FA_ERR_INVALID_ARG, "lse must be 4-byte aligned");

    DeviceState *dev = nullptr;
    if ((st = device_state(&dev))) return st;

    fa::Params p = {};
    p.q = q->data;
    p.q_sb = q->stride[0];
    p.q_sl = q->stride[1];
    p.q_sh = q->stride[2];
    p.o = o->data;
    p.o_sb = o->stride[0];
    p.o_sl = o->stride[1];
    p.o_sh = o->stride[2];
    p.lse = lse;
    char *wsb = static_cast<char *>(workspace);
    p.ws_o = pl.ws_bytes ? reinterpret_cast<float *>(wsb + pl.ws_o_off) : nullptr;
    p.ws_lse = pl.ws_bytes ? reinterpret_cast<float *>(wsb + pl.ws_lse_off) : nullptr;
    p.W_host = pl.W >= 0 ? (int)pl.W : -1;
    p.seqlens = seqlens;
    p.status = dev->status;
    p.B = s.B;
    p.Lq = s.Lq;
    p.Hq = s.Hq;
    p.Hkv = s.Hkv;
    p.g = s.g;
    p.R = s.R;
    p.RB = s.RB;
    p.rpc = s.rpc;
    p.Lk = s.Lk;
    p.dqk = s.Dqk;
    p.dv = s.Dv;
    p.wait_limit_ns = kWaitLimitNs;
    p.stall = 0;
    if (const unsigned long long lim = g_stall_next.exchange(0)) {  // test hook, any kernel
        p.wait_limit_ns = lim;
        p.stall = 1;
    }
    p.causal = causal ? 1 : 0;
    float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)s.Dqk);
    p.scale_log2 = sc * 1.4426950408889634f;
    p.P = pl.P_param;
    p.min_share = pl.min_share;
    p.tile_keys = pl.main.tile_keys;
    p.tile_shift = log2_exact(pl.main.tile_keys);
    p.seg_cost = pl.seg_cost;
    p.lse_sb = (int64_t)s.Hq * s.Lq;
    p.lse_sh = s.Lq;
    if (vl) {
        p.cu_q = vl->cu_q;
        p.cu_k = vl->cu_k;
        p.total_q = vl->total_q;
        p.q_sb = 0;
        p.o_sb = 0;
        p.lse_sb = 0;
        p.lse_sh = vl->total_q;
    }
    if (pg) {
        p.block_table = pg->block_table;
        p.bt_stride = pg->bt_stride;
        p.max_pages = pg->max_pages;
        p.page_shift = log2_exact((int)k->shape[1]);
        p.num_blocks = (int)k->shape[0];
        // pages smaller than a tile on the mma.sync kernel's page-interleaved
        // instance: one 5-D box per page
        p.kv_ilv = pl.main.ilv;
    }

    if (ap) {
        // KV append first: the split-KV kernel then sees seqlens[b] + Lnew keys
        p.seqlen_add = ap->Lnew;
        fa::KernelInfo ak;
        fa::append_kernel_info(&ak);
        int occ = 0;
        if ((st = prepare_fn(ak.fn, ak.threads, 0, &occ))) return st;
        const long long rows = (long long)ap->B * ap->Lnew * ap->Hkv;
        if (rows > 0) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)((rows + ak.threads / 32 - 1) / (ak.threads / 32)));
            cfg.blockDim = dim3((unsigned)ak.threads);
            cfg.stream = stream;
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            at[0].val.programmaticStreamSerializationAllowed = 1;
            cfg.attrs = at;
            cfg.numAttrs = 1;
            fa::AppendParams a = *ap;
            void *args[] = {&a};
            cudaError_t e = cudaLaunchKernelExC(&cfg, ak.fn, args);
            if (e != cudaSuccess) return cuda_fail(e, "launch of the KV append kernel");
            g_launches.fetch_add(1);
        }
    }

    bool prof = false;
    ProfRec *rec = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_prof_mu);
        if (g_prof_on) {
            if (g_prof_used == g_prof.size() && g_prof.size() < 65536) {
                ProfRec r = {};
                if (cudaEventCreate(&r.e0) == cudaSuccess && cudaEventCreate(&r.e1) == cudaSuccess &&
                    cudaEventCreate(&r.e2) == cudaSuccess)
                    g_prof.push_back(r);
            }
            if (g_prof_used < g_prof.size()) {
                rec = &g_prof[g_prof_used++];
                prof = true;
            }
        }
    }

    if (pl.prefill) {
        CUtensorMap tmK, tmV;
        if ((st = encode_kv_map(k, pl.main.tile_keys, &tmK, "k"))) return st;
        if ((st = encode_kv_map(v, pl.main.tile_keys, &tmV, "v"))) return st;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)pl.row_blocks, (unsigned)s.Hkv, (unsigned)s.B);
        cfg.blockDim = dim3((unsigned)pl.main.threads);
        cfg.dynamicSmemBytes = (size_t)pl.main.smem;
        cfg.stream = stream;
        void *args[] = {&tmK, &tmV, &p};
        if (prof && (st = prof_record(&rec->e0, stream))) return st;
        cudaError_t e = cudaLaunchKernelExC(&cfg, pl.main.fn, args);
        if (e != cudaSuccess) return cuda_fail(e, "launch of the tcgen05 kernel");
        g_launches.fetch_add(1);
        if (prof) {
            rec->has_comb = false;
            if ((st = prof_record(&rec->e1, stream)) || (st = prof_record(&rec->e2, stream))) return st;
        }
    }
    const bool launch_main = pl.P > 0 && !pl.prefill;
    if (launch_main) {
        CUtensorMap tmK, tmV;
        const int box_rows = pg ? (int)std::min<int64_t>(k->shape[1], pl.main.tile_keys) : pl.main.tile_keys;
        if (p.kv_ilv) {
            if ((st = encode_page_map(k, &tmK, "k_pages"))) return st;
            if ((st = encode_page_map(v, &tmV, "v_pages"))) return st;
        } else {
            if ((st = encode_kv_map(k, box_rows, &tmK, "k"))) return st;
            if ((st = encode_kv_map(v, box_rows, &tmV, "v"))) return st;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)pl.P);
        cfg.blockDim = dim3((unsigned)pl.main.threads);
        cfg.dynamicSmemBytes = (size_t)pl.main.smem;
        cfg.stream = stream;
        // Programmatic dependent launch: the kernel's prologue may overlap the
        // previous kernel in the stream; it waits for it before touching memory.
        cudaLaunchAttribute mattr[1];
        mattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        mattr[0].val.programmaticStreamSerializationAllowed = 1;
        if (!prof) {
            cfg.attrs = mattr;
            cfg.numAttrs = 1;
        }
        void *args[] = {&tmK, &tmV, &p};
        if (prof && (st = prof_record(&rec->e0, stream))) return st;
        cudaError_t e = cudaLaunchKernelExC(&cfg, pl.main.fn, args);
        if (e != cudaSuccess) return cuda_fail(e, "launch of the split-KV kernel");
        g_launches.fetch_add(1);
        if (prof && (st = prof_record(&rec->e1, stream))) return st;
    } else if (prof && !pl.prefill) {
        if ((st = prof_record(&rec->e0, stream)) || (st = prof_record(&rec->e1, stream))) return st;
    }
    if (pl.need_combine) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)pl.comb_grid);
        cfg.blockDim = dim3((unsigned)pl.comb.threads);
        cfg.dynamicSmemBytes = (size_t)pl.comb_smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        if (launch_main && !prof) {  // an event between the kernels would break the overlap anyway
            cfg.attrs = attr;
            cfg.numAttrs = 1;
        }
        void *args[] = {&p};
        cudaError_t e = cudaLaunchKernelExC(&cfg, pl.comb.fn, args);
        if (e != cudaSuccess) return cuda_fail(e, "launch of the combine kernel");
        g_launches.fetch_add(1);
    }
    if (prof && !pl.prefill) {
        rec->has_comb = pl.need_combine;
        if ((st = prof_record(&rec->e2, stream))) return st;
    }

    fa_dispatch_info d = {};
    d.variant = pl.main.variant;
    d.grid = pl.P;
    d.block = pl.main.threads;
    d.smem_bytes = pl.main.smem;
    d.tile_keys = pl.main.tile_keys;
    d.stages = pl.main.stages;
    d.rows_per_cta = pl.prefill ? pl.main.rows : s.rpc;
    d.units = (int)((int64_t)s.B * s.RB * s.Hkv);
    d.min_share_tiles = pl.min_share;
    d.combine_launched = pl.need_combine ? 1 : 0;
    d.work_tiles = pl.W;
    d.tcgen05_form = pl.prefill ? pl.main.form : 0;
    t_disp = d;
    t_err.clear();
    return FA_OK;
}

}  // namespace

void fa::set_last_error(const char *msg) { t_err = msg ? msg : ""; }

// ====================================================================== C ABI
extern "C" {

fa_status fa_fwd(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v, fa_tensor *o, float *lse, int causal,
                 float scale, int num_splits, void *workspace, size_t workspace_bytes, void *stream) {
    Shapes s;
    fa_status st = check_shapes(q, k, v, o, &s);
    if (st) return st;
    if (!o) return fail(FA_ERR_INVALID_ARG, "o: null descriptor");
    if (!std::isfinite(scale)) return fail(FA_ERR_INVALID_ARG, "scale must be finite");
    return run(s, q, k, v, o, nullptr, lse, causal, scale, num_splits, workspace, workspace_bytes,
               static_cast<cudaStream_t>(stream));
}

fa_status fa_fwd_workspace_size(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v, int causal,
                                int num_splits, size_t *bytes) {
    if (!bytes) return fail(FA_ERR_INVALID_ARG, "bytes: null pointer");
    Shapes s;
    fa_status st = check_shapes(q, k, v, nullptr, &s);
    if (st) return st;
    if (s.B == 0 || s.Lq == 0) {
        *bytes = 0;
        return FA_OK;
    }
    Plan pl;
    if ((st = make_plan(s, causal, num_splits, false, s.Lk, &pl))) return st;
    *bytes = pl.ws_bytes;
    return FA_OK;
}

fa_status fa_decode_kvcache(const fa_tensor *q, const fa_tensor *k_cache, const fa_tensor *v_cache,
                            const int32_t *cache_seqlens, fa_tensor *o, float *lse, int num_splits, int causal,
                            float scale, void *workspace, size_t workspace_bytes, void *stream) {
    Shapes s;
    fa_status st = check_shapes(q, k_cache, v_cache, o, &s);
    if (st) return st;
    if (!o) return fail(FA_ERR_INVALID_ARG, "o: null descriptor");
    if (!cache_seqlens && s.B > 0) return fail(FA_ERR_INVALID_ARG, "cache_seqlens: null pointer");
    if (cache_seqlens && (reinterpret_cast<uintptr_t>(cache_seqlens) & 3u))
        return fail(FA_ERR_INVALID_ARG, "cache_seqlens must be 4-byte aligned");
    if (!std::isfinite(scale)) return fail(FA_ERR_INVALID_ARG, "scale must be finite");
    return run(s, q, k_cache, v_cache, o, cache_seqlens, lse, causal, scale, num_splits, workspace,
               workspace_bytes, static_cast<cudaStream_t>(stream));
}

fa_status fa_decode_kvcache_workspace_size(const fa_tensor *q, const fa_tensor *k_cache, const fa_tensor *v_cache,
                                           int num_splits, size_t *bytes) {
    if (!bytes) return fail(FA_ERR_INVALID_ARG, "bytes: null pointer");
    Shapes s;
    fa_status st = check_shapes(q, k_cache, v_cache, nullptr, &s);
    if (st) return st;
    if (s.B == 0 || s.Lq == 0) {
        *bytes = 0;
        return FA_OK;
    }
    Plan pl;
    if ((st = make_plan(s, 0, num_splits, true, s.Lk, &pl))) return st;
    *bytes = pl.ws_bytes;
    return FA_OK;
}

fa_status fa_decode_kvcache_paged(const fa_tensor *q, const fa_tensor *k_pages, const fa_tensor *v_pages,
                                  const int32_t *block_table, int64_t block_table_stride, int max_blocks_per_seq,
                                  const int32_t *cache_seqlens, fa_tensor *o, float *lse, int num_splits, int causal,
                                  float scale, void *workspace, size_t workspace_bytes, void *stream) {
    const Paging pg = {block_table, block_table_stride, max_blocks_per_seq, 0, 0};
    Shapes s;
    fa_status st = check_shapes(q, k_pages, v_pages, o, &s, &pg);
    if (st) return st;
    if (!o) return fail(FA_ERR_INVALID_ARG, "o: null descriptor");
    if (s.B > 0 && !cache_seqlens) return fail(FA_ERR_INVALID_ARG, "cache_seqlens: null pointer");
    if (s.B > 0 && !block_table) return fail(FA_ERR_INVALID_ARG, "block_table: null pointer");
    if ((reinterpret_cast<uintptr_t>(cache_seqlens) | reinterpret_cast<uintptr_t>(block_table)) & 3u)
        return fail(FA_ERR_INVALID_ARG, "cache_seqlens and block_table must be 4-byte aligned");
    if (!std::isfinite(scale)) return fail(FA_ERR_INVALID_ARG, "scale must be finite");
    return run(s, q, k_pages, v_pages, o, cache_seqlens, lse, causal, scale, num_splits, workspace, workspace_bytes,
               static_cast<cudaStream_t>(stream), &pg);
}

fa_status fa_decode_kvcache_paged_workspace_size(const fa_tensor *q, const fa_tensor *k_pages,
                                                 const fa_tensor *v_pages, int max_blocks_per_seq, int num_splits,
                                                 size_t *bytes) {
    if (!bytes) return fail(FA_ERR_INVALID_ARG, "bytes: null pointer");
    const Paging pg = {nullptr, max_blocks_per_seq, max_blocks_per_seq, 0, 0};
    Shapes s;
    fa_status st = check_shapes(q, k_pages, v_pages, nullptr, &s, &pg);
    if (st) return st;
    if (s.B == 0 || s.Lq == 0) {
        *bytes = 0;
        return FA_OK;
    }
    Plan pl;
    if ((st = make_plan(s, 0, num_splits, true, s.Lk, &pl))) return st;
    *bytes = pl.ws_bytes;
    return FA_OK;
}

fa_status fa_decode_kvcache_append(const fa_tensor *q, const fa_tensor *k_new, const fa_tensor *v_new,
                                   fa_tensor *k_cache, fa_tensor *v_cache, const int32_t *block_table,
                                   int64_t block_table_stride, int max_blocks_per_seq, const int32_t *cache_seqlens,
                                   fa_tensor *o, float *lse, int num_splits, int causal, float scale, void *workspace,
                                   size_t workspace_bytes, void *stream) {
    const Paging pg = {block_table, block_table_stride, max_blocks_per_seq, 0, 0};
    Shapes s;
    fa_status st = check_shapes(q, k_cache, v_cache, o, &s, block_table ? &pg : nullptr);
    if (st) return st;
    if (!o) return fail(FA_ERR_INVALID_ARG, "o: null descriptor");
    if (s.B > 0 && !cache_seqlens) return fail(FA_ERR_INVALID_ARG, "cache_seqlens: null pointer");
    if ((reinterpret_cast<uintptr_t>(cache_seqlens) | reinterpret_cast<uintptr_t>(block_table)) & 3u)
        return fail(FA_ERR_INVALID_ARG, "cache_seqlens and block_table must be 4-byte aligned");
    if (!std::isfinite(scale)) return fail(FA_ERR_INVALID_ARG, "scale must be finite");
    if ((st = check_tensor(k_new, "k_new")) || (st = check_tensor(v_new, "v_new"))) return st;
    if (k_new->dtype != q->dtype || v_new->dtype != q->dtype)
        return fail(FA_ERR_INVALID_ARG, "k_new and v_new must have q's element type");
    const int64_t Lnew = k_new->shape[1];
    if (k_new->shape[0] != s.B || k_new->shape[2] != s.Hkv || k_new->shape[3] != s.Dqk || v_new->shape[0] != s.B ||
        v_new->shape[1] != Lnew || v_new->shape[2] != s.Hkv || v_new->shape[3] != s.Dv)
        return fail(FA_ERR_INVALID_ARG, "k_new / v_new must be [B, Lnew, Hkv, Dqk] / [B, Lnew, Hkv, Dv]");
    if (Lnew > INT32_MAX / 4) return fail(FA_ERR_UNSUPPORTED, "Lnew too large");
    fa::AppendParams a = {};
    a.k_new = k_new->data;
    a.v_new = v_new->data;
    for (int i = 0; i < 3; ++i) {
        a.kn[i] = k_new->stride[i];
        a.vn[i] = v_new->stride[i];
        a.kc[i] = k_cache->stride[i];
        a.vc[i] = v_cache->stride[i];
    }
    a.k_cache = k_cache->data;
    a.v_cache = v_cache->data;
    a.seqlens = cache_seqlens;
    a.block_table = block_table;
    a.bt_stride = block_table_stride;
    a.max_pages = max_blocks_per_seq;
    a.page_shift = block_table ? log2_exact((int)k_cache->shape[1]) : 0;
    a.num_blocks = block_table ? (int)k_cache->shape[0] : 0;
    a.B = s.B;
    a.Lnew = (int)Lnew;
    a.Hkv = s.Hkv;
    a.Dqk = s.Dqk;
    a.Dv = s.Dv;
    a.capacity = s.Lk;
    return run(s, q, k_cache, v_cache, o, cache_seqlens, lse, causal, scale, num_splits, workspace, workspace_bytes,
               static_cast<cudaStream_t>(stream), block_table ? &pg : nullptr, &a);
}

// q [1, total_q, Hq, Dqk], k [1, total_k, Hkv, Dqk], v [1, total_k, Hkv, Dv],
// o [1, total_q, Hq, Dv] (o may be null for the workspace query).
fa_status check_varlen(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v, const fa_tensor *o, int batch,
                       int max_q, int max_k, Shapes *s) {
    fa_status st;
    if ((st = check_tensor(q, "q")) || (st = check_tensor(k, "k")) || (st = check_tensor(v, "v"))) return st;
    if (o && (st = check_tensor(o, "o"))) return st;
    if (k->dtype != q->dtype || v->dtype != q->dtype || (o && o->dtype != q->dtype))
        return fail(FA_ERR_INVALID_ARG, "q, k, v and o must share one element type");
    if (q->shape[0] != 1 || k->shape[0] != 1 || v->shape[0] != 1 || (o && o->shape[0] != 1))
        return fail(FA_ERR_INVALID_ARG, "packed tensors are [1, total, H, D]");
    if (batch < 0 || max_q < 0 || max_k < 0) return fail(FA_ERR_INVALID_ARG, "negative batch or length");
    if (q->shape[1] > INT32_MAX / 2 || k->shape[1] > INT32_MAX / 2)
        return fail(FA_ERR_UNSUPPORTED, "too many packed tokens");
    s->dtype = q->dtype;
    s->B = batch;
    s->Lq = max_q;
    s->Hq = (int)q->shape[2];
    s->Dqk = (int)q->shape[3];
    s->Lk = max_k;
    s->Hkv = (int)k->shape[2];
    s->Dv = (int)v->shape[3];
    if (k->shape[3] != s->Dqk || v->shape[1] != k->shape[1] || v->shape[2] != s->Hkv)
        return fail(FA_ERR_INVALID_ARG, "k / v must be [1, total_k, Hkv, D] with q's Dqk");
    if (o && (o->shape[1] != q->shape[1] || o->shape[2] != s->Hq || o->shape[3] != s->Dv))
        return fail(FA_ERR_INVALID_ARG, "o must be [1, total_q, Hq, Dv]");
    if (s->Hkv <= 0 || s->Hq <= 0 || s->Hq % s->Hkv)
        return fail(FA_ERR_INVALID_ARG, "Hq (%d) must be a positive multiple of Hkv (%d)", s->Hq, s->Hkv);
    if ((st = kernel_dims(s))) return st;
    s->g = s->Hq / s->Hkv;
    const int64_t R = (int64_t)s->g * s->Lq;
    if (R > INT32_MAX / 2) return fail(FA_ERR_UNSUPPORTED, "g * max_seqlen_q too large");
    s->R = (int)R;
    return set_row_blocks(s, fa::kRowsPerCta);
}

fa_status fa_fwd_varlen(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v, const int32_t *cu_seqlens_q,
                        const int32_t *cu_seqlens_k, int batch, int max_seqlen_q, int max_seqlen_k, fa_tensor *o,
                        float *lse, int causal, float scale, int num_splits, void *workspace, size_t workspace_bytes,
                        void *stream) {
    Shapes s;
    fa_status st = check_varlen(q, k, v, o, batch, max_seqlen_q, max_seqlen_k, &s);
    if (st) return st;
    if (!o) return fail(FA_ERR_INVALID_ARG, "o: null descriptor");
    if (batch > 0 && (!cu_seqlens_q || !cu_seqlens_k))
        return fail(FA_ERR_INVALID_ARG, "cu_seqlens_q / cu_seqlens_k: null pointer");
    if ((reinterpret_cast<uintptr_t>(cu_seqlens_q) | reinterpret_cast<uintptr_t>(cu_seqlens_k)) & 3u)
        return fail(FA_ERR_INVALID_ARG, "cu_seqlens must be 4-byte aligned");
    if (!std::isfinite(scale)) return fail(FA_ERR_INVALID_ARG, "scale must be finite");
    const Varlen vl = {cu_seqlens_q, cu_seqlens_k, (int)q->shape[1]};
    if (vl.total_q == 0) {
        t_disp = {};
        return FA_OK;
    }
    return run(s, q, k, v, o, nullptr, lse, causal, scale, num_splits, workspace, workspace_bytes,
               static_cast<cudaStream_t>(stream), nullptr, nullptr, &vl);
}

fa_status fa_fwd_varlen_workspace_size(const fa_tensor *q, const fa_tensor *k, const fa_tensor *v, int batch,
                                       int max_seqlen_q, int max_seqlen_k, int num_splits, size_t *bytes) {
    if (!bytes) return fail(FA_ERR_INVALID_ARG, "bytes: null pointer");
    Shapes s;
    fa_status st = check_varlen(q, k, v, nullptr, batch, max_seqlen_q, max_seqlen_k, &s);
    if (st) return st;
    if (s.B == 0 || s.Lq == 0) {
        *bytes = 0;
        return FA_OK;
    }
    Plan pl;
    if ((st = make_plan(s, 0, num_splits, true, s.Lk, &pl))) return st;
    *bytes = pl.ws_bytes;
    return FA_OK;
}

fa_status fa_check_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    DeviceState *dev = nullptr;
    fa_status st = device_state(&dev);
    if (st) return st;
    unsigned v = 0;
    e = cudaMemcpy(&v, dev->status, sizeof(v), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
    if (v) {
        unsigned zero = 0;
        cudaMemcpy(dev->status, &zero, sizeof(zero), cudaMemcpyHostToDevice);
        if (v & fa::kStatusLayout)
            return fail(FA_ERR_CUDA, "a kernel found its shared-memory base misaligned and wrote nothing (status 0x%x)",
                        v);
        return fail(FA_ERR_TIMEOUT, "a kernel gave up waiting on its copy pipeline (status 0x%x)", v);
    }
    t_err.clear();
    return FA_OK;
}

const char *fa_last_error(void) { return t_err.c_str(); }

void fa_last_dispatch(fa_dispatch_info *info) {
    if (info) *info = t_disp;
}

fa_status fa_force_variant(int variant) {
    if (variant < FA_VARIANT_AUTO || variant > FA_VARIANT_TCGEN05_SPLIT)
        return fail(FA_ERR_INVALID_ARG, "unknown variant %d", variant);
    g_force_variant.store(variant);
    return FA_OK;
}

fa_status fa_test_stall_next_call(unsigned long long wait_limit_ns) {
    if (wait_limit_ns == 0 || wait_limit_ns > kWaitLimitNs)
        return fail(FA_ERR_INVALID_ARG, "wait limit %llu ns: must be in (0, %llu]", wait_limit_ns, kWaitLimitNs);
    g_stall_next.store(wait_limit_ns);
    return FA_OK;
}

fa_status fa_force_tcgen05_form(int form) {
    if (form < FA_TCGEN05_AUTO || form > FA_TCGEN05_ONE_TILE_MMA || form == FA_TCGEN05_ONE_TILE)
        return fail(FA_ERR_INVALID_ARG, "unknown or retired tcgen05 form %d", form);
    g_force_tc_form.store(form);
    return FA_OK;
}

fa_status fa_profile_enable(int on) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_on = on != 0;
    if (g_prof_on) g_prof_used = 0;
    return FA_OK;
}

fa_status fa_profile_read(double *main_ms, int64_t *main_launches, double *combine_ms, int64_t *combine_launches) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    double mm = 0, cm = 0;
    int64_t mn = 0, cn = 0;
    for (size_t i = 0; i < g_prof_used; ++i) {
        float a = 0, b = 0;
        cudaError_t e = cudaEventElapsedTime(&a, g_prof[i].e0, g_prof[i].e1);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventElapsedTime");
        mm += a;
        ++mn;
        if (g_prof[i].has_comb) {
            e = cudaEventElapsedTime(&b, g_prof[i].e1, g_prof[i].e2);
            if (e != cudaSuccess) return cuda_fail(e, "cudaEventElapsedTime");
            cm += b;
            ++cn;
        }
    }
    if (main_ms) *main_ms = mm;
    if (main_launches) *main_launches = mn;
    if (combine_ms) *combine_ms = cm;
    if (combine_launches) *combine_launches = cn;
    return FA_OK;
}

fa_status fa_schedule(int B, int Lq, int Hq, int Hkv, int Lk, int causal, const int32_t *seqlens, int num_ctas,
                      int min_share, int tile_keys, int rows_per_cta, int seg_cost, int64_t *work_tiles,
                      int64_t *ctas_used, int32_t *unit_tiles, int64_t *unit_first_cta, int64_t *unit_last_cta,
                      int64_t max_units) {
    if (B < 0 || Lq < 0 || Hq <= 0 || Hkv <= 0 || Lk < 0 || Hq % Hkv || num_ctas < 1 || min_share < 1 ||
        tile_keys < 1 || (tile_keys & (tile_keys - 1)) || max_units < 0 || rows_per_cta < 1 ||
        rows_per_cta > fa::kMaxRowsPerCta || seg_cost < 0 || seg_cost > 1024)
        return fail(FA_ERR_INVALID_ARG, "fa_schedule: inconsistent sizes");
    const int g = Hq / Hkv, R = g * Lq, RB = (R + rows_per_cta - 1) / rows_per_cta;
    const int shift = log2_exact(tile_keys);
    const int64_t BR = (int64_t)B * RB;
    if (BR * Hkv * (((int64_t)Lk + tile_keys - 1) / tile_keys + seg_cost) >= (int64_t(1) << 31) - 1)
        return fail(FA_ERR_UNSUPPORTED, "fa_schedule: problem too large");
    std::vector<int> pre(BR + 1, 0);
    std::vector<int32_t> tx(BR, 0);
    for (int64_t x = 0; x < BR; ++x) {
        int n = fa::batch_keys(seqlens, (int)(x / RB), Lk);
        tx[x] = fa::unit_tiles(n, (int)(x % RB), R, Lq, causal, shift, rows_per_cta);
        pre[x + 1] = pre[x] + Hkv * fa::unit_weight(tx[x], seg_cost);
    }
    const int W = pre[BR];
    const fa::Partition pt = fa::make_partition(W, num_ctas, min_share);
    if (work_tiles) *work_tiles = W;
    if (ctas_used) *ctas_used = pt.P;
    int64_t u = 0;
    for (int64_t x = 0; x < BR && u < max_units; ++x)
        for (int h = 0; h < Hkv && u < max_units; ++h, ++u) {
            const int u0 = pre[x] + h * fa::unit_weight(tx[x], seg_cost);
            if (unit_tiles) unit_tiles[u] = tx[x];
            const bool has = tx[x] > 0;
            if (unit_first_cta) unit_first_cta[u] = has ? fa::piece_of(pt, u0) : -1;
            if (unit_last_cta) unit_last_cta[u] = has ? fa::piece_of(pt, u0 + tx[x] - 1) : -1;
        }
    t_err.clear();
    return FA_OK;
}

int64_t fa_launch_count(void) { return g_launches.load(); }

const char *fa_version(void) { return "fa_b200 0.1.0 (sm_100a)"; }

}  // extern "C"
