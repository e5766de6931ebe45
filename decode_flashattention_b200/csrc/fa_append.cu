// fa_append.cu -- KV append: copy the new tokens' K and V rows into the cache
// before the attention kernels read it.
//
// Token t of batch b (t < Lnew) goes to cache position cache_seqlens[b] + t:
// row pos of batch b in a dense cache [B, Lmax, Hkv, D], or row pos % page of
// block block_table[b, pos / page] in a paged one [num_blocks, page, Hkv, D].
// A position outside [0, capacity) or a block number outside [0, num_blocks)
// is skipped (nothing is written).  The attention that follows sees
// cache_seqlens[b] + Lnew keys ("paged KV append" is among the verified cases
// of the MXFlashAttn README's capability table; the append-then-attend order
// is that of flash_attn_with_kvcache with new k / v).
//
// One warp per (b, t, kv head) row; lanes move 16-byte chunks.  Launched with
// programmatic dependent launch: it waits for the previous kernel before
// reading or writing memory, and lets the split-KV kernel start its prologue
// early (that kernel waits for this grid to complete before reading K / V).
#include "fa_common.cuh"
#include "fa_internal.h"

namespace fa {

constexpr int kAppendThreads = 256;

__global__ void __launch_bounds__(kAppendThreads) append_kv_kernel(const AppendParams a) {
    pdl_launch_dependents();
    pdl_wait_primary();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * (kAppendThreads / 32) + warp;
    if (row >= (long long)a.B * a.Lnew * a.Hkv) return;
    const int h = (int)(row % a.Hkv);
    const int t = (int)((row / a.Hkv) % a.Lnew);
    const int b = (int)(row / ((long long)a.Hkv * a.Lnew));
    const long long pos = (long long)a.seqlens[b] + t;
    if (pos < 0 || pos >= a.capacity) return;
    long long c0, c1;  // index along the cache's first two dims
    if (a.block_table) {
        const long long page = pos >> a.page_shift;
        if (page >= a.max_pages) return;
        const int blk = a.block_table[(long long)b * a.bt_stride + page];
        if (blk < 0 || blk >= a.num_blocks) return;
        c0 = blk;
        c1 = pos & ((1LL << a.page_shift) - 1);
    } else {
        c0 = b;
        c1 = pos;
    }
    const char *ks = static_cast<const char *>(a.k_new) + 2 * (b * a.kn[0] + t * a.kn[1] + h * a.kn[2]);
    const char *vs = static_cast<const char *>(a.v_new) + 2 * (b * a.vn[0] + t * a.vn[1] + h * a.vn[2]);
    char *kd = static_cast<char *>(a.k_cache) + 2 * (c0 * a.kc[0] + c1 * a.kc[1] + h * a.kc[2]);
    char *vd = static_cast<char *>(a.v_cache) + 2 * (c0 * a.vc[0] + c1 * a.vc[1] + h * a.vc[2]);
    const int kchunks = a.Dqk / 8, vchunks = a.Dv / 8;  // 16-byte chunks per row
    for (int c = lane; c < kchunks + vchunks; c += 32) {
        if (c < kchunks)
            reinterpret_cast<uint4 *>(kd)[c] = reinterpret_cast<const uint4 *>(ks)[c];
        else
            reinterpret_cast<uint4 *>(vd)[c - kchunks] = reinterpret_cast<const uint4 *>(vs)[c - kchunks];
    }
}

void append_kernel_info(KernelInfo *out) {
    out->fn = reinterpret_cast<const void *>(&append_kv_kernel);
    out->threads = kAppendThreads;
    out->smem = 0;
    out->tile_keys = 0;
    out->stages = 0;
    out->variant = 0;
}

}  // namespace fa
