// fa_internal.h -- what the host library needs to know about each compiled
// kernel (shared between the kernel translation units and fa_api.cu).
#pragma once

#include <stdint.h>

namespace fa {

struct KernelInfo {
    const void *fn;  // __global__ function (host stub address)
    int threads;     // block size
    int smem;        // dynamic shared memory bytes
    int tile_keys;   // keys per pipeline stage (main kernels)
    int stages;      // pipeline depth (main kernels)
    int variant;     // fa_variant
    int rows;        // packed query rows per CTA (tcgen05 kernels)
    int form;        // fa_tcgen05_form (tcgen05 kernels)
    int ilv = 0;     // mma.sync kernel: paged pages gathered in 5-D boxes (Params::kv_ilv)
};

// Main split-KV kernel using mma.sync (keys as M, packed rows as N).  page > 0:
// a paged cache whose pages are whole 64-column chunks of the call's head
// dims; pages smaller than the instance's tile take its page-interleaved form.
bool get_mma_kernel(int dtype, int dqk, int dv, int page, KernelInfo *out);
// LSE-weighted combine of split partials (per-row or per-unit form), the
// choice of form for `units` units of row blocks of rpc rows on `sms` SMs, and
// its grid for `rows` output rows (R packed rows per kv head).
bool get_combine_kernel(int dtype, int dv, bool per_unit, KernelInfo *out);
bool combine_per_unit(long long units, int rpc, int sms);
int combine_grid(long long rows, long long units, int rpc, int R, bool per_unit);

// Dense attention on tcgen05 for calls with many packed rows (fa_prefill.cu).
// form: an fa_tcgen05_form other than FA_TCGEN05_AUTO.
bool get_prefill_kernel(int dtype, int dqk, int dv, int form, KernelInfo *out);

// Main split-KV kernel using fp32 FMA dot products (one packed row).
bool get_scalar_kernel(int dtype, int dqk, int dv, KernelInfo *out);

// Split-KV kernel on tcgen05 (fa_splitkv_tc.cu) for row blocks of nr = 16,
// 32 or 64 packed rows; instances (dqk, dv) = (128, 128) and (192, 128).
bool get_tc_split_kernel(int dtype, int dqk, int dv, int nr, KernelInfo *out);

// KV append (fa_append.cu): new K / V rows [B, Lnew, Hkv, D] into a dense
// cache [B, Lmax, Hkv, D] or a paged one [num_blocks, page, Hkv, D] at
// positions cache_seqlens[b] + t.  Strides in elements ({batch or block, row,
// head}); the last dim is contiguous.
struct AppendParams {
    const void *k_new, *v_new;
    int64_t kn[3], vn[3];
    void *k_cache, *v_cache;
    int64_t kc[3], vc[3];
    const int *seqlens;
    const int *block_table;  // null for a dense cache
    int64_t bt_stride;
    int max_pages, page_shift, num_blocks;
    int B, Lnew, Hkv, Dqk, Dv;
    long long capacity;      // keys a batch's cache can hold
};
void append_kernel_info(KernelInfo *out);

// Sets the calling thread's fa_last_error() message (for entry points that
// live outside fa_api.cu).
void set_last_error(const char *msg);

}  // namespace fa
