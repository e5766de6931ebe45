// fa_splitkv_mma.cu -- the split-KV kernel's tensor-core variant: instances
// and registry (the kernel itself is in fa_splitkv.cuh).
#include "fa_splitkv.cuh"

namespace fa {

template <typename T, int DQK, int DV, int STAGES, int KB, bool ILV>
static void fill_one(KernelInfo *out) {
    using C = SplitCfg<DQK, DV, STAGES, false, KB, ILV>;
    out->fn = reinterpret_cast<const void *>(&splitkv_kernel<T, DQK, DV, STAGES, false, KB, ILV>);
    out->threads = kThreads;
    out->smem = C::SMEM;
    out->tile_keys = C::TK;
    out->stages = STAGES;
    out->variant = 1;  // FA_VARIANT_MMA
    out->ilv = ILV ? 1 : 0;
}

// The instance for a dense cache, or its page-interleaved form for pages
// smaller than its tile.
template <typename T, int DQK, int DV, int STAGES, int KB = 2>
static void fill(int page, KernelInfo *out) {
    if (page > 0 && page < SplitCfg<DQK, DV, STAGES, false, KB>::TK) fill_one<T, DQK, DV, STAGES, KB, true>(out);
    else fill_one<T, DQK, DV, STAGES, KB, false>(out);
}

bool get_mma_kernel(int dtype, int dqk, int dv, int page, KernelInfo *out) {
    if (dtype == 0) {
        if (dqk == 64 && dv == 64) { fill<__half, 64, 64, 6>(page, out); return true; }
        if (dqk == 128 && dv == 128) { fill<__half, 128, 128, 3>(page, out); return true; }
        if (dqk == 192 && dv == 128) { fill<__half, 192, 128, 2>(page, out); return true; }
        if (dqk == 256 && dv == 256) { fill<__half, 256, 256, 2, 1>(page, out); return true; }
    } else if (dtype == 1) {
        if (dqk == 64 && dv == 64) { fill<__nv_bfloat16, 64, 64, 6>(page, out); return true; }
        if (dqk == 128 && dv == 128) { fill<__nv_bfloat16, 128, 128, 3>(page, out); return true; }
        if (dqk == 192 && dv == 128) { fill<__nv_bfloat16, 192, 128, 2>(page, out); return true; }
        if (dqk == 256 && dv == 256) { fill<__nv_bfloat16, 256, 256, 2, 1>(page, out); return true; }
    }
    return false;
}

}  // namespace fa
