// fa_splitkv_mma.cu -- the split-KV kernel's tensor-core variant: instances
// and registry (the kernel itself is in fa_splitkv.cuh).
#include "fa_splitkv.cuh"

namespace fa {

template <typename T, int DQK, int DV, int STAGES, int KB = 2>
static void fill(KernelInfo *out) {
    using C = SplitCfg<DQK, DV, STAGES, false, KB>;
    out->fn = reinterpret_cast<const void *>(&splitkv_kernel<T, DQK, DV, STAGES, false, KB>);
    out->threads = kThreads;
    out->smem = C::SMEM;
    out->tile_keys = C::TK;
    out->stages = STAGES;
    out->variant = 1;  // FA_VARIANT_MMA
}

bool get_mma_kernel(int dtype, int dqk, int dv, KernelInfo *out) {
    if (dtype == 0) {
        if (dqk == 64 && dv == 64) { fill<__half, 64, 64, 6>(out); return true; }
        if (dqk == 128 && dv == 128) { fill<__half, 128, 128, 3>(out); return true; }
        if (dqk == 192 && dv == 128) { fill<__half, 192, 128, 2>(out); return true; }
        if (dqk == 256 && dv == 256) { fill<__half, 256, 256, 2, 1>(out); return true; }
    } else if (dtype == 1) {
        if (dqk == 64 && dv == 64) { fill<__nv_bfloat16, 64, 64, 6>(out); return true; }
        if (dqk == 128 && dv == 128) { fill<__nv_bfloat16, 128, 128, 3>(out); return true; }
        if (dqk == 192 && dv == 128) { fill<__nv_bfloat16, 192, 128, 2>(out); return true; }
        if (dqk == 256 && dv == 256) { fill<__nv_bfloat16, 256, 256, 2, 1>(out); return true; }
    }
    return false;
}

}  // namespace fa
