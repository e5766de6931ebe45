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
};

// Main split-KV kernel using mma.sync (keys as M, packed rows as N).
bool get_mma_kernel(int dtype, int dqk, int dv, KernelInfo *out);
// LSE-weighted combine of split partials.
bool get_combine_kernel(int dtype, int dv, KernelInfo *out);

// Main split-KV kernel using fp32 FMA dot products (one packed row).
bool get_scalar_kernel(int dtype, int dqk, int dv, KernelInfo *out);

// Sets the calling thread's fa_last_error() message (for entry points that
// live outside fa_api.cu).
void set_last_error(const char *msg);

}  // namespace fa
