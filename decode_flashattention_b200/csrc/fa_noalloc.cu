// fa_noalloc.cu -- fa_decode_kvcache_noalloc: the KV-cache decode call for
// callers that cannot allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is off limits -- a plugin
// inside a serving runtime that owns every byte of device memory and forbids
// allocation once it has started, or a latency-critical decode loop that must
// not risk the implicit device-wide synchronisation cudaMalloc/cudaFree may
// perform.  Such a caller can still pass its inputs and outputs, but cannot
// provide the split-KV workspace that fa_decode_kvcache asks for.
//
// How: the workspace comes from a file-scope device array of fixed size
// (kNoAllocScratchBytes) that is part of this library's module, so every GPU
// that loads the library holds it until the process exits.  Host code cannot
// use the array's name as a device address, so once per device, with that
// device current, we ask the runtime for the array's address
// (cudaGetSymbolAddress) and pass that pointer down as the workspace.  That
// set-up happens on the first call made on each device; make that first call
// before any stream capture.  Nothing in the scratch has to start at zero:
// every partial result the combine kernel reads is written earlier in the
// same call.  All calls on a device share the one array and it keeps whatever
// the last call left there, so calls whose GPU work overlaps (different
// streams, or host threads racing on one device) race on it: serialise them.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "fa.h"
#include "fa_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
constexpr int kMaxNoAllocDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxNoAllocDevices] = {};

// Device address of the scratch array on the current device (looked up once).
fa_status scratch_address(void **out, const char **why) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        *why = "cudaGetDevice failed";
        return FA_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxNoAllocDevices) {
        *why = "device index out of range";
        return FA_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            *why = "cudaGetSymbolAddress of the static scratch array failed";
            return FA_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return FA_OK;
}

}  // namespace

extern "C" {

FA_API size_t fa_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

FA_API fa_status fa_decode_kvcache_noalloc(const fa_tensor *q, const fa_tensor *k_cache,
                                           const fa_tensor *v_cache, const int32_t *cache_seqlens,
                                           fa_tensor *o, float *lse, int num_splits, int causal,
                                           float scale, void *stream) {
    size_t need = 0;
    fa_status st = fa_decode_kvcache_workspace_size(q, k_cache, v_cache, num_splits, &need);
    if (st != FA_OK) return st;  // the size query already set the message
    if (need > kNoAllocScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "fa_decode_kvcache_noalloc: these shapes need %zu bytes of scratch, more than the "
                 "library's fixed %zu-byte array; use fa_decode_kvcache with a caller workspace",
                 need, kNoAllocScratchBytes);
        fa::set_last_error(msg);
        return FA_ERR_UNSUPPORTED;
    }
    void *ws = nullptr;
    const char *why = nullptr;
    st = scratch_address(&ws, &why);
    if (st != FA_OK) {
        fa::set_last_error(why);
        return st;
    }
    return fa_decode_kvcache(q, k_cache, v_cache, cache_seqlens, o, lse, num_splits, causal, scale, ws,
                             kNoAllocScratchBytes, stream);
}

}  // extern "C"
