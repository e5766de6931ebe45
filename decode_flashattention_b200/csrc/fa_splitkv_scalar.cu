// fa_splitkv_scalar.cu -- split-KV attention with fp32 FMA dot products for a
// single packed query row (placeholder registry until the kernel lands).
#include "fa_internal.h"

namespace fa {

bool get_scalar_kernel(int, int, int, KernelInfo *) { return false; }

}  // namespace fa
