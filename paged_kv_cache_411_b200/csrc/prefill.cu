// Placeholder until the tcgen05 prefill kernel lands: reports "unsupported".
#include "kernels.h"

namespace pagedkv {

bool prefill_supported(int32_t, int32_t, int32_t) { return false; }

cudaError_t launch_prefill(const PrefillArgs&, cudaStream_t, const char** why) {
    if (why) *why = "prefill kernel not built";
    return cudaErrorNotSupported;
}

}  // namespace pagedkv
