// pa_paged_attention_decode_noalloc: paged decode with library-owned scratch.
//
// pa_paged_attention_decode needs a caller-provided device workspace (its
// split-K plan, work items and fp32 partial results).  Some callers cannot
// allocate one: code that runs inside an allocator-less runtime (an embedded
// inference loop that was handed fixed buffers, a plugin whose host forbids
// cudaMalloc after start-up, or a process that must not take the implicit
// synchronisation and fragmentation a cudaMalloc/cudaFree pair brings).  This
// entry point gives them the same kernels with the scratch taken from a
// fixed-size array that the library itself places in device memory.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds its kNoallocScratchBytes for the life of the process.  Host
// code must not hand the array's name to a kernel: on the host that name is
// only a stand-in.  Its device address is looked up once per device with
// cudaGetSymbolAddress, with that device current, on the first call made on
// that device (so make that first call before any stream capture), and then
// passed to the kernels like any workspace pointer.
//
// All calls on a device share the one array and it keeps whatever the last
// call left in it; the decode kernels write every scratch word they read
// (the plan kernel rewrites the header and the item counter at the start of
// each call), so nothing needs clearing between calls.  Two calls whose
// kernels overlap on the GPU (different streams without ordering, or several
// host threads) race on the array and give wrong results: serialise them.
#include <cuda_runtime.h>

#include <mutex>

#include "common.h"
#include "kernels.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(64) << 20;   // 64 MiB per device

static __device__ __align__(256) unsigned char g_decode_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up once per device).
pa_status scratch_for_current_device(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return pagedkv::fail(PA_ERR_CUDA, "pa_paged_attention_decode_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices)
        return pagedkv::fail(PA_ERR_INVALID_ARG, "pa_paged_attention_decode_noalloc: device %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess || !p)
            return pagedkv::fail(PA_ERR_CUDA, "pa_paged_attention_decode_noalloc: cudaGetSymbolAddress: %s",
                                 cudaGetErrorString(e));
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return PA_OK;
}

}  // namespace

extern "C" pa_status pa_paged_attention_decode_noalloc(pa_half* out, const pa_half* q, const pa_half* k_cache,
                                                       const pa_half* v_cache, const int32_t* block_tables,
                                                       const int32_t* seq_lens, int32_t num_seqs,
                                                       int32_t num_heads, int32_t head_dim, int32_t block_size,
                                                       int32_t max_blocks, int32_t num_blocks, float scale,
                                                       int32_t* err_flag, void* stream) {
    if (num_seqs < 0 || num_heads <= 0 || head_dim <= 0 || block_size <= 0 || max_blocks < 0)
        return pagedkv::fail(PA_ERR_INVALID_ARG, "pa_paged_attention_decode_noalloc: bad sizes");
    // the workspace arithmetic below is only meaningful inside the decode entry point's own limit
    if (static_cast<int64_t>(max_blocks) * block_size > (1 << 30))
        return pagedkv::fail(PA_ERR_INVALID_ARG, "pa_paged_attention_decode_noalloc: max_blocks*block_size too large");
    const size_t need = pagedkv::decode_workspace_bytes(num_seqs, num_heads, head_dim, max_blocks, block_size);
    if (need > kNoallocScratchBytes)
        return pagedkv::fail(PA_ERR_INVALID_ARG,
                             "pa_paged_attention_decode_noalloc: this batch needs %zu bytes of scratch but the "
                             "library's static scratch holds %zu; use pa_paged_attention_decode with a workspace",
                             need, kNoallocScratchBytes);
    void* scratch = nullptr;
    pa_status st = scratch_for_current_device(&scratch);
    if (st != PA_OK) return st;
    return pa_paged_attention_decode(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads,
                                     head_dim, block_size, max_blocks, num_blocks, scale, scratch,
                                     kNoallocScratchBytes, err_flag, stream);
}
