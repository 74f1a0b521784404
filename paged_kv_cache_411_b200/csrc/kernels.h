// Internal launcher interface between the C ABI (capi.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <stddef.h>
#include <stdint.h>

namespace pagedkv {

cudaError_t launch_reshape_and_cache(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                                     const int64_t* slot_mapping, int32_t num_tokens, int32_t num_heads,
                                     int32_t head_dim, int32_t block_size, int32_t num_blocks,
                                     int32_t* err_flag, cudaStream_t stream);

// Heads per decode work item for (num_heads, head_dim); 0 if no kernel instance fits.
int32_t decode_head_group(int32_t num_heads, int32_t head_dim);
bool decode_block_size_ok(int32_t block_size);
size_t decode_workspace_bytes(int32_t num_seqs, int32_t num_heads, int32_t head_dim, int32_t max_blocks,
                              int32_t block_size);

struct DecodeArgs {
    void* out;
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* seq_lens;
    int32_t num_seqs, num_heads, head_dim, block_size, max_blocks, num_blocks;
    float scale;
    void* workspace;
    size_t workspace_bytes;
    int32_t* err_flag;
};

// Returns a CUDA error, or cudaErrorNotSupported / cudaErrorInvalidValue for
// argument problems the caller should have caught.
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream, const char** why);

struct PrefillArgs {
    void* out;
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* q_start;
    const int32_t* ctx_before;
    int32_t num_reqs, num_tokens, num_heads, head_dim, block_size, max_blocks, num_blocks;
    float scale;
    int32_t* err_flag;
};

bool prefill_supported(int32_t num_heads, int32_t head_dim, int32_t block_size);
cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t stream, const char** why);
// The one-query-tile prefill kernel (prefill_q128.cu) that launch_prefill uses for small launches;
// wait_ns and stall are the launch's pipeline-wait limit and failure-detection test switch.
cudaError_t launch_prefill_q128(const PrefillArgs& a, uint64_t wait_ns, bool stall, cudaStream_t stream,
                                const char** why);

// Tensor-map encoding through the driver entry point (no libcuda link).
// Returns false and sets *why on failure.
bool encode_tensor_map_3d(void* map_out, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                          uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1,
                          uint32_t b2, int swizzle_128b, const char** why);

int32_t device_sm_count();
// Raises func's dynamic shared-memory limit to `bytes` on the current device, once per device (the setting
// lives in each device's context); `done` is the caller's per-kernel bitmask of devices already set.
cudaError_t ensure_dynamic_smem(const void* func, int bytes, std::atomic<uint64_t>* done);

// Failure-detection test hook (pa_debug_inject_stall): the next launch of the given kernel
// (kStallDecode / kStallPrefill) gets this pipeline-wait limit and makes its consumer role wait on a
// barrier nothing completes.  Returns 0 (no stall; the default limit) or the limit in ns, and
// clears the request.
constexpr int32_t kStallDecode = 1;
constexpr int32_t kStallPrefill = 2;
uint64_t take_injected_stall(int32_t kernel);
void inject_stall(int32_t kernel, uint64_t limit_ns);

}  // namespace pagedkv
