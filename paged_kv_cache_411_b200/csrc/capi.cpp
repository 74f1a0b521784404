// extern "C" device entry points of libpagedkv: argument checks on the host,
// then the launchers.  Nothing here allocates device memory or synchronises.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "common.h"
#include "kernels.h"

namespace pagedkv {
const char* last_error();
}

using pagedkv::fail;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

pa_status cuda_status(cudaError_t e, const char* where, const char* why) {
    if (e == cudaSuccess) return PA_OK;
    if (e == cudaErrorInvalidValue && why) return fail(PA_ERR_INVALID_ARG, "%s: %s", where, why);
    return fail(PA_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorString(e), why ? why : "launch");
}

}  // namespace

extern "C" {

int32_t pa_abi_version(void) { return 2; }

const char* pa_last_error(void) { return pagedkv::last_error(); }

const char* pa_status_string(pa_status s) {
    switch (s) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
        case PA_ERR_OOM: return "PA_ERR_OOM";
        case PA_ERR_NOT_FOUND: return "PA_ERR_NOT_FOUND";
        case PA_ERR_EXISTS: return "PA_ERR_EXISTS";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
        case PA_ERR_CUDA: return "PA_ERR_CUDA";
        case PA_ERR_DEVICE_CHECK: return "PA_ERR_DEVICE_CHECK";
        default: return "PA_ERR_UNKNOWN";
    }
}

pa_status pa_debug_inject_stall(int32_t kernel, uint64_t wait_limit_ns) {
    if (kernel != PA_KERNEL_DECODE && kernel != PA_KERNEL_PREFILL)
        return fail(PA_ERR_INVALID_ARG, "pa_debug_inject_stall: kernel must be PA_KERNEL_DECODE or PA_KERNEL_PREFILL");
    if (wait_limit_ns == 0 || wait_limit_ns > 2000000000ull)
        return fail(PA_ERR_INVALID_ARG, "pa_debug_inject_stall: wait_limit_ns must be in 1 .. 2e9");
    pagedkv::inject_stall(kernel == PA_KERNEL_DECODE ? pagedkv::kStallDecode : pagedkv::kStallPrefill, wait_limit_ns);
    return PA_OK;
}

pa_status pa_check_device_flag(int32_t flag_value) {
    if (flag_value == 0) return PA_OK;
    return fail(PA_ERR_DEVICE_CHECK, "device check flag 0x%x", flag_value);
}

pa_status pa_reshape_and_cache(const pa_half* k_new, const pa_half* v_new, pa_half* k_cache, pa_half* v_cache,
                               const int64_t* slot_mapping, int32_t num_tokens, int32_t num_heads,
                               int32_t head_dim, int32_t block_size, int32_t num_blocks, int32_t* err_flag,
                               void* stream) {
    if (num_tokens < 0 || num_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks < 0)
        return fail(PA_ERR_INVALID_ARG, "pa_reshape_and_cache: bad sizes");
    if ((static_cast<int64_t>(num_heads) * head_dim) % 8 != 0)
        return fail(PA_ERR_UNSUPPORTED, "pa_reshape_and_cache: num_heads*head_dim must be a multiple of 8");
    if (static_cast<int64_t>(num_heads) * head_dim > (1 << 24))
        return fail(PA_ERR_INVALID_ARG, "pa_reshape_and_cache: row too large");
    if (num_tokens == 0) return PA_OK;
    if (!k_new || !v_new || !k_cache || !v_cache || !slot_mapping)
        return fail(PA_ERR_INVALID_ARG, "pa_reshape_and_cache: NULL pointer");
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache))
        return fail(PA_ERR_INVALID_ARG, "pa_reshape_and_cache: buffers must be 16-byte aligned");
    cudaError_t e = pagedkv::launch_reshape_and_cache(k_new, v_new, k_cache, v_cache, slot_mapping, num_tokens,
                                                      num_heads, head_dim, block_size, num_blocks, err_flag,
                                                      static_cast<cudaStream_t>(stream));
    return cuda_status(e, "pa_reshape_and_cache", nullptr);
}

size_t pa_decode_workspace_bytes(int32_t num_seqs, int32_t num_heads, int32_t head_dim, int32_t max_blocks,
                                 int32_t block_size) {
    return pagedkv::decode_workspace_bytes(num_seqs, num_heads, head_dim, max_blocks, block_size);
}

pa_status pa_paged_attention_decode(pa_half* out, const pa_half* q, const pa_half* k_cache, const pa_half* v_cache,
                                    const int32_t* block_tables, const int32_t* seq_lens, int32_t num_seqs,
                                    int32_t num_heads, int32_t head_dim, int32_t block_size, int32_t max_blocks,
                                    int32_t num_blocks, float scale, void* workspace, size_t workspace_bytes,
                                    int32_t* err_flag, void* stream) {
    if (num_seqs < 0 || num_heads <= 0 || head_dim <= 0 || block_size <= 0 || max_blocks < 0 || num_blocks < 0)
        return fail(PA_ERR_INVALID_ARG, "pa_paged_attention_decode: bad sizes");
    if (pagedkv::decode_head_group(num_heads, head_dim) == 0 || !pagedkv::decode_block_size_ok(block_size))
        return fail(PA_ERR_UNSUPPORTED, "pa_paged_attention_decode: no kernel for num_heads=%d head_dim=%d block_size=%d",
                    num_heads, head_dim, block_size);
    if (static_cast<int64_t>(max_blocks) * block_size > (1 << 30))
        return fail(PA_ERR_INVALID_ARG, "pa_paged_attention_decode: max_blocks*block_size too large");
    if (!std::isfinite(scale) || !(scale > 0.f))
        return fail(PA_ERR_INVALID_ARG, "pa_paged_attention_decode: scale must be finite and > 0");
    if (num_seqs == 0) return PA_OK;
    if (num_blocks == 0 || max_blocks == 0)
        return fail(PA_ERR_INVALID_ARG, "pa_paged_attention_decode: empty pool or table with sequences to decode");
    const size_t need = pagedkv::decode_workspace_bytes(num_seqs, num_heads, head_dim, max_blocks, block_size);
    const int64_t max_splits = (static_cast<int64_t>(max_blocks) * block_size + 63) / 64;
    if (static_cast<int64_t>(num_seqs) * num_heads * max_splits >= (int64_t(1) << 31))
        return fail(PA_ERR_INVALID_ARG, "pa_paged_attention_decode: too many work items");
    if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens || !workspace)
        return fail(PA_ERR_INVALID_ARG, "pa_paged_attention_decode: NULL pointer");
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
        return fail(PA_ERR_INVALID_ARG, "pa_paged_attention_decode: fp16 buffers must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(PA_ERR_INVALID_ARG, "pa_paged_attention_decode: workspace must be 256-byte aligned");
    if (workspace_bytes < need)
        return fail(PA_ERR_INVALID_ARG, "pa_paged_attention_decode: workspace %zu < %zu bytes", workspace_bytes, need);
    pagedkv::DecodeArgs a{out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads, head_dim,
                          block_size, max_blocks, num_blocks, scale, workspace, workspace_bytes, err_flag};
    const char* why = nullptr;
    cudaError_t e = pagedkv::launch_decode(a, static_cast<cudaStream_t>(stream), &why);
    return cuda_status(e, "pa_paged_attention_decode", why);
}

pa_status pa_paged_attention_prefill_chunk(pa_half* out, const pa_half* q, const pa_half* k_cache,
                                           const pa_half* v_cache, const int32_t* block_tables,
                                           const int32_t* q_start, const int32_t* ctx_before, int32_t num_reqs,
                                           int32_t num_tokens, int32_t num_heads, int32_t head_dim,
                                           int32_t block_size, int32_t max_blocks, int32_t num_blocks, float scale,
                                           int32_t* err_flag, void* stream) {
    if (num_reqs < 0 || num_tokens < 0 || num_heads <= 0 || head_dim <= 0 || block_size <= 0 || max_blocks < 0 ||
        num_blocks < 0)
        return fail(PA_ERR_INVALID_ARG, "pa_paged_attention_prefill_chunk: bad sizes");
    if (!pagedkv::prefill_supported(num_heads, head_dim, block_size))
        return fail(PA_ERR_UNSUPPORTED, "pa_paged_attention_prefill_chunk: no kernel for num_heads=%d head_dim=%d block_size=%d",
                    num_heads, head_dim, block_size);
    if (!std::isfinite(scale) || !(scale > 0.f))
        return fail(PA_ERR_INVALID_ARG, "pa_paged_attention_prefill_chunk: scale must be finite and > 0");
    if (static_cast<int64_t>(max_blocks) * block_size > (1 << 30))
        return fail(PA_ERR_INVALID_ARG, "pa_paged_attention_prefill_chunk: max_blocks*block_size too large");
    if (num_reqs == 0 || num_tokens == 0) return PA_OK;
    if (num_blocks == 0 || max_blocks == 0)
        return fail(PA_ERR_INVALID_ARG, "pa_paged_attention_prefill_chunk: empty pool or table");
    if (!out || !q || !k_cache || !v_cache || !block_tables || !q_start || !ctx_before)
        return fail(PA_ERR_INVALID_ARG, "pa_paged_attention_prefill_chunk: NULL pointer");
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
        return fail(PA_ERR_INVALID_ARG, "pa_paged_attention_prefill_chunk: fp16 buffers must be 16-byte aligned");
    pagedkv::PrefillArgs a{out, q, k_cache, v_cache, block_tables, q_start, ctx_before, num_reqs, num_tokens,
                           num_heads, head_dim, block_size, max_blocks, num_blocks, scale, err_flag};
    const char* why = nullptr;
    cudaError_t e = pagedkv::launch_prefill(a, static_cast<cudaStream_t>(stream), &why);
    return cuda_status(e, "pa_paged_attention_prefill_chunk", why);
}

}  // extern "C"
