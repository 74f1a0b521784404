// Swapping KV blocks between the GPU pool and a host pool.
//
// The page "LLM 推理引擎 Continuous Batching 与 PagedAttention" (§4.4 Swap：
// CPU offload) keeps one block manager per pool and moves a request by
// allocating it in the destination pool, copying its blocks and freeing it in
// the source pool; §5.4 uses this as the alternative to recomputation when a
// request is preempted.  Here:
//   * pa_swap_blocks copies listed (source block, destination block) pairs of
//     the K and V pools; runs of consecutive pairs are merged into one
//     cudaMemcpyAsync each (cudaMemcpyDefault: device or pinned host memory on
//     either side), issued in list order on the caller's stream;
//   * pa_alloc_swap_out / pa_alloc_swap_in do the bookkeeping of §4.4 with two
//     allocators and call pa_swap_blocks.  The source's blocks are released
//     on the host at once: reuse them only from work ordered after the copy on
//     the same stream.
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "common.h"

using pagedkv::fail;

namespace {

cudaError_t copy_runs(const uint8_t* src, uint8_t* dst, const int64_t* mapping, int32_t n, int64_t block_bytes,
                      cudaStream_t stream) {
    int32_t i = 0;
    while (i < n) {
        int32_t j = i + 1;
        while (j < n && mapping[2 * j] == mapping[2 * (j - 1)] + 1 && mapping[2 * j + 1] == mapping[2 * (j - 1) + 1] + 1)
            ++j;
        cudaError_t e = cudaMemcpyAsync(dst + mapping[2 * i + 1] * block_bytes, src + mapping[2 * i] * block_bytes,
                                        static_cast<size_t>(j - i) * block_bytes, cudaMemcpyDefault, stream);
        if (e != cudaSuccess) return e;
        i = j;
    }
    return cudaSuccess;
}

}  // namespace

extern "C" {

pa_status pa_swap_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v, const int64_t* mapping,
                         int32_t num_pairs, int64_t block_bytes, int32_t src_num_blocks, int32_t dst_num_blocks,
                         void* stream) {
    if (num_pairs < 0 || block_bytes < 0 || src_num_blocks < 0 || dst_num_blocks < 0)
        return fail(PA_ERR_INVALID_ARG, "pa_swap_blocks: bad sizes");
    if (num_pairs == 0 || block_bytes == 0) return PA_OK;
    if (!src_k || !src_v || !dst_k || !dst_v || !mapping) return fail(PA_ERR_INVALID_ARG, "pa_swap_blocks: NULL pointer");
    for (int32_t i = 0; i < num_pairs; ++i) {
        if (mapping[2 * i] < 0 || mapping[2 * i] >= src_num_blocks || mapping[2 * i + 1] < 0 ||
            mapping[2 * i + 1] >= dst_num_blocks)
            return fail(PA_ERR_INVALID_ARG, "pa_swap_blocks: pair %d (%lld -> %lld) outside the pools", i,
                        (long long)mapping[2 * i], (long long)mapping[2 * i + 1]);
    }
    auto s = static_cast<cudaStream_t>(stream);
    cudaError_t e = copy_runs(static_cast<const uint8_t*>(src_k), static_cast<uint8_t*>(dst_k), mapping, num_pairs,
                              block_bytes, s);
    if (e == cudaSuccess)
        e = copy_runs(static_cast<const uint8_t*>(src_v), static_cast<uint8_t*>(dst_v), mapping, num_pairs,
                      block_bytes, s);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "pa_swap_blocks: %s", cudaGetErrorString(e));
    return PA_OK;
}

// Moves `req` from allocator `from` to allocator `to`, copying its blocks from (fk, fv) to (tk, tv).
static pa_status move_request(pa_alloc* from, pa_alloc* to, int64_t req, const void* fk, const void* fv, void* tk,
                              void* tv, int64_t block_bytes, void* stream, const char* who) {
    if (!from || !to) return fail(PA_ERR_INVALID_ARG, "%s: NULL allocator", who);
    pa_alloc_stats_t sf, st;
    pa_alloc_stats(from, &sf);
    pa_alloc_stats(to, &st);
    if (sf.block_size != st.block_size) return fail(PA_ERR_INVALID_ARG, "%s: pools differ in block size", who);
    int32_t len = 0;
    if (pa_alloc_seq_len(from, req, &len) != PA_OK) return fail(PA_ERR_NOT_FOUND, "%s: request %lld not found", who, (long long)req);
    int32_t dummy = 0;
    if (pa_alloc_seq_len(to, req, &dummy) == PA_OK) return fail(PA_ERR_EXISTS, "%s: request %lld already in the destination", who, (long long)req);
    int32_t nsrc = 0;
    pa_alloc_get_block_table(from, req, nullptr, 0, &nsrc);
    std::vector<int32_t> src(nsrc);
    if (nsrc) pa_alloc_get_block_table(from, req, src.data(), nsrc, &nsrc);
    pa_status s = pa_alloc_allocate(to, req, len);
    if (s != PA_OK) return s;                                  // OOM: nothing changed
    std::vector<int32_t> dst(nsrc);
    int32_t ndst = 0;
    if (nsrc) pa_alloc_get_block_table(to, req, dst.data(), nsrc, &ndst);
    std::vector<int64_t> mapping(2 * static_cast<size_t>(nsrc));
    for (int32_t i = 0; i < nsrc; ++i) {
        mapping[2 * i] = src[i];
        mapping[2 * i + 1] = dst[i];
    }
    s = pa_swap_blocks(fk, fv, tk, tv, mapping.data(), nsrc, block_bytes, sf.num_blocks, st.num_blocks, stream);
    if (s != PA_OK) {
        pa_alloc_free(to, req);                                // roll the destination back
        return s;
    }
    return pa_alloc_free(from, req);
}

pa_status pa_alloc_swap_out(pa_alloc* gpu, pa_alloc* cpu, int64_t req, const void* gpu_k, const void* gpu_v,
                            void* cpu_k, void* cpu_v, int64_t block_bytes, void* stream) {
    return move_request(gpu, cpu, req, gpu_k, gpu_v, cpu_k, cpu_v, block_bytes, stream, "pa_alloc_swap_out");
}

pa_status pa_alloc_swap_in(pa_alloc* gpu, pa_alloc* cpu, int64_t req, void* gpu_k, void* gpu_v, const void* cpu_k,
                           const void* cpu_v, int64_t block_bytes, void* stream) {
    return move_request(cpu, gpu, req, cpu_k, cpu_v, gpu_k, gpu_v, block_bytes, stream, "pa_alloc_swap_in");
}

}  // extern "C"
