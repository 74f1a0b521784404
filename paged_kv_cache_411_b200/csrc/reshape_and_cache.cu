// reshape_and_cache: scatter the step's new K/V rows into the paged pool.
//
// The slots come from the block manager's append_token (page "LLM 推理引擎
// Continuous Batching 与 PagedAttention", §3.2) and name the rows the paged
// attention kernel reads (§3.3): slot = block * block_size + row.  With the
// pool laid out [num_blocks, block_size, num_heads, head_dim], one token's
// K (or V) row of num_heads * head_dim fp16 values is contiguous both in the
// source [num_tokens, num_heads, head_dim] and in the pool, so the scatter is
// one contiguous row copy per token and tensor: 16-byte vector loads and
// stores, fully coalesced, bit-exact.
//
// Roofline: HBM-bound, 2 (K, V) x 2 (read + write) x num_heads x head_dim x 2
// bytes per token.
#include "device_common.cuh"
#include "kernels.h"

namespace pagedkv {

// One CTA per token; the CTA copies the K row then the V row with uint4
// (16-byte) accesses.  row_vecs = num_heads * head_dim / 8.
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const uint4* __restrict__ k_new, const uint4* __restrict__ v_new, uint4* __restrict__ k_cache,
    uint4* __restrict__ v_cache, const int64_t* __restrict__ slot_mapping, int32_t row_vecs,
    int64_t num_slots, int32_t* err_flag) {
    const int64_t t = blockIdx.x;
    const int64_t slot = slot_mapping[t];
    if (slot < 0) return;                       // padding token
    if (slot >= num_slots) {                    // outside the pool: skip and report
        if (threadIdx.x == 0) flag_error(err_flag, PA_DEVCHK_SLOT);
        return;
    }
    const uint4* ks = k_new + t * row_vecs;
    const uint4* vs = v_new + t * row_vecs;
    uint4* kd = k_cache + slot * row_vecs;
    uint4* vd = v_cache + slot * row_vecs;
    for (int32_t i = threadIdx.x; i < row_vecs; i += blockDim.x) {
        uint4 a = __ldg(ks + i);
        uint4 b = __ldg(vs + i);
        kd[i] = a;
        vd[i] = b;
    }
}

cudaError_t launch_reshape_and_cache(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                                     const int64_t* slot_mapping, int32_t num_tokens, int32_t num_heads,
                                     int32_t head_dim, int32_t block_size, int32_t num_blocks,
                                     int32_t* err_flag, cudaStream_t stream) {
    if (num_tokens == 0) return cudaSuccess;
    const int32_t row_vecs = num_heads * head_dim / 8;
    const int threads = row_vecs >= 256 ? 256 : ((row_vecs + 31) / 32) * 32;
    reshape_and_cache_kernel<<<num_tokens, threads, 0, stream>>>(
        static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), static_cast<uint4*>(k_cache),
        static_cast<uint4*>(v_cache), slot_mapping, row_vecs,
        static_cast<int64_t>(num_blocks) * block_size, err_flag);
    return cudaGetLastError();
}

}  // namespace pagedkv
