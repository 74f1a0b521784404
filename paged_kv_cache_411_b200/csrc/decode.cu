// Paged-attention decode for sm_100a.
//
// Computes, for every sequence s and head h,
//     out[s, h] = sum_j softmax_j(scale * q[s, h] . K_j) V_j ,  j < seq_lens[s],
// where token j of sequence s lives in physical block block_tables[s][j / bs]
// at row j % bs of the pool [num_blocks, bs, H, D] -- the paged read of the
// page "LLM 推理引擎 Continuous Batching 与 PagedAttention" (§3.3, GPU Kernel
// 中的分页读取), completed with the weighted sum of V that the page's sketch
// leaves out, and the decode phase of §1.1 (one query per sequence; bound by
// reading the KV cache from HBM).
//
// Design (B200): the whole step is an HBM stream of K and V, ~1 flop per byte,
// so no tensor cores; what matters is keeping >= ~40 KB of loads in flight per
// SM, 100% sector efficiency and no tail imbalance on ragged batches.
//
//  1. plan kernel (1 CTA): splits every sequence into partitions of
//     `split` tokens (flash-decoding), choosing the largest split in
//     {512, 256, 128, 64} that still yields >= 8 work items per SM; an item is
//     (sequence, head group of HG heads, partition).  Full partitions are
//     listed first and the ragged tails last, so the dynamic scheduler hands
//     out the small items at the end.
//  2. main kernel (persistent, one CTA per SM, 16 consumer warps + 1
//     producer warp): the producer takes item b first (CTA b), then pulls
//     items from an atomic counter, reads
//     the item's block ids (one table entry per lane) and streams 16-token
//     stages of K and V with one 3-D TMA box each ([16 tokens][HG heads][D],
//     straight from the paged layout, no gather instructions) into a ring of
//     shared-memory stages guarded by mbarriers (K and V complete separately
//     so QK^T starts before V lands).  Consumer warps run the online softmax
//     in fp32: each lane holds 8 contiguous d of q, scores are reduced with a
//     transposing warp-shuffle reduction, and P.V accumulates in registers.
//     The warps sharing a head merge their (max, sum, acc) through shared
//     memory at the end of the item; single-partition sequences are written
//     straight to `out`, others write an fp32 partial.  The consumer warps
//     hand their (m, l, acc) to an epilogue warp through a double-buffered
//     shared-memory slot, so the head merge and the global stores never hold
//     up the stage ring.
//  3. combine kernel (one warp per (sequence, head) with several partitions):
//     m* = max m_i, l* = sum l_i 2^(m_i - m*), o* = sum acc_i 2^(m_i - m*) / l*;
//     up to 16 partitions are loaded in one round trip.
//  Each kernel is launched as a programmatic dependent of the one before: its
//  CTAs become resident (barriers, TMA descriptors) while the previous kernel
//  finishes, and wait for it with griddepcontrol before reading its output.
//
// The combine order is the partition order and the in-item merge order is
// fixed, so the result does not depend on physical block placement (bitwise)
// nor on which CTA ran which item.
#include <algorithm>
#include <type_traits>

#include "device_common.cuh"
#include "kernels.h"

namespace pagedkv {
namespace {

constexpr int kConsumerWarps = 16;
constexpr int kProducer = kConsumerWarps;          // warp index of the TMA producer
constexpr int kEpilogue = kConsumerWarps + 1;      // warp index of the epilogue
constexpr int kThreads = (kConsumerWarps + 2) * 32;
constexpr int kStageTok = 16;
constexpr int kMinSplit = 64;
constexpr int kSmemBudget = 192 * 1024;          // K + V stage ring
constexpr float kLog2e = 1.4426950408889634f;

// Stage-info flags (bits 8.. of info.w; bits 0..7 hold the valid token count).
constexpr int kFirst = 1 << 8;
constexpr int kLast = 1 << 9;
constexpr int kSingle = 1 << 10;
constexpr int kTerminate = 1 << 11;

// Item record: x = seq, y = first token, z = tokens | (head group << 10), w = partition | (partitions << 16).
struct WsLayout {
    size_t hdr, n_splits, items, part_ml, part_acc, total;
    int32_t max_splits;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WsLayout ws_layout(int32_t S, int32_t H, int32_t D, int32_t max_blocks, int32_t bs) {
    WsLayout w;
    const int64_t max_len = static_cast<int64_t>(max_blocks) * bs;
    w.max_splits = static_cast<int32_t>(std::max<int64_t>(1, (max_len + kMinSplit - 1) / kMinSplit));
    const size_t pairs = static_cast<size_t>(S) * w.max_splits;
    size_t off = 0;
    w.hdr = off;        off += 256;
    w.n_splits = off;   off = align256(off + sizeof(int32_t) * S);
    w.items = off;      off = align256(off + sizeof(int4) * pairs * H);
    w.part_ml = off;    off = align256(off + sizeof(float2) * pairs * H);
    w.part_acc = off;   off = align256(off + sizeof(float) * pairs * H * D);
    w.total = off;
    return w;
}

struct DecodeParams {
    __half* out;
    const int32_t* block_tables;
    const int32_t* seq_lens;
    int32_t S, H, max_blocks, bs, num_blocks, max_len;
    float qscale;                       // scale * log2(e): scores live in the log2 domain
    int32_t* hdr;                       // [0] item counter, [1] item count, [2] split tokens
    int32_t* n_splits;
    int4* items;
    float2* part_ml;
    float* part_acc;
    int32_t max_splits;
    int32_t* err_flag;
    uint64_t wait_ns;                   // limit of every pipeline wait (kWaitLimitNs by default)
    int32_t stall;                      // test hook: the consumers first wait on a barrier nothing completes
};

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <int D, int HG>
struct Cfg {
    static constexpr int kWPH = kConsumerWarps / HG;          // consumer warps per head
    static constexpr int kTPW = kStageTok / kWPH;              // tokens per warp per stage
    static constexpr int kLPT = D / 8;                         // lanes covering one token row (16 B each)
    static constexpr int kTPL = 32 / kLPT;                     // token rows per warp-wide load
    static constexpr int kNV = kTPW / kTPL;                    // loads (partial scores) per lane per stage
    static constexpr int kRep = kLPT / kNV;                    // lanes holding the same reduced score
    static constexpr int kTileBytes = kStageTok * HG * D * 2;  // one of K or V per stage
    static constexpr int kStagesRaw = kSmemBudget / (2 * kTileBytes);
    static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
    static constexpr int kQBytes = HG * D * 2;
    static constexpr int kHandStride = D + 4;                    // floats per warp: acc[D], m, l, pad
    static constexpr int kHandFloats = kConsumerWarps * kHandStride;   // one hand-off slot
    static constexpr size_t kOffK = 0;
    static constexpr size_t kOffV = kOffK + size_t(kStages) * kTileBytes;
    static constexpr size_t kOffQ = kOffV + size_t(kStages) * kTileBytes;
    static constexpr size_t kOffHand = kOffQ + size_t(kStages) * kQBytes;
    static constexpr size_t kOffInfo = kOffHand + size_t(2) * kHandFloats * 4;    // stage infos, then 2 hand-off infos
    static constexpr size_t kOffBar = (kOffInfo + size_t(kStages + 2) * 16 + 15) & ~size_t(15);
    static constexpr size_t kNumBars = 3 * kStages + 5;
    static constexpr size_t kOffAbort = kOffBar + kNumBars * 8;
    static constexpr size_t kSmemBytes = kOffAbort + 16 + 1024;   // + alignment slack
    static_assert(kWPH >= 1 && kTPW >= kTPL && kTPW % kTPL == 0, "bad warp split");
    static_assert(kNV >= 1 && kNV <= kLPT, "bad reduction shape");
    static_assert(kStages >= 2, "need at least double buffering");
};

__device__ __forceinline__ uint4 lds128(const void* p) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "r"(smem_u32(p)));
    return r;
}

__device__ __forceinline__ float dot8(const float* q, uint4 k) {
    float2 a = h2_to_f2(k.x), b = h2_to_f2(k.y), c = h2_to_f2(k.z), d = h2_to_f2(k.w);
    float s = q[0] * a.x;
    s = fmaf(q[1], a.y, s);
    s = fmaf(q[2], b.x, s);
    s = fmaf(q[3], b.y, s);
    s = fmaf(q[4], c.x, s);
    s = fmaf(q[5], c.y, s);
    s = fmaf(q[6], d.x, s);
    s = fmaf(q[7], d.y, s);
    return s;
}

__device__ __forceinline__ void axpy8(float* acc, float p, uint4 v) {
    float2 a = h2_to_f2(v.x), b = h2_to_f2(v.y), c = h2_to_f2(v.z), d = h2_to_f2(v.w);
    acc[0] = fmaf(p, a.x, acc[0]);
    acc[1] = fmaf(p, a.y, acc[1]);
    acc[2] = fmaf(p, b.x, acc[2]);
    acc[3] = fmaf(p, b.y, acc[3]);
    acc[4] = fmaf(p, c.x, acc[4]);
    acc[5] = fmaf(p, c.y, acc[5]);
    acc[6] = fmaf(p, d.x, acc[6]);
    acc[7] = fmaf(p, d.y, acc[7]);
}

// Transposing reduction: lane holds NV partial dot products (one per token it
// loaded) spread over LPT lanes; after log2(NV) halving exchanges and the
// remaining butterflies, every lane holds one complete score, for token index
// (lane % LPT) / (LPT / NV).
template <int NV, int LPT>
__device__ __forceinline__ float reduce_scores(float (&v)[NV], int lane) {
#pragma unroll
    for (int step = 0; (NV >> step) > 1; ++step) {
        const int n = NV >> step;
        const int off = LPT >> (step + 1);
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int k = 0; k < n / 2; ++k) {
            const float send = upper ? v[k] : v[k + n / 2];
            const float keep = upper ? v[k + n / 2] : v[k];
            v[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    float s = v[0];
#pragma unroll
    for (int off = LPT / (2 * NV); off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    return s;
}

// ------------------------------------------------------------------ plan ----
__global__ void __launch_bounds__(256) decode_plan_kernel(DecodeParams p, int32_t hg_count,
                                                           int32_t target_items, int32_t max_split,
                                                           int32_t head_dim) {
    constexpr int kNC = 4;
    const int cand[kNC] = {512, 256, 128, 64};
    __shared__ long long red[kNC][32];
    __shared__ int32_t s_split;
    __shared__ long long s_scan[2][32];
    __shared__ long long s_tot[2];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    pdl_wait();                       // inputs may come from the kernel before us on the stream
    pdl_launch_dependents();          // let the streaming kernel's CTAs set up meanwhile

    long long cnt[kNC] = {0, 0, 0, 0};
    for (int s = tid; s < p.S; s += blockDim.x) {
        int len = p.seq_lens[s];
        if (len < 0 || len > p.max_len) {
            flag_error(p.err_flag, PA_DEVCHK_SEQ_LEN);
            len = len < 0 ? 0 : p.max_len;
        }
#pragma unroll
        for (int c = 0; c < kNC; ++c) cnt[c] += (len + cand[c] - 1) / cand[c];
    }
#pragma unroll
    for (int c = 0; c < kNC; ++c) {
        long long v = cnt[c];
        for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[c][warp] = v;
    }
    __syncthreads();
    if (tid == 0) {
        int split = kMinSplit;
        for (int c = 0; c < kNC; ++c) {
            long long tot = 0;
            for (int w = 0; w < nwarps; ++w) tot += red[c][w];
            if (cand[c] <= max_split && tot * hg_count >= target_items) {
                split = cand[c];
                break;
            }
        }
        s_split = split;
    }
    __syncthreads();
    const int split = s_split;

    // Contiguous chunk of sequences per thread; exclusive scans of full and tail partitions.
    const int chunk = (p.S + blockDim.x - 1) / blockDim.x;
    const int s0 = min(p.S, tid * chunk), s1 = min(p.S, s0 + chunk);
    long long my_full = 0, my_part = 0;
    for (int s = s0; s < s1; ++s) {
        int len = min(max(p.seq_lens[s], 0), p.max_len);
        my_full += len / split;
        my_part += (len % split) != 0;
    }
    long long inc_f = my_full, inc_p = my_part;
    for (int o = 1; o < 32; o <<= 1) {
        long long a = __shfl_up_sync(0xffffffffu, inc_f, o), b = __shfl_up_sync(0xffffffffu, inc_p, o);
        if (lane >= o) { inc_f += a; inc_p += b; }
    }
    if (lane == 31) { s_scan[0][warp] = inc_f; s_scan[1][warp] = inc_p; }
    __syncthreads();
    if (tid == 0) {
        long long af = 0, ap = 0;
        for (int w = 0; w < nwarps; ++w) {
            long long f = s_scan[0][w], q = s_scan[1][w];
            s_scan[0][w] = af; s_scan[1][w] = ap;
            af += f; ap += q;
        }
        s_tot[0] = af; s_tot[1] = ap;
    }
    __syncthreads();
    long long off_f = s_scan[0][warp] + inc_f - my_full;
    long long off_p = s_tot[0] + s_scan[1][warp] + inc_p - my_part;
    for (int s = s0; s < s1; ++s) {
        int len = min(max(p.seq_lens[s], 0), p.max_len);
        const int nfull = len / split, tail = len % split;
        const int nsp = nfull + (tail != 0);
        p.n_splits[s] = nsp;
        for (int k = 0; k < nfull; ++k, ++off_f)
            for (int g = 0; g < hg_count; ++g)
                p.items[off_f * hg_count + g] = make_int4(s, k * split, split | (g << 10), k | (nsp << 16));
        if (tail) {
            for (int g = 0; g < hg_count; ++g)
                p.items[off_p * hg_count + g] = make_int4(s, nfull * split, tail | (g << 10), nfull | (nsp << 16));
            ++off_p;
        }
        if (nsp == 0) {                 // empty sequence: zeros
            uint4* o = reinterpret_cast<uint4*>(p.out + static_cast<int64_t>(s) * p.H * head_dim);
            for (int i = 0; i < p.H * head_dim / 8; ++i) o[i] = make_uint4(0, 0, 0, 0);
        }
    }
    if (tid == 0) {
        p.hdr[0] = 0;
        p.hdr[1] = static_cast<int32_t>((s_tot[0] + s_tot[1]) * hg_count);
        p.hdr[2] = split;
    }
}

// ---------------------------------------------------------------- combine ----
// One warp per (sequence, head) of a multi-partition sequence: merge its fp32 partials with the
// log-sum-exp rule, in partition order, and write the fp16 output.  Launched as a programmatic
// dependent of the streaming kernel; waits for it before reading anything.
template <int D>
__global__ void __launch_bounds__(256) decode_combine_kernel(DecodeParams p) {
    pdl_wait();
    constexpr int VEC = D / 32;
    constexpr int kBatch = 8;                   // partitions whose loads are in flight together
    constexpr int kOneTrip = 16;                // up to this many partitions: all loads in one round trip
    using Vec = typename std::conditional<VEC == 4, float4, float2>::type;
    const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (gw >= p.S * p.H) return;
    const int s = gw / p.H, h = gw % p.H;
    const int n = p.n_splits[s];
    if (n <= 1) return;
    const int64_t base = static_cast<int64_t>(s) * p.max_splits * p.H + h;
    float M = -INFINITY, L = 0.f, acc[VEC];
#pragma unroll
    for (int k = 0; k < VEC; ++k) acc[k] = 0.f;
    if (n <= kOneTrip) {
        // every load at once (one L2 round trip), then the max and the merge in partition order
        float2 ml[kOneTrip];
        Vec a[kOneTrip];
#pragma unroll
        for (int b = 0; b < kOneTrip; ++b) {
            const int64_t pi = base + static_cast<int64_t>(min(b, n - 1)) * p.H;
            ml[b] = p.part_ml[pi];
            a[b] = *reinterpret_cast<const Vec*>(p.part_acc + pi * D + lane * VEC);
        }
#pragma unroll
        for (int b = 0; b < kOneTrip; ++b)
            if (b < n) M = fmaxf(M, ml[b].x);
#pragma unroll
        for (int b = 0; b < kOneTrip; ++b) {
            if (b >= n) break;
            const float w = exp2f(ml[b].x - M);
            L = fmaf(ml[b].y, w, L);
            const float* av = reinterpret_cast<const float*>(&a[b]);
#pragma unroll
            for (int k = 0; k < VEC; ++k) acc[k] = fmaf(av[k], w, acc[k]);
        }
    } else {
        for (int i = lane; i < n; i += 32) M = fmaxf(M, p.part_ml[base + static_cast<int64_t>(i) * p.H].x);
        for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        for (int i0 = 0; i0 < n; i0 += kBatch) {
            // every load of the batch first, then the merge in partition order
            float2 ml[kBatch];
            Vec a[kBatch];
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
                const int64_t pi = base + static_cast<int64_t>(min(i0 + b, n - 1)) * p.H;
                ml[b] = p.part_ml[pi];
                a[b] = *reinterpret_cast<const Vec*>(p.part_acc + pi * D + lane * VEC);
            }
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
                if (i0 + b >= n) break;
                const float w = exp2f(ml[b].x - M);
                L = fmaf(ml[b].y, w, L);
                const float* av = reinterpret_cast<const float*>(&a[b]);
#pragma unroll
                for (int k = 0; k < VEC; ++k) acc[k] = fmaf(av[k], w, acc[k]);
            }
        }
    }
    const float r = 1.f / L;
    __half* o = p.out + static_cast<int64_t>(gw) * D + lane * VEC;
#pragma unroll
    for (int k = 0; k < VEC; k += 2) *reinterpret_cast<uint32_t*>(o + k) = f2_to_h2(acc[k] * r, acc[k + 1] * r);
}

// ------------------------------------------------------------------ main ----
template <int D, int HG>
__global__ void __launch_bounds__(kThreads, 1)
decode_main_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_q, DecodeParams p) {
    using C = Cfg<D, HG>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* tile_k = smem + C::kOffK;
    uint8_t* tile_v = smem + C::kOffV;
    uint8_t* qbuf = smem + C::kOffQ;
    float* hand = reinterpret_cast<float*>(smem + C::kOffHand);
    int4* info = reinterpret_cast<int4*>(smem + C::kOffInfo);
    uint64_t* full_k = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* full_v = full_k + C::kStages;
    uint64_t* empty = full_v + C::kStages;
    int4* hand_info = info + C::kStages;
    uint64_t* hand_full = empty + C::kStages;     // [2] every consumer warp has handed its state over
    uint64_t* hand_empty = hand_full + 2;         // [2] the epilogue has read the slot
    uint64_t* never = hand_empty + 2;             // no thread ever arrives on it (failure-detection test)
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffAbort);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full_k[s], 1);
            mbar_init(&full_v[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&hand_full[i], kConsumerWarps);
            mbar_init(&hand_empty[i], 1);
        }
        mbar_init(never, 1);
        *abort_flag = 0;
        mbar_init_fence();
    }
    __syncthreads();
    pdl_wait();                       // the plan (and everything before it) has completed
    pdl_launch_dependents();          // the combine grid may be scheduled as our CTAs retire

    const int n_items = p.hdr[1];

    if (warp == kProducer) {
        // ================================================= producer warp
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_q);
        }
        const uint64_t pol_stream = l2_policy_evict_first();
        const uint64_t pol_keep = l2_policy_evict_last();
        const int bs = p.bs;
        const int box_tok = bs >= kStageTok ? kStageTok : bs;         // 16, or 8 for bs == 8
        const uint32_t box_bytes = box_tok * HG * D * 2;
        uint32_t stage = 0, phase = 0;
        uint32_t issued_mask = 0, issued_par = 0;     // per slot: ever issued / parity of its last issue
        bool ok = true;

        // CTA b starts with item b (no counter round trip before its first copies); the counter hands out
        // the items from gridDim.x on
        const int idx = static_cast<int>(blockIdx.x);
        int4 rec = idx < n_items ? p.items[idx] : make_int4(-1, 0, 0, 0);
        while (rec.x >= 0 && ok) {
            const int seq = rec.x, tok0 = rec.y, ntok_item = rec.z & 1023, hg = rec.z >> 10;
            const int part = rec.w & 0xffff, nsp = rec.w >> 16;
            const int single = nsp == 1;
            int nidx = 0;
            if (lane == 0) nidx = atomicAdd(&p.hdr[0], 1) + static_cast<int>(gridDim.x);   // next item, in flight
            const int blk0 = tok0 / bs;
            const int nblk = (tok0 + ntok_item - 1) / bs - blk0 + 1;
            int bid = 0;
            if (lane < nblk) {
                bid = p.block_tables[static_cast<int64_t>(seq) * p.max_blocks + blk0 + lane];
                if (bid < 0 || bid >= p.num_blocks) {
                    flag_error(p.err_flag, PA_DEVCHK_BLOCK_ID);
                    bid = 0;
                }
            }
            const int nst = (ntok_item + kStageTok - 1) / kStageTok;
            for (int st = 0; st < nst; ++st) {
                const int tok = tok0 + st * kStageTok;
                const int ntok = min(kStageTok, tok0 + ntok_item - tok);
                const int b_first = __shfl_sync(0xffffffffu, bid, tok / bs - blk0);
                const int b_second = __shfl_sync(0xffffffffu, bid, min(tok / bs - blk0 + 1, 31));
                if (!mbar_wait(&empty[stage], phase ^ 1, p.wait_ns)) { ok = false; break; }
                if (*abort_flag) { ok = false; break; }
                if (lane == 0) {
                    int flags = ntok;
                    if (st == 0) flags |= kFirst;
                    if (st == nst - 1) flags |= kLast | (single ? kSingle : 0);
                    info[stage] = make_int4(seq, part | (nsp << 16), hg, flags);
                    const int nbox = (bs >= kStageTok) ? 1 : (ntok + box_tok - 1) / box_tok;
                    const uint32_t kv_bytes = nbox * box_bytes;
                    uint8_t* dk = tile_k + size_t(stage) * C::kTileBytes;
                    uint8_t* dv = tile_v + size_t(stage) * C::kTileBytes;
                    mbar_arrive_expect_tx(&full_k[stage], kv_bytes + (st == 0 ? C::kQBytes : 0));
                    if (st == 0)
                        tma_load_3d(qbuf + size_t(stage) * C::kQBytes, &tm_q, &full_k[stage], 0, hg * HG, seq, pol_keep);
                    const int row0 = (bs >= kStageTok) ? b_first * bs + (tok % bs) : b_first * bs;
                    tma_load_3d(dk, &tm_k, &full_k[stage], 0, hg * HG, row0, pol_stream);
                    if (nbox > 1) tma_load_3d(dk + box_bytes, &tm_k, &full_k[stage], 0, hg * HG, b_second * bs, pol_stream);
                    mbar_arrive_expect_tx(&full_v[stage], kv_bytes);
                    tma_load_3d(dv, &tm_v, &full_v[stage], 0, hg * HG, row0, pol_stream);
                    if (nbox > 1) tma_load_3d(dv + box_bytes, &tm_v, &full_v[stage], 0, hg * HG, b_second * bs, pol_stream);
                }
                __syncwarp();
                issued_mask |= 1u << stage;
                issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                if (++stage == C::kStages) { stage = 0; phase ^= 1; }
            }
            nidx = __shfl_sync(0xffffffffu, nidx, 0);
            rec = nidx < n_items ? p.items[nidx] : make_int4(-1, 0, 0, 0);
        }
        if (ok) ok = mbar_wait(&empty[stage], phase ^ 1, p.wait_ns);
        if (!ok) {
            // Unwind: report, stop the consumers, and let every copy this warp
            // issued land before the CTA can exit (each wait again bounded).
            flag_error(p.err_flag, kDevchkTimeout);
            *abort_flag = 1;
            for (int s = 0; s < C::kStages; ++s) {
                if (!((issued_mask >> s) & 1u)) continue;
                (void)mbar_wait(&full_k[s], (issued_par >> s) & 1u);
                (void)mbar_wait(&full_v[s], (issued_par >> s) & 1u);
            }
        }
        // In the normal path the consumers reach this stage only after every
        // earlier stage's copies completed, so nothing is left in flight.
        if (lane == 0) {
            info[stage] = make_int4(0, 0, 0, kTerminate);
            mbar_arrive(&full_k[stage]);
            mbar_arrive(&full_v[stage]);
        }
        return;
    }

    if (warp == kEpilogue) {
        // ================================================= epilogue warp
        // Per finished item: merge the warps of each head, then write the output (single-partition
        // sequences) or the fp32 partial that the combine kernel merges.  Off the streaming path.
        constexpr int VEC = D / 32;
        uint32_t uses = 0;
        while (true) {
            const int hs = uses & 1;
            if (!mbar_wait(&hand_full[hs], (uses >> 1) & 1, p.wait_ns)) {
                flag_error(p.err_flag, kDevchkTimeout);
                *abort_flag = 1;
                break;
            }
            const int4 inf = hand_info[hs];
            if (inf.w & kTerminate) break;
            const int seq = inf.x, part = inf.y & 0xffff, nsp = inf.y >> 16, hg = inf.z;
            const float* hb = hand + hs * C::kHandFloats;
            float accs[HG][VEC];
            float Ms[HG], Ls[HG];
#pragma unroll
            for (int hh = 0; hh < HG; ++hh) {
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < C::kWPH; ++w) M = fmaxf(M, hb[(hh * C::kWPH + w) * C::kHandStride + D]);
                const float Mu = M == -INFINITY ? 0.f : M;
                float L = 0.f;
#pragma unroll
                for (int k = 0; k < VEC; ++k) accs[hh][k] = 0.f;
#pragma unroll
                for (int w = 0; w < C::kWPH; ++w) {
                    const float* ws_ = hb + (hh * C::kWPH + w) * C::kHandStride;
                    const float wt = exp2f(ws_[D] - Mu);
                    L = fmaf(ws_[D + 1], wt, L);
#pragma unroll
                    for (int k = 0; k < VEC; ++k) accs[hh][k] = fmaf(ws_[lane * VEC + k], wt, accs[hh][k]);
                }
                Ms[hh] = M;
                Ls[hh] = L;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&hand_empty[hs]);
            ++uses;
            if (nsp == 1) {
#pragma unroll
                for (int hh = 0; hh < HG; ++hh) {
                    const float r = 1.f / Ls[hh];
                    __half* o = p.out + (static_cast<int64_t>(seq) * p.H + hg * HG + hh) * D + lane * VEC;
#pragma unroll
                    for (int k = 0; k < VEC; k += 2) *reinterpret_cast<uint32_t*>(o + k) = f2_to_h2(accs[hh][k] * r, accs[hh][k + 1] * r);
                }
                continue;
            }
#pragma unroll
            for (int hh = 0; hh < HG; ++hh) {
                const int64_t pi = (static_cast<int64_t>(seq) * p.max_splits + part) * p.H + hg * HG + hh;
                float* dst = p.part_acc + pi * D + lane * VEC;
#pragma unroll
                for (int k = 0; k < VEC; ++k) dst[k] = accs[hh][k];
                if (lane == 0) p.part_ml[pi] = make_float2(Ms[hh], Ls[hh]);
            }
        }
        return;
    }

    // ===================================================== consumer warps
    if (p.stall && !mbar_wait(never, 0, p.wait_ns)) {
        // failure-detection test: the wait ran out; report it and stop the other roles, whose own
        // waits then run out too and unwind (the producer lets its copies land before exiting)
        flag_error(p.err_flag, kDevchkTimeout);
        *abort_flag = 1;
        return;
    }
    const int hh = warp / C::kWPH;        // head within the group
    const int ww = warp % C::kWPH;        // slice of the stage's tokens
    const int tq = lane / C::kLPT;        // token row within one warp-wide load
    const int sub = lane % C::kLPT;       // 16-byte chunk of the head dimension
    const int my_tok0 = ww * C::kTPW;
    const int score_tok = my_tok0 + (sub / C::kRep) * C::kTPL + tq;

    float qf[8];
    float acc[8];
    float m_run = -INFINITY, l_lane = 0.f;
    uint32_t stage = 0, phase = 0, hand_uses = 0;
    while (true) {
        if (!mbar_wait(&full_k[stage], phase, p.wait_ns)) { flag_error(p.err_flag, kDevchkTimeout); *abort_flag = 1; break; }
        const int4 inf = info[stage];
        const int flags = inf.w;
        if (flags & kTerminate) {
            // tell the epilogue warp there is nothing more to merge
            const int hs = hand_uses & 1;
            if (mbar_wait(&hand_empty[hs], ((hand_uses >> 1) & 1) ^ 1, p.wait_ns)) {
                if (warp == 0 && lane == 0) hand_info[hs] = make_int4(0, 0, 0, kTerminate);
                __syncwarp();
                if (lane == 0) mbar_arrive(&hand_full[hs]);
            }
            break;
        }
        const int ntok = flags & 0xff;
        const uint8_t* tk = tile_k + size_t(stage) * C::kTileBytes;
        const uint8_t* tv = tile_v + size_t(stage) * C::kTileBytes;
        if (flags & kFirst) {
            const uint4 qv = lds128(qbuf + size_t(stage) * C::kQBytes + (hh * D + sub * 8) * 2);
            const float2 a = h2_to_f2(qv.x), b = h2_to_f2(qv.y), c = h2_to_f2(qv.z), d = h2_to_f2(qv.w);
            qf[0] = a.x * p.qscale; qf[1] = a.y * p.qscale; qf[2] = b.x * p.qscale; qf[3] = b.y * p.qscale;
            qf[4] = c.x * p.qscale; qf[5] = c.y * p.qscale; qf[6] = d.x * p.qscale; qf[7] = d.y * p.qscale;
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[k] = 0.f;
            m_run = -INFINITY;
            l_lane = 0.f;
        }
        // ---- scores of this warp's tokens
        float sv[C::kNV];
#pragma unroll
        for (int i = 0; i < C::kNV; ++i) {
            const int t = my_tok0 + i * C::kTPL + tq;
            const uint4 kv = lds128(tk + ((t * HG + hh) * D + sub * 8) * 2);
            sv[i] = dot8(qf, kv);
        }
        float s = reduce_scores<C::kNV, C::kLPT>(sv, lane);
        s = score_tok < ntok ? s : -INFINITY;
        float m_blk = s;
#pragma unroll
        for (int off = C::kRep; off < 32; off <<= 1) m_blk = fmaxf(m_blk, __shfl_xor_sync(0xffffffffu, m_blk, off));
        const float m_new = fmaxf(m_run, m_blk);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        const float alpha = exp2f(m_run - m_use);
        const float pr = exp2f(s - m_use);
        l_lane = fmaf(l_lane, alpha, pr);
        m_run = m_new;
        // ---- P.V
        if (!mbar_wait(&full_v[stage], phase, p.wait_ns)) { flag_error(p.err_flag, kDevchkTimeout); *abort_flag = 1; break; }
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] *= alpha;
#pragma unroll
        for (int i = 0; i < C::kNV; ++i) {
            const float pi = __shfl_sync(0xffffffffu, pr, tq * C::kLPT + i * C::kRep);
            const int t = my_tok0 + i * C::kTPL + tq;
            if (t < ntok) {
                const uint4 vv = lds128(tv + ((t * HG + hh) * D + sub * 8) * 2);
                axpy8(acc, pi, vv);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);

        if (flags & kLast) {
            // ---- finish the item: fold the token rows and hand (m, l, acc) to the epilogue warp.
            float a8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                float v = acc[k];
#pragma unroll
                for (int off = C::kLPT; off < 32; off <<= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                a8[k] = v;
            }
            float l = l_lane;
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
            l *= 1.0f / C::kRep;
            const int hs = hand_uses & 1;
            if (!mbar_wait(&hand_empty[hs], ((hand_uses >> 1) & 1) ^ 1, p.wait_ns)) { flag_error(p.err_flag, kDevchkTimeout); *abort_flag = 1; break; }
            float* slot = hand + hs * C::kHandFloats + warp * C::kHandStride;
            if (tq == 0) {
                *reinterpret_cast<float4*>(slot + sub * 8) = make_float4(a8[0], a8[1], a8[2], a8[3]);
                *reinterpret_cast<float4*>(slot + sub * 8 + 4) = make_float4(a8[4], a8[5], a8[6], a8[7]);
            }
            if (lane == 0) {
                slot[D] = m_run;
                slot[D + 1] = l;
                if (warp == 0) hand_info[hs] = inf;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&hand_full[hs]);
            ++hand_uses;
        }
        if (*abort_flag) break;
        if (++stage == C::kStages) { stage = 0; phase ^= 1; }
    }
}

template <int D, int HG>
cudaError_t run_main(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq, const DecodeParams& p,
                     int grid, cudaStream_t stream) {
    using C = Cfg<D, HG>;
    static std::atomic<uint64_t> smem_set{0};          // devices whose limit is raised
    const cudaError_t attr_err = ensure_dynamic_smem(reinterpret_cast<const void*>(decode_main_kernel<D, HG>),
                                                     static_cast<int>(C::kSmemBytes), &smem_set);
    if (attr_err != cudaSuccess) return attr_err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_main_kernel<D, HG>, tk, tv, tq, p);
}

}  // namespace

int32_t decode_head_group(int32_t H, int32_t D) {
    if (D != 64 && D != 128) return 0;
    if (H % 8 == 0) return 8;
    if (H % 4 == 0) return 4;
    if (H % 2 == 0 && D == 128) return 2;
    return 0;
}

bool decode_block_size_ok(int32_t bs) { return bs == 8 || (bs >= 16 && bs % 16 == 0 && bs <= 4096); }

size_t decode_workspace_bytes(int32_t S, int32_t H, int32_t D, int32_t max_blocks, int32_t bs) {
    if (S < 0 || H <= 0 || D <= 0 || max_blocks < 0 || bs <= 0) return 0;
    return ws_layout(S, H, D, max_blocks, bs).total;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream, const char** why) {
    const int HG = decode_head_group(a.num_heads, a.head_dim);
    const WsLayout w = ws_layout(a.num_seqs, a.num_heads, a.head_dim, a.max_blocks, a.block_size);
    uint8_t* ws = static_cast<uint8_t*>(a.workspace);
    DecodeParams p;
    p.out = static_cast<__half*>(a.out);
    p.block_tables = a.block_tables;
    p.seq_lens = a.seq_lens;
    p.S = a.num_seqs;
    p.H = a.num_heads;
    p.max_blocks = a.max_blocks;
    p.bs = a.block_size;
    p.num_blocks = a.num_blocks;
    p.max_len = a.max_blocks * a.block_size;
    p.qscale = a.scale * kLog2e;
    p.hdr = reinterpret_cast<int32_t*>(ws + w.hdr);
    p.n_splits = reinterpret_cast<int32_t*>(ws + w.n_splits);
    p.items = reinterpret_cast<int4*>(ws + w.items);
    p.part_ml = reinterpret_cast<float2*>(ws + w.part_ml);
    p.part_acc = reinterpret_cast<float*>(ws + w.part_acc);
    p.max_splits = w.max_splits;
    p.err_flag = a.err_flag;
    const uint64_t stall_ns = take_injected_stall(kStallDecode);
    p.wait_ns = stall_ns ? stall_ns : kWaitLimitNs;
    p.stall = stall_ns != 0;
    if (a.num_seqs == 0) return cudaSuccess;

    const int box_tok = a.block_size >= kStageTok ? kStageTok : a.block_size;
    const uint64_t rows = static_cast<uint64_t>(a.num_blocks) * a.block_size;
    const uint64_t s1 = static_cast<uint64_t>(a.head_dim) * 2, s2 = s1 * a.num_heads;
    alignas(64) CUtensorMap tk, tv, tq;
    if (!encode_tensor_map_3d(&tk, a.k_cache, a.head_dim, a.num_heads, rows, s1, s2, a.head_dim, HG, box_tok, 0, why) ||
        !encode_tensor_map_3d(&tv, a.v_cache, a.head_dim, a.num_heads, rows, s1, s2, a.head_dim, HG, box_tok, 0, why) ||
        !encode_tensor_map_3d(&tq, a.q, a.head_dim, a.num_heads, a.num_seqs, s1, s2, a.head_dim, HG, 1, 0, why))
        return cudaErrorInvalidValue;

    const int sms = device_sm_count();
    const int max_split = a.block_size >= 16 ? 512 : 32 * a.block_size;
    cudaError_t e;
    {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(1);
        cfg.blockDim = dim3(256);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, decode_plan_kernel, p, a.num_heads / HG, 8 * sms, max_split, a.head_dim);
        if (e != cudaSuccess) return e;
    }
    if (a.head_dim == 128) {
        if (HG == 8) e = run_main<128, 8>(tk, tv, tq, p, sms, stream);
        else if (HG == 4) e = run_main<128, 4>(tk, tv, tq, p, sms, stream);
        else e = run_main<128, 2>(tk, tv, tq, p, sms, stream);
    } else {
        if (HG == 8) e = run_main<64, 8>(tk, tv, tq, p, sms, stream);
        else e = run_main<64, 4>(tk, tv, tq, p, sms, stream);
    }
    if (e != cudaSuccess) return e;
    {
        const int warps = a.num_seqs * a.num_heads;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((warps + 7) / 8);
        cfg.blockDim = dim3(256);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (a.head_dim == 128) e = cudaLaunchKernelEx(&cfg, decode_combine_kernel<128>, p);
        else e = cudaLaunchKernelEx(&cfg, decode_combine_kernel<64>, p);
    }
    return e;
}

}  // namespace pagedkv
