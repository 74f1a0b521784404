// Chunked-prefill attention over the paged KV cache, on the sm_100a tensor cores.
//
// Request b owns query rows q_start[b] .. q_start[b+1]-1; its row i sits at
// absolute position ctx_before[b] + i and attends causally to positions
// 0 .. ctx_before[b] + i of its sequence, read through its block table -- the
// chunked prefill of the page "LLM 推理引擎 Continuous Batching 与
// PagedAttention" (§4.3: a long prompt is split into chunks that run between
// decode steps; §1.1: prefill is the compute-bound phase) over the paged read
// of §3.3.  The chunk's own K/V must already be in the pool.
//
// One CTA computes one tile of 128 query rows x one head (FlashAttention
// order, online softmax over 128-key tiles):
//   * warps 8 and 10 (producers) load the Q tile once and stream the K and the
//     V tiles into two-stage rings with TMA: a tile of 128 keys is gathered from
//     the paged pool with one 3-D box per (physical block, 64-dim chunk) ([box
//     rows][1 head][64 dims], 128-byte swizzle), landing directly in the
//     canonical UMMA layout; each lane issues one box, so a tile is one TMA
//     instruction, and the next tile's block ids are read a tile ahead;
//   * warp 9 (one elected thread) issues tcgen05.mma: S = Q K^T (A and B
//     K-major) into a double-buffered fp32 TMEM tile, and O_j = P_j V_j (B
//     MN-major straight from the V tile) into a second double-buffered TMEM
//     tile; completions are signalled with tcgen05.commit on mbarriers;
//   * warps 0-7 (two threads per query row = per TMEM lane, each owning half
//     of the columns) read S with tcgen05.ld, apply the causal mask on the
//     diagonal tiles, agree on the row max through shared memory, run the
//     online softmax in fp32 (exp2 of prescaled logits), write P as fp16 into
//     shared memory in the swizzled K-major layout the next MMA reads, and
//     fold O_j into a register accumulator with the running rescale one tile
//     behind, so the MMA of tile j+1 overlaps the softmax of tile j.
// Keys past the tile's last query position are masked; rows of V past the
// sequence end are zeroed before P.V so stale or poisoned pool rows never
// reach the MMA.  Every wait is bounded; on a timeout the CTA records
// PA_DEVCHK_TIMEOUT, lets its copies and MMAs drain, frees its TMEM and exits.
#include <mutex>

#include "device_common.cuh"
#include "kernels.h"

namespace pagedkv {
namespace {

constexpr int kTile = 128;
constexpr int kSoftmaxWarps = 8;          // two warpgroups: each owns half of the S / O columns
constexpr int kProducerWarp = 8;          // Q and K tiles
constexpr int kMmaWarp = 9;
constexpr int kProducerVWarp = 10;        // V tiles
constexpr int kThreadsP = 11 * 32;
constexpr float kLog2eP = 1.4426950408889634f;

struct PrefillParams {
    __half* out;
    const int32_t* block_tables;
    const int32_t* q_start;
    const int32_t* ctx_before;
    int32_t B, T, H, max_blocks, bs, num_blocks, grid_tiles, box_rows;
    float qscale;
    int32_t* err_flag;
};

template <int D>
struct PCfg {
    static constexpr int kChunks = D / 64;                        // 64-element (128-byte) column chunks
    static constexpr int kChunkBytes = kTile * 128;               // 128 rows x 128 B = 16 KB
    static constexpr int kOpBytes = kChunks * kChunkBytes;        // one Q, K or V tile
    static constexpr int kStages = 2;
    static constexpr size_t kOffQ = 0;
    static constexpr size_t kOffK = kOffQ + kOpBytes;
    static constexpr size_t kOffV = kOffK + size_t(kStages) * kOpBytes;
    static constexpr size_t kOffP = kOffV + size_t(kStages) * kOpBytes;
    static constexpr size_t kOffBar = kOffP + 2 * kChunkBytes;    // P: 128 rows x 128 keys fp16
    static constexpr int kNumBars = 23;
    static constexpr size_t kOffSlot = kOffBar + kNumBars * 8;
    static constexpr size_t kOffRed = kOffSlot + 64;                 // row-max exchange [2][2][128] + row sums [2][128]
    // Every CTA takes all 512 TMEM columns, so the request is kept above half the SM's shared
    // memory: one CTA per SM, and tcgen05.alloc never has to wait for a neighbour.
    static constexpr size_t kSmemUsed = kOffRed + 6 * 128 * 4 + 1024;
    static constexpr size_t kSmemBytes = kSmemUsed > 120 * 1024 ? kSmemUsed : 120 * 1024;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS = 0;                          // S buffers: columns 0 and 128
    static constexpr uint32_t kColO = 256;                        // O buffers: 256 and 256 + D
};

__device__ __forceinline__ void st_shared_u4(void* p, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(p)), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

template <int D>
__global__ void __launch_bounds__(kThreadsP, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, PrefillParams p) {
    using C = PCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + C::kOffQ;
    uint8_t* sK = smem + C::kOffK;
    uint8_t* sV = smem + C::kOffV;
    uint8_t* sP = smem + C::kOffP;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* q_full = bars + 0;
    uint64_t* k_full = bars + 1;     // [2]
    uint64_t* v_full = bars + 3;     // [2]
    uint64_t* k_empty = bars + 5;    // [2] released by the S MMA
    uint64_t* v_empty = bars + 21;   // [2] released by the P.V MMA
    uint64_t* s_full = bars + 7;     // [2]
    uint64_t* s_empty = bars + 9;    // [2]
    uint64_t* p_full = bars + 11;
    uint64_t* p_empty = bars + 12;
    uint64_t* o_full = bars + 13;    // [2]
    uint64_t* o_empty = bars + 15;   // [2]
    uint64_t* drain = bars + 17;
    uint64_t* red_bar = bars + 18;   // [2] row-max exchange between the two softmax warpgroups
    uint64_t* sum_bar = bars + 20;   // final row-sum exchange
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffSlot);
    volatile int* info = reinterpret_cast<volatile int*>(smem + C::kOffSlot + 16);   // b, qt, abort

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y;

    if (threadIdx.x == 0) {
        int g = p.grid_tiles - 1 - static_cast<int>(blockIdx.x);   // heaviest (latest) tiles first
        int bsel = -1, qt = 0;
        for (int b = 0; b < p.B; ++b) {
            const int s0 = p.q_start[b], s1 = p.q_start[b + 1];
            if (s0 < 0 || s1 < s0 || s1 > p.T) {
                flag_error(p.err_flag, PA_DEVCHK_QUERY_RANGE);
                bsel = -1;
                break;
            }
            const int nt = (s1 - s0 + kTile - 1) / kTile;
            if (bsel < 0 && g >= 0 && g < nt) { bsel = b; qt = g; }
            g -= nt;
        }
        if (bsel >= 0) {
            const int L = p.q_start[bsel + 1] - p.q_start[bsel];
            const int ctx = p.ctx_before[bsel];
            if (ctx < 0 || static_cast<int64_t>(ctx) + L > static_cast<int64_t>(p.max_blocks) * p.bs) {
                flag_error(p.err_flag, PA_DEVCHK_SEQ_LEN);
                bsel = -1;
            }
        }
        info[0] = bsel;
        info[1] = qt;
        info[2] = 0;
        mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&k_empty[i], 1);
            mbar_init(&v_empty[i], 1);
            mbar_init(&s_full[i], 1);
            mbar_init(&s_empty[i], kSoftmaxWarps);
            mbar_init(&o_full[i], 1);
            mbar_init(&o_empty[i], kSoftmaxWarps);
        }
        mbar_init(p_full, kSoftmaxWarps);
        mbar_init(p_empty, 1);
        mbar_init(drain, 1);
        mbar_init(&red_bar[0], kSoftmaxWarps);
        mbar_init(&red_bar[1], kSoftmaxWarps);
        mbar_init(sum_bar, kSoftmaxWarps);
        mbar_init_fence();
    }
    __syncthreads();
    const int b = info[0];
    if (b < 0) return;                                  // uniform: no tile for this CTA
    const int qt = info[1];
    const int s0 = p.q_start[b];
    const int L = p.q_start[b + 1] - s0;
    const int ctx = p.ctx_before[b];
    const int q0 = s0 + qt * kTile;                     // first query row of the tile
    const int rows = min(kTile, L - qt * kTile);
    const int kv_len = ctx + qt * kTile + rows;         // keys 0 .. kv_len-1 are visible to some row
    const int n_tiles = (kv_len + kTile - 1) / kTile;

    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    auto abort_now = [&]() {
        flag_error(p.err_flag, kDevchkTimeout);
        info[2] = 1;
    };

    if (warp == kProducerWarp || warp == kProducerVWarp) {
        // ======================================================= TMA producers (K warp, V warp)
        // A 128-key tile is one box per (physical block, 64-dim chunk): lane L issues box L of the tile,
        // so a tile goes out as one TMA instruction.  The next tile's block ids are read while the
        // current tile's copies go out.
        const bool is_k = warp == kProducerWarp;
        const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
        uint64_t* full = is_k ? k_full : v_full;
        uint64_t* empty = is_k ? k_empty : v_empty;
        uint8_t* base = is_k ? sK : sV;
        const uint64_t pol = l2_policy_evict_last();     // K/V tiles are re-read by the head's other q-tiles
        if (lane == 0) {
            tma_prefetch_desc(tm);
            if (is_k) {
                tma_prefetch_desc(&tm_q);
                mbar_arrive_expect_tx(q_full, C::kOpBytes);
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c)
                    tma_load_3d(sQ + c * C::kChunkBytes, &tm_q, q_full, c * 64, h, q0, pol);
            }
        }
        const int br = p.box_rows;
        const int64_t tbase = static_cast<int64_t>(b) * p.max_blocks;
        auto load_ids = [&](int j) -> int {
            const int key0 = j * kTile;
            const int nbox = (min(kTile, kv_len - key0) + br - 1) / br;
            int bid = 0;
            if (j < n_tiles && lane < nbox) {
                bid = p.block_tables[tbase + (key0 + lane * br) / p.bs];
                if (bid < 0 || bid >= p.num_blocks) {
                    flag_error(p.err_flag, PA_DEVCHK_BLOCK_ID);
                    bid = 0;
                }
            }
            return bid;
        };
        int last = -1;                                   // last tile whose copies this warp issued
        int bid = load_ids(0);
        for (int j = 0; j < n_tiles; ++j) {
            const int st = j & 1;
            const int key0 = j * kTile;
            const int nbox = (min(kTile, kv_len - key0) + br - 1) / br;
            const int bid_next = load_ids(j + 1);
            const int box = lane / C::kChunks, chunk = lane % C::kChunks;
            const int my_bid = __shfl_sync(0xffffffffu, bid, box);
            const uint32_t bytes = static_cast<uint32_t>(nbox * br * 128 * C::kChunks);
            if (!mbar_wait(&empty[st], ((j >> 1) & 1) ^ 1)) { abort_now(); break; }
            if (info[2]) break;
            if (lane == 0) mbar_arrive_expect_tx(&full[st], bytes);
            __syncwarp();
            if (box < nbox) {
                const int key = key0 + box * br;
                tma_load_3d(base + st * C::kOpBytes + chunk * C::kChunkBytes + box * br * 128, tm, &full[st],
                            chunk * 64, h, my_bid * p.bs + key % p.bs, pol);
            }
            last = j;
            bid = bid_next;
        }
        if (info[2]) {
            // unwind: let the copies this warp issued land
            for (int j = max(0, last - 1); j <= last; ++j) (void)mbar_wait(&full[j & 1], (j >> 1) & 1);
        }
    } else if (warp == kMmaWarp) {
        // ======================================================= MMA issuer
        if (lane == 0) {
            const uint32_t idesc_qk = umma_idesc_f16(kTile, kTile, false);
            const uint32_t idesc_pv = umma_idesc_f16(kTile, D, true);
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);
            bool ok = mbar_wait(q_full, 0);
            auto issue_s = [&](int j) -> bool {
                const int st = j & 1;
                if (!mbar_wait(&k_full[st], (j >> 1) & 1)) return false;
                if (!mbar_wait(&s_empty[j & 1], ((j >> 1) & 1) ^ 1)) return false;
                tc_fence_after_sync();
                const uint32_t d = tmem + C::kColS + (j & 1) * kTile;
                const uint32_t kb = aK + st * C::kOpBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
                    umma_f16_ss(d, umma_desc_sw128(aQ + off, 16, 1024), umma_desc_sw128(kb + off, 16, 1024), idesc_qk,
                                kk > 0);
                }
                umma_commit(&s_full[j & 1]);
                umma_commit(&k_empty[st]);
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int j = 0; ok && j < n_tiles; ++j) {
                if (j + 1 < n_tiles && !(ok = issue_s(j + 1))) break;
                const int st = j & 1;
                if (!(ok = mbar_wait(p_full, j & 1))) break;
                if (!(ok = mbar_wait(&v_full[st], (j >> 1) & 1))) break;
                if (!(ok = mbar_wait(&o_empty[j & 1], ((j >> 1) & 1) ^ 1))) break;
                if (info[2]) { ok = false; break; }
                tc_fence_after_sync();
                const uint32_t d = tmem + C::kColO + (j & 1) * D;
                const uint32_t vb = aV + st * C::kOpBytes;
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk) {
                    const uint32_t poff = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
                    umma_f16_ss(d, umma_desc_sw128(aP + poff, 16, 1024),
                                umma_desc_sw128(vb + kk * 16 * 128, C::kChunkBytes, 1024), idesc_pv, kk > 0);
                }
                umma_commit(&o_full[j & 1]);
                umma_commit(p_empty);
                umma_commit(&v_empty[st]);
            }
            if (!ok) {
                abort_now();
            }
            // every MMA this thread issued has completed before TMEM can be released
            umma_commit(drain);
            (void)mbar_wait(drain, 0);
        }
        __syncwarp();
    } else {
        // ======================================================= softmax warps
        // Thread (warpgroup g, row r): row r of the tile (TMEM lane r), columns g*64 .. g*64+63 of S
        // and g*D/2 .. (g+1)*D/2-1 of O.  The two threads of a row agree on the running max through
        // shared memory once per tile; each keeps a partial row sum, added at the end.
        const int g = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const int row_in_req = qt * kTile + r;
        const bool row_valid = row_in_req < L;
        const int row_pos = min(ctx + row_in_req, kv_len - 1);
        const int tile_pos0 = ctx + qt * kTile;          // smallest query position in the tile
        const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        constexpr int DH = D / 2;
        float* red = reinterpret_cast<float*>(smem + C::kOffRed);    // [parity][g][row], then sums [g][row]
        const float qs = p.qscale;
        float acc[DH];
#pragma unroll
        for (int i = 0; i < DH; ++i) acc[i] = 0.f;
        float m = -INFINITY, l = 0.f, alpha_prev = 0.f;
        bool ok = true;
        for (int j = 0; j < n_tiles && ok; ++j) {
            if (!(ok = mbar_wait(&s_full[j & 1], (j >> 1) & 1))) break;
            tc_fence_after_sync();
            const int key0 = j * kTile;
            const bool diag = key0 + kTile - 1 > tile_pos0;          // some key of the tile is masked
            const uint32_t sa = lane_base + C::kColS + (j & 1) * kTile + g * 64;
            float sv[64];
            {
                uint32_t r0[32], r1[32];                  // both loads in flight, one wait
                tmem_ld_32cols_nowait(sa, r0);
                tmem_ld_32cols_nowait(sa + 32, r1);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) { sv[i] = __uint_as_float(r0[i]); sv[32 + i] = __uint_as_float(r1[i]); }
            }
            if (diag) {
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    if (key0 + g * 64 + i > row_pos) sv[i] = -INFINITY;
            }
            float mx8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) mx8[k] = sv[k];
#pragma unroll
            for (int i = 8; i < 64; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], sv[i]);
            float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
            // raw scores: scale > 0 keeps the order, so the max is taken before scaling
            float* rm = red + (j & 1) * 256;
            rm[g * 128 + r] = mx;
            __syncwarp();
            if (lane == 0) mbar_arrive(&red_bar[j & 1]);
            if (!(ok = mbar_wait(&red_bar[j & 1], (j >> 1) & 1))) break;
            mx = fmaxf(mx, rm[(g ^ 1) * 128 + r]) * qs;
            const float m_new = fmaxf(m, mx);
            const float m_use = m_new == -INFINITY ? 0.f : m_new;
            const float alpha = exp2f(m - m_use);
            if (!(ok = mbar_wait(p_empty, (j & 1) ^ 1))) break;
            // P = 2^(s*scale*log2e - m) computed two at a time in fp16 (P is stored in fp16 for the
            // P.V MMA anyway); the row sum adds exactly the fp16 values that MMA will use.
            float rs4[4] = {0.f, 0.f, 0.f, 0.f};
            uint8_t* prow = sP + g * C::kChunkBytes + r * 128;
#pragma unroll
            for (int u = 0; u < 8; ++u) {                     // 8 keys = one 16-byte unit of P
                uint32_t pk[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const __half2 x = __floats2half2_rn(fmaf(sv[8 * u + 2 * i], qs, -m_use),
                                                        fmaf(sv[8 * u + 2 * i + 1], qs, -m_use));
                    const __half2 e = h2exp2(x);
                    const float2 ef = __half22float2(e);
                    rs4[i] += ef.x + ef.y;
                    pk[i] = *reinterpret_cast<const uint32_t*>(&e);
                }
                st_shared_u4(prow + ((u ^ (r & 7)) * 16), make_uint4(pk[0], pk[1], pk[2], pk[3]));
            }
            const float rs = (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[j & 1]);
            if (j == n_tiles - 1 && kv_len < key0 + kTile) {
                // rows of V past the sequence end may hold anything: zero them before P.V reads them
                if (!(ok = mbar_wait(&v_full[j & 1], (j >> 1) & 1))) break;
                if (key0 + r >= kv_len) {
                    uint8_t* vrow = sV + (j & 1) * C::kOpBytes + r * 128;
#pragma unroll
                    for (int c = 0; c < C::kChunks; ++c)
#pragma unroll
                        for (int u = 0; u < 8 / 2; ++u)
                            st_shared_u4(vrow + c * C::kChunkBytes + (g * 4 + u) * 16, make_uint4(0, 0, 0, 0));
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
            l = fmaf(l, alpha, rs);
            if (j > 0) {
                const int jp = j - 1;
                if (!(ok = mbar_wait(&o_full[jp & 1], (jp >> 1) & 1))) break;
                tc_fence_after_sync();
                const uint32_t oa = lane_base + C::kColO + (jp & 1) * D + g * DH;
#pragma unroll
                for (int c = 0; c < DH / 32; ++c) {
                    float v[32];
                    tmem_ld_32cols(oa + c * 32, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) acc[c * 32 + i] = fmaf(acc[c * 32 + i], alpha_prev, v[i]);
                }
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&o_empty[jp & 1]);
            }
            alpha_prev = alpha;
            m = m_new;
            if (info[2]) ok = false;
        }
        if (ok) {
            const int jp = n_tiles - 1;
            ok = mbar_wait(&o_full[jp & 1], (jp >> 1) & 1);
            if (ok) {
                tc_fence_after_sync();
                const uint32_t oa = lane_base + C::kColO + (jp & 1) * D + g * DH;
#pragma unroll
                for (int c = 0; c < DH / 32; ++c) {
                    float v[32];
                    tmem_ld_32cols(oa + c * 32, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) acc[c * 32 + i] = fmaf(acc[c * 32 + i], alpha_prev, v[i]);
                }
            }
        }
        // both threads of a row add their partial sums (every softmax thread reaches this barrier)
        float* rsum = red + 512;
        rsum[g * 128 + r] = l;
        __syncwarp();
        if (lane == 0) mbar_arrive(sum_bar);
        if (ok) ok = mbar_wait(sum_bar, 0);
        l += rsum[(g ^ 1) * 128 + r];
        if (ok && row_valid) {
            const float inv = 1.f / l;
            __half* orow = p.out + (static_cast<int64_t>(q0 + r) * p.H + h) * D + g * DH;
#pragma unroll
            for (int c = 0; c < DH / 8; ++c) {
                uint4 o;
                o.x = f2_to_h2(acc[8 * c + 0] * inv, acc[8 * c + 1] * inv);
                o.y = f2_to_h2(acc[8 * c + 2] * inv, acc[8 * c + 3] * inv);
                o.z = f2_to_h2(acc[8 * c + 4] * inv, acc[8 * c + 5] * inv);
                o.w = f2_to_h2(acc[8 * c + 6] * inv, acc[8 * c + 7] * inv);
                *reinterpret_cast<uint4*>(orow + 8 * c) = o;
            }
        }
        if (!ok) abort_now();
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int D>
cudaError_t run_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const PrefillParams& p,
                        dim3 grid, cudaStream_t stream) {
    using C = PCfg<D>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(C::kSmemBytes));
    });
    if (attr_err != cudaSuccess) return attr_err;
    prefill_kernel<D><<<grid, kThreadsP, C::kSmemBytes, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace

bool prefill_supported(int32_t H, int32_t D, int32_t bs) {
    return (D == 64 || D == 128) && H > 0 && H <= 65535 && bs >= 8 && bs % 8 == 0;
}

cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t stream, const char** why) {
    const int br = std::min(kTile, a.block_size & -a.block_size);    // largest power of two dividing bs, <= 128
    const uint64_t s1 = static_cast<uint64_t>(a.head_dim) * 2, s2 = s1 * a.num_heads;
    const uint64_t rows = static_cast<uint64_t>(a.num_blocks) * a.block_size;
    alignas(64) CUtensorMap tq, tk, tv;
    if (!encode_tensor_map_3d(&tq, a.q, a.head_dim, a.num_heads, a.num_tokens, s1, s2, 64, 1, kTile, 1, why) ||
        !encode_tensor_map_3d(&tk, a.k_cache, a.head_dim, a.num_heads, rows, s1, s2, 64, 1, br, 1, why) ||
        !encode_tensor_map_3d(&tv, a.v_cache, a.head_dim, a.num_heads, rows, s1, s2, 64, 1, br, 1, why))
        return cudaErrorInvalidValue;
    PrefillParams p;
    p.out = static_cast<__half*>(a.out);
    p.block_tables = a.block_tables;
    p.q_start = a.q_start;
    p.ctx_before = a.ctx_before;
    p.B = a.num_reqs;
    p.T = a.num_tokens;
    p.H = a.num_heads;
    p.max_blocks = a.max_blocks;
    p.bs = a.block_size;
    p.num_blocks = a.num_blocks;
    p.grid_tiles = (a.num_tokens + kTile - 1) / kTile + a.num_reqs;
    p.box_rows = br;
    p.qscale = a.scale * kLog2eP;
    p.err_flag = a.err_flag;
    const dim3 grid(p.grid_tiles, a.num_heads);
    if (a.head_dim == 128) return run_prefill<128>(tq, tk, tv, p, grid, stream);
    return run_prefill<64>(tq, tk, tv, p, grid, stream);
}

}  // namespace pagedkv
