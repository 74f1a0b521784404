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
// This is the kernel for small launches: when a chunk has too few (256-row
// query block, head) pairs to fill the GPU with prefill.cu's two-query-tile
// CTAs (a short chunk after a long cached prefix, e.g. 512 rows after 1536
// cached tokens), the launcher runs it instead, twice as many CTAs of half
// the rows each.
//
// One CTA computes one tile of 128 query rows x one head (FlashAttention
// order, online softmax over 128-key tiles):
//   * kIssueWarps K warps and kIssueWarps V warps (producers, from warp 8) load
//     the Q tile once and stream the K and the V tiles into two-stage rings
//     with TMA: a tile of 128 keys is gathered from the paged pool with one 3-D
//     box per (physical block, 64-dim chunk) ([box rows][1 head][64 dims],
//     128-byte swizzle), landing directly in the canonical UMMA layout; the
//     boxes are dealt to the lanes of the operand's warps, one each, and the
//     next tile's block ids are read a tile ahead;
//   * the last warp (one elected thread) issues tcgen05.mma: S = Q K^T (A and B
//     K-major) into a double-buffered fp32 TMEM tile, and P V (A = P read from
//     TMEM, B MN-major straight from the V tile) accumulated in TMEM across all
//     key tiles as two partial outputs, O_0 over the first 64 keys of every
//     tile and O_1 over the last 64; completions are signalled with
//     tcgen05.commit on mbarriers;
//   * warps 0-7 (two threads per query row = per TMEM lane; thread g of a row
//     owns key columns g*64 .. g*64+63 of every tile and so the partial output
//     O_g) read S with tcgen05.ld, apply the causal mask on the diagonal tiles
//     and run the online softmax of their half on their own: each keeps its own
//     running max m_g and sum l_g, and P = 2^(s*scale*log2e - m_g) is written
//     as fp16 pairs over the first half of the thread's own S columns in TMEM,
//     where the P V MMA reads it (shared memory carries only Q, K and V).
//     m_g only moves when a tile's max exceeds it by more than kRescaleLog2
//     (P then stays <= 2^kRescaleLog2, exact in fp16 up to its 11-bit
//     mantissa); when it moves, the warp rescales its rows of O_g in TMEM
//     (after the previous P V has completed) before the next P V adds to it.
//     The two halves of a row are merged once, after the last tile:
//     O = (O_0 2^(m_0-M) + O_1 2^(m_1-M)) / (l_0 2^(m_0-M) + l_1 2^(m_1-M)),
//     M = max(m_0, m_1).  The MMA of tile j+1 overlaps the softmax of tile j.
// Keys past the tile's last query position are masked; rows of V past the
// sequence end are zeroed before P.V so stale or poisoned pool rows never
// reach the MMA.  Every wait is bounded; on a timeout the CTA records
// PA_DEVCHK_TIMEOUT, lets its copies and MMAs drain, frees its TMEM and exits.

#include "device_common.cuh"
#include "kernels.h"

namespace pagedkv {
namespace {

constexpr int kTile = 128;
constexpr int kSoftmaxWarps = 8;          // two warpgroups: each owns half of the key columns of S
constexpr int kIssueWarps = 2;                        // TMA-issuing warps per operand (K, V)
constexpr int kFirstKWarp = 8;                        // K warps (the first also loads Q)
constexpr int kFirstVWarp = kFirstKWarp + kIssueWarps;
constexpr int kMmaWarp = kFirstVWarp + kIssueWarps;
constexpr int kThreadsP = (kMmaWarp + 1) * 32;
constexpr float kLog2eP = 1.4426950408889634f;
// A thread's running max (log2 domain) is raised only when a tile's max exceeds it by more than this;
// P <= 2^kRescaleLog2 = 256 is exact enough in fp16 and far from its overflow.
constexpr float kRescaleLog2 = 8.f;

struct PrefillParams {
    __half* out;
    const int32_t* block_tables;
    const int32_t* q_start;
    const int32_t* ctx_before;
    int32_t B, T, H, max_blocks, bs, num_blocks, grid_tiles, box_rows;
    float qscale;
    int32_t* err_flag;
    uint64_t wait_ns;          // limit of every pipeline wait (kWaitLimitNs by default)
    int32_t stall;             // test hook: the softmax warps first wait on a barrier nothing completes
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
    static constexpr size_t kOffBar = kOffV + size_t(kStages) * kOpBytes;
    static constexpr int kNumBars = 13;
    static constexpr size_t kOffSlot = kOffBar + kNumBars * 8;
    static constexpr size_t kOffRed = kOffSlot + 64;                 // final exchange: maxes [2][128], sums [2][128]
    // Every CTA takes all 512 TMEM columns, so the request is kept above half the SM's shared
    // memory: one CTA per SM, and tcgen05.alloc never has to wait for a neighbour.
    static constexpr size_t kSmemUsed = kOffRed + 4 * 128 * 4 + 1024;
    static constexpr size_t kSmemBytes = kSmemUsed > 120 * 1024 ? kSmemUsed : 120 * 1024;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS = 0;                          // S buffers: columns 0 and 128
    static constexpr uint32_t kColO = 256;                        // O_0 at 256, O_1 at 256 + D
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
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* q_full = bars + 0;
    uint64_t* k_full = bars + 1;     // [2]
    uint64_t* v_full = bars + 3;     // [2]
    uint64_t* s_full = bars + 5;     // [2] S(j) is in TMEM, which also frees K stage j % 2
    uint64_t* p_full = bars + 7;
    uint64_t* pv_done = bars + 8;    // [2] P.V(j) has landed in O_0/O_1, which also frees V stage j % 2
    uint64_t* drain = bars + 10;
    uint64_t* sum_bar = bars + 11;   // final (max, sum) exchange between the two halves of a row
    uint64_t* never = bars + 12;     // no thread ever arrives on it (failure-detection test)
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
            mbar_init(&k_full[i], kIssueWarps);
            mbar_init(&v_full[i], kIssueWarps);
            mbar_init(&s_full[i], 1);
            mbar_init(&pv_done[i], 1);
        }
        mbar_init(p_full, kSoftmaxWarps);
        mbar_init(drain, 1);
        mbar_init(sum_bar, kSoftmaxWarps);
        mbar_init(never, 1);
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

    if (warp >= kFirstKWarp && warp < kMmaWarp) {
        // ======================================================= TMA producers (K warps, V warps)
        // A 128-key tile is one box per (physical block, 64-dim chunk).  The boxes of a tile are dealt
        // round-robin to the operand's kIssueWarps warps, one per lane, so a tile goes out as one TMA
        // instruction per warp; every warp arrives on the stage's barrier with its own byte count.
        // Each lane reads the block id of its box of the next tile while the current tile's copies go
        // out, and checks it only when it uses it, so the read's latency stays off the issue path.
        const bool is_k = warp < kFirstVWarp;
        const int wsub = warp - (is_k ? kFirstKWarp : kFirstVWarp);
        const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
        uint64_t* full = is_k ? k_full : v_full;
        uint64_t* empty = is_k ? s_full : pv_done;      // stage j % 2 is free once S / P.V of tile j-2 is done
        uint8_t* base = is_k ? sK : sV;
        const uint64_t pol = l2_policy_evict_last();     // K/V tiles are re-read by the head's other q-tiles
        if (lane == 0) {
            tma_prefetch_desc(tm);
            if (is_k && wsub == 0) {
                tma_prefetch_desc(&tm_q);
                mbar_arrive_expect_tx(q_full, C::kOpBytes);
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c)
                    tma_load_3d(sQ + c * C::kChunkBytes, &tm_q, q_full, c * 64, h, q0, pol);
            }
        }
        const int br = p.box_rows;
        const int64_t tbase = static_cast<int64_t>(b) * p.max_blocks;
        const int my_i = lane * kIssueWarps + wsub;      // this lane's box of every tile
        const int box = my_i / C::kChunks, chunk = my_i % C::kChunks;
        auto nbox_of = [&](int j) { return (min(kTile, kv_len - j * kTile) + br - 1) / br; };
        auto read_id = [&](int j) -> int {               // raw table entry; checked at use
            return (j < n_tiles && box < nbox_of(j)) ? p.block_tables[tbase + (j * kTile + box * br) / p.bs] : 0;
        };
        int last = -1;                                   // last tile whose copies this warp issued
        int bid = read_id(0);
        for (int j = 0; j < n_tiles; ++j) {
            const int st = j & 1;
            const int nbox = nbox_of(j);
            const int bid_next = read_id(j + 1);
            const int n_mine = (nbox * C::kChunks - wsub + kIssueWarps - 1) / kIssueWarps;
            const uint32_t bytes = static_cast<uint32_t>(n_mine * br * 128);
            if (!mbar_wait(&empty[st], ((j >> 1) & 1) ^ 1, p.wait_ns)) { abort_now(); break; }
            if (info[2]) break;
            if (lane == 0) mbar_arrive_expect_tx(&full[st], bytes);
            __syncwarp();
            if (box < nbox) {
                int my_bid = bid;
                if (my_bid < 0 || my_bid >= p.num_blocks) {
                    flag_error(p.err_flag, PA_DEVCHK_BLOCK_ID);
                    my_bid = 0;
                }
                const int key = j * kTile + box * br;
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
            // base descriptors, built once: a k-step's operand is the base advanced by a constant
            const uint64_t dQ = umma_desc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t dK = umma_desc_sw128(smem_u32(sK), 16, 1024);
            const uint64_t dV = umma_desc_sw128(smem_u32(sV), C::kChunkBytes, 1024);
            bool ok = mbar_wait(q_full, 0, p.wait_ns);
            // An mbarrier answers after ~150 cycles even when its phase is complete, so this thread asks
            // early (mbar_test_wait) and collects the answers after the MMAs it issues meanwhile; it only
            // blocks when a phase really is still open.
            auto issue_s = [&](int j, bool k_ready) -> bool {
                const int st = j & 1;
                if (!k_ready && !mbar_wait(&k_full[st], (j >> 1) & 1, p.wait_ns)) return false;
                // S(j) reuses the buffer of S(j-2)/P(j-2): it is issued after P.V(j-2), which the
                // tensor core runs first, and P.V(j-2) waited for every softmax warp to finish that tile
                tc_fence_after_sync();
                const uint32_t d = tmem + C::kColS + (j & 1) * kTile;
                const uint64_t dKs = umma_desc_advance(dK, st * C::kOpBytes);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
                    umma_f16_ss(d, umma_desc_advance(dQ, off), umma_desc_advance(dKs, off), idesc_qk, kk > 0);
                }
                umma_commit(&s_full[st]);
                return true;
            };
            if (ok) ok = issue_s(0, false);
            bool k_ready = ok && n_tiles > 1 && mbar_test_wait(&k_full[1], 0);
            for (int j = 0; ok && j < n_tiles; ++j) {
                const int st = j & 1;
                const bool p_ready = mbar_test_wait(p_full, j & 1);
                const bool v_ready = mbar_test_wait(&v_full[st], (j >> 1) & 1);
                if (j + 1 < n_tiles && !(ok = issue_s(j + 1, k_ready))) break;
                if (!p_ready && !(ok = mbar_wait(p_full, j & 1, p.wait_ns))) break;
                if (!v_ready && !(ok = mbar_wait(&v_full[st], (j >> 1) & 1, p.wait_ns))) break;
                if (info[2]) { ok = false; break; }
                k_ready = j + 2 < n_tiles && mbar_test_wait(&k_full[st], ((j + 2) >> 1) & 1);   // for S(j+2)
                tc_fence_after_sync();
                const uint64_t dVs = umma_desc_advance(dV, st * C::kOpBytes);
                const uint32_t pbase = tmem + C::kColS + (j & 1) * kTile;
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk) {
                    // keys 0-63 of the tile add to O_0, keys 64-127 to O_1; tile 0 starts both.  P of
                    // keys 64h .. 64h+63 is fp16 in columns 64h .. 64h+31 of the tile's S buffer.
                    const uint32_t d = tmem + C::kColO + (kk >> 2) * D;
                    const uint32_t pa = pbase + (kk >> 2) * 64 + (kk & 3) * 8;
                    umma_f16_ts(d, pa, umma_desc_advance(dVs, kk * 16 * 128), idesc_pv, j > 0 || (kk & 3) != 0);
                }
                umma_commit(&pv_done[st]);
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
        // Thread (warpgroup g, row r): row r of the tile (TMEM lane r), key columns g*64 .. g*64+63 of
        // every S tile, and the partial output O_g of those keys (all D columns of row r).
        const int g = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const int row_in_req = qt * kTile + r;
        const bool row_valid = row_in_req < L;
        const int row_pos = min(ctx + row_in_req, kv_len - 1);
        const int tile_pos0 = ctx + qt * kTile;          // smallest query position in the tile
        const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const uint32_t o_mine = lane_base + C::kColO + g * D;
        const float qs = p.qscale;
        float m = -INFINITY, l = 0.f;                    // log2-domain running max and sum of this half
        // failure-detection test: the wait runs out and the softmax role stops; the MMA issuer and the
        // producers then run out of their own waits and unwind
        bool ok = !p.stall || mbar_wait(never, 0, p.wait_ns);
        for (int j = 0; j < n_tiles && ok; ++j) {
            if (!(ok = mbar_wait(&s_full[j & 1], (j >> 1) & 1, p.wait_ns))) break;
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
            // raw scores: scale > 0 keeps the order, so the max is taken before scaling (three operands per
            // instruction)
            float mx8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) mx8[k] = fmax3(sv[k], sv[k + 8], sv[k + 16]);
#pragma unroll
            for (int i = 24; i < 64; i += 2) mx8[(i >> 1) & 7] = fmax3(mx8[(i >> 1) & 7], sv[i], sv[i + 1]);
            const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                                   fmaxf(mx8[6], mx8[7])) * qs;
            float alpha = 1.f;
            const bool raise = mx > m + kRescaleLog2;                // false while both are -inf
            if (raise) {
                alpha = exp2f(m - mx);                               // 0 when m is still -inf
                m = mx;
            }
            const float m_use = m == -INFINITY ? 0.f : m;
            uint32_t pk[32];
            float rs4[4] = {0.f, 0.f, 0.f, 0.f};
            const uint64_t qs2 = f32x2_pack(qs, qs), nm2 = f32x2_pack(-m_use, -m_use);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                float x0, x1;                             // the scaling in packed f32x2 arithmetic
                f32x2_unpack(fma_f32x2(f32x2_pack(sv[2 * i], sv[2 * i + 1]), qs2, nm2), x0, x1);
                pk[i] = f2_to_h2(exp2f(x0), exp2f(x1));
                rs4[i & 3] = add_h2_f32(rs4[i & 3], pk[i]);   // the fp16 values the P.V MMA adds
            }
            l = fmaf(l, alpha, (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]));
            if (j > 0 && __any_sync(0xffffffffu, raise)) {
                // O_g holds the sum up to tile j-1: wait for that P.V, then rescale this warp's rows
                if (!(ok = mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, p.wait_ns))) break;
                tc_fence_after_sync();
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    float v[32];
                    tmem_ld_32cols(o_mine + c * 32, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] *= alpha;
                    tmem_st_32cols(o_mine + c * 32, v);
                }
            }
            // P (fp16 pairs) over the first half of this thread's S columns, which it has already read;
            // the P.V of tile j-2, the last reader of this buffer, completed before S(j) did
            tmem_st_32cols_u(sa, pk);
            tmem_wait_st();
            if (j == n_tiles - 1 && kv_len < key0 + kTile) {
                // rows of V past the sequence end may hold anything: zero them before P.V reads them
                if (!(ok = mbar_wait(&v_full[j & 1], (j >> 1) & 1, p.wait_ns))) break;
                if (key0 + r >= kv_len) {
                    uint8_t* vrow = sV + (j & 1) * C::kOpBytes + r * 128;
#pragma unroll
                    for (int c = 0; c < C::kChunks; ++c)
#pragma unroll
                        for (int u = 0; u < 8 / 2; ++u)
                            st_shared_u4(vrow + c * C::kChunkBytes + (g * 4 + u) * 16, make_uint4(0, 0, 0, 0));
                }
                fence_proxy_async_smem();                     // the zeros reach the tensor core's view
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
            if (info[2]) ok = false;
        }
        // merge the two halves of the row (every softmax thread reaches this barrier)
        float* red = reinterpret_cast<float*>(smem + C::kOffRed);    // maxes [g][row], then sums [g][row]
        red[g * 128 + r] = m;
        red[256 + g * 128 + r] = l;
        __syncwarp();
        if (lane == 0) mbar_arrive(sum_bar);
        if (ok) ok = mbar_wait(sum_bar, 0, p.wait_ns);
        if (ok) ok = mbar_wait(&pv_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, p.wait_ns);   // the last P.V has landed
        if (ok) {
            tc_fence_after_sync();
            const float m0 = red[r], m1 = red[128 + r];
            const float mm = fmaxf(m0, m1);
            const float c0 = exp2f(m0 - mm), c1 = exp2f(m1 - mm);    // a half that saw no key: 0
            const float inv = 1.f / (red[256 + r] * c0 + red[384 + r] * c1);
            const float s0 = c0 * inv, s1 = c1 * inv;
            constexpr int DH = D / 2;                                // this thread writes columns g*DH ..
            __half* orow = p.out + (static_cast<int64_t>(q0 + r) * p.H + h) * D + g * DH;
#pragma unroll 1
            for (int c = 0; c < DH / 32; ++c) {
                uint32_t a0[32], a1[32];
                tmem_ld_32cols_nowait(lane_base + C::kColO + g * DH + c * 32, a0);
                tmem_ld_32cols_nowait(lane_base + C::kColO + D + g * DH + c * 32, a1);
                tmem_wait_ld();
                if (row_valid) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 o;
                        uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i = 8 * q + 2 * e;
                            ow[e] = f2_to_h2(__uint_as_float(a0[i]) * s0 + __uint_as_float(a1[i]) * s1,
                                             __uint_as_float(a0[i + 1]) * s0 + __uint_as_float(a1[i + 1]) * s1);
                        }
                        *reinterpret_cast<uint4*>(orow + c * 32 + 8 * q) = o;
                    }
                }
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
    static std::atomic<uint64_t> smem_set{0};          // devices whose limit is raised
    const cudaError_t attr_err = ensure_dynamic_smem(reinterpret_cast<const void*>(prefill_kernel<D>),
                                                     static_cast<int>(C::kSmemBytes), &smem_set);
    if (attr_err != cudaSuccess) return attr_err;
    prefill_kernel<D><<<grid, kThreadsP, C::kSmemBytes, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_q128(const PrefillArgs& a, uint64_t wait_ns, bool stall, cudaStream_t stream,
                                const char** why) {
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
    p.wait_ns = wait_ns;
    p.stall = stall;
    const dim3 grid(p.grid_tiles, a.num_heads);
    if (a.head_dim == 128) return run_prefill<128>(tq, tk, tv, p, grid, stream);
    return run_prefill<64>(tq, tk, tv, p, grid, stream);
}

}  // namespace pagedkv
