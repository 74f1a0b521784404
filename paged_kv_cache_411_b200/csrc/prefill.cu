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
// One CTA computes 256 query rows of one head as two 128-row query tiles, Q0
// and Q1, that share every K and V tile (FlashAttention order, online softmax
// over 128-key tiles).  The two tiles exist so that the tensor core always has
// independent work queued: while softmax warpgroup 0 turns S0(j) into P0(j),
// the tensor core runs P1(j-1) V and S1(j), and the other way round.
//   * Producers (warp 8: K, warp 9: V; warp 8 also loads Q0 and Q1 once)
//     stream 128-key tiles into two-stage rings with TMA.  A tile is gathered
//     from the paged pool with one 3-D box per (physical block, 64-dim chunk)
//     ([box rows][1 head][64 dims], 128-byte swizzle), landing directly in the
//     canonical UMMA layouts; each lane issues one box and reads the block id
//     of its box of the next tile a tile ahead.  After the last V tile has
//     landed, the V warp zeroes its rows past the sequence end (pool rows
//     there may hold anything, and 0 * NaN would poison P V).
//   * MMA issuer (warp 10, one thread): tcgen05.mma kind::f16 with fp32
//     accumulators in TMEM.  S_g(j) = Q_g K_j^T into the tile's S buffer;
//     O_g += P_g(j) V_j with A = P_g read from TMEM (fp16, over the first half
//     of the S buffer) and B = V_j from shared memory.  Issue order per key
//     tile: P0 V, S0(j+1), P1 V, S1(j+1); a commit after each group signals the
//     softmax warps (S landed, P V landed) and the producers (K / V stage free).
//   * Softmax warpgroups 0 and 1 (warps 0-3 and 4-7; one thread per query row
//     = TMEM lane): read the 128 scores of S_g(j) with tcgen05.ld into
//     registers (11 warps leave each thread 168), take the row max (causal
//     mask on the diagonal tiles only), and write P = 2^(s*scale*log2e - m) as
//     fp16 pairs over the first half of the S buffer with tcgen05.st.  The running
//     max m only moves when a tile's max exceeds it by more than kRescaleLog2
//     (P then stays <= 2^kRescaleLog2, exact in fp16 to its 11-bit mantissa);
//     when it moves, the warp rescales its rows of O_g in TMEM after the
//     previous P V has landed and before the next one is issued.  The scaling
//     runs in packed f32x2 arithmetic, the row max takes three operands per
//     instruction, and the row sum adds the same fp16 values of P that the P V
//     MMA adds.  After the last tile each thread normalises its row of O_g and
//     stores it as fp16.
// When a launch has too few (256-row query block, head) pairs to fill the GPU
// (a short chunk after a long cached prefix), the launcher runs the
// one-query-tile kernel of prefill_q128.cu instead, with twice as many CTAs.
// Every wait is bounded; on a timeout the CTA records PA_DEVCHK_TIMEOUT, lets
// its copies and MMAs drain, frees its TMEM and exits.
#include <algorithm>
#include <cstdlib>

#include "device_common.cuh"
#include "kernels.h"

namespace pagedkv {
namespace {

constexpr int kTile = 128;                      // query rows of a query tile = keys of a key tile
constexpr int kQTiles = 2;                      // query tiles per CTA, one softmax warpgroup each
constexpr int kRowsPerCta = kQTiles * kTile;
constexpr int kSoftmaxWarps = 4 * kQTiles;
constexpr int kIssueWarps = 1;                  // TMA-issuing warps per operand (K, V)
constexpr int kFirstKWarp = kSoftmaxWarps;      // K warps (the first also loads Q)
constexpr int kFirstVWarp = kFirstKWarp + kIssueWarps;
constexpr int kMmaWarp = kFirstVWarp + kIssueWarps;
constexpr int kThreadsP = (kMmaWarp + 1) * 32;
constexpr float kLog2eP = 1.4426950408889634f;
// A row's running max (log2 domain) is raised only when a tile's max exceeds it by more than this;
// P <= 2^kRescaleLog2 = 256 is exact enough in fp16 and far from its overflow.
constexpr float kRescaleLog2 = 8.f;

struct PrefillParams {
    __half* out;
    const int32_t* block_tables;
    const int32_t* q_start;
    const int32_t* ctx_before;
    int32_t B, T, H, max_blocks, bs, num_blocks, grid_blocks, box_rows;
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
    static constexpr size_t kOffQ = 0;                            // Q0, Q1
    static constexpr size_t kOffK = kOffQ + size_t(kQTiles) * kOpBytes;
    static constexpr size_t kOffV = kOffK + size_t(kStages) * kOpBytes;
    static constexpr size_t kOffBar = kOffV + size_t(kStages) * kOpBytes;
    static constexpr int kNumBars = 18;
    static constexpr size_t kOffSlot = kOffBar + kNumBars * 8;
    // Every CTA takes all 512 TMEM columns, so the request is kept above half the SM's shared
    // memory: one CTA per SM, and tcgen05.alloc never has to wait for a neighbour.
    static constexpr size_t kSmemUsed = kOffSlot + 64 + 1024;
    static constexpr size_t kSmemBytes = kSmemUsed > 120 * 1024 ? kSmemUsed : 120 * 1024;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS = 0;                          // S_g at g * 128 (P_g over its first 64)
    static constexpr uint32_t kColO = kQTiles * kTile;            // O_g at 256 + g * D
    static_assert(kColO + kQTiles * D <= kTmemCols, "TMEM budget");
    static_assert(kSmemUsed <= 227 * 1024, "shared-memory budget");
};

__device__ __forceinline__ void st_shared_zero16(uint32_t addr) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0) : "memory");
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
    uint64_t* k_full = bars + 1;     // [2] K stage landed
    uint64_t* k_empty = bars + 3;    // [2] every S MMA reading the K stage has completed
    uint64_t* v_full = bars + 5;     // [2] V stage landed
    uint64_t* v_empty = bars + 7;    // [2] every P V MMA reading the V stage has completed
    uint64_t* v_tail = bars + 9;     // the last V tile's rows past the sequence end are zero
    uint64_t* s_full = bars + 10;    // [g] S_g(j) is in TMEM
    uint64_t* p_full = bars + 12;    // [g] P_g(j) is in TMEM (and O_g rescaled if needed)
    uint64_t* pv_done = bars + 14;   // [g] O_g += P_g(j) V_j has landed
    uint64_t* drain = bars + 16;
    uint64_t* never = bars + 17;     // no thread ever arrives on it (failure-detection test)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffSlot);
    // b, qb, abort, and the request's first row, chunk length and cached length
    volatile int* info = reinterpret_cast<volatile int*>(smem + C::kOffSlot + 16);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const unsigned work = blockIdx.x;                   // the (query block, head) pair of this CTA
    const int h = static_cast<int>(work % static_cast<unsigned>(p.H));
    const int rank = static_cast<int>(work / static_cast<unsigned>(p.H));

    if (warp == kMmaWarp) {                             // TMEM while thread 0 finds the work item
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        int g = p.grid_blocks - 1 - rank;        // the latest (heaviest) query blocks go first
        int bsel = -1, qb = 0, s_sel = 0, l_sel = 0, c_sel = 0;
        for (int b = 0; b < p.B; ++b) {
            // the request's cached length is read with its rows, so finding the item is one round trip
            const int s0 = p.q_start[b], s1 = p.q_start[b + 1], cb = p.ctx_before[b];
            if (s0 < 0 || s1 < s0 || s1 > p.T) {
                flag_error(p.err_flag, PA_DEVCHK_QUERY_RANGE);
                bsel = -1;
                break;
            }
            const int nb = (s1 - s0 + kRowsPerCta - 1) / kRowsPerCta;
            if (bsel < 0 && g >= 0 && g < nb) { bsel = b; qb = g; s_sel = s0; l_sel = s1 - s0; c_sel = cb; }
            g -= nb;
        }
        if (bsel >= 0 && (c_sel < 0 || static_cast<int64_t>(c_sel) + l_sel > static_cast<int64_t>(p.max_blocks) * p.bs)) {
            flag_error(p.err_flag, PA_DEVCHK_SEQ_LEN);
            bsel = -1;
        }
        info[0] = bsel;
        info[1] = qb;
        info[2] = 0;
        info[3] = s_sel;
        info[4] = l_sel;
        info[5] = c_sel;
        mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&k_full[i], kIssueWarps);
            mbar_init(&v_full[i], kIssueWarps);
            mbar_init(&k_empty[i], 1);
            mbar_init(&v_empty[i], 1);
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 4);
            mbar_init(&pv_done[i], 1);
        }
        mbar_init(v_tail, 1);
        mbar_init(drain, 1);
        mbar_init(never, 1);
        mbar_init_fence();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const int b = info[0];
    if (b < 0) {                                        // uniform: no work for this CTA
        if (warp == kMmaWarp) tmem_dealloc(tmem, C::kTmemCols);
        return;
    }
    const int qb = info[1];
    const int s0 = info[3];
    const int L = info[4];
    const int ctx = info[5];
    const int row0 = qb * kRowsPerCta;                  // first row of Q0 within the request
    const int q0 = s0 + row0;                           // ... within q / out
    // query tile g: its valid rows, the keys its last valid row sees, and the key tiles that covers
    int rows_g[kQTiles], kvl_g[kQTiles], n_g[kQTiles];
#pragma unroll
    for (int g = 0; g < kQTiles; ++g) {
        rows_g[g] = max(0, min(kTile, L - row0 - g * kTile));
        kvl_g[g] = rows_g[g] > 0 ? ctx + row0 + g * kTile + rows_g[g] : 0;
        n_g[g] = (kvl_g[g] + kTile - 1) / kTile;
    }
    const int kv_len = max(kvl_g[0], kvl_g[1]);
    const int n_tiles = max(n_g[0], n_g[1]);            // >= 1: Q0 always has a valid row
    // this CTA's key tiles [jb, je) and query tile g's share of them [jb, je_g)
    const int jb = 0, je = n_tiles;
    const int n_loc = je - jb;
    int je_g[kQTiles];
#pragma unroll
    for (int g = 0; g < kQTiles; ++g) je_g[g] = max(jb, min(je, n_g[g]));

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
        uint64_t* empty = is_k ? k_empty : v_empty;
        uint8_t* base = is_k ? sK : sV;
        const uint64_t pol = l2_policy_evict_last();     // K/V tiles are re-read by the head's other CTAs
        if (lane == 0) {
            tma_prefetch_desc(tm);
            if (is_k && wsub == 0 && n_loc > 0) {
                tma_prefetch_desc(&tm_q);
                mbar_arrive_expect_tx(q_full, kQTiles * C::kOpBytes);
#pragma unroll
                for (int g = 0; g < kQTiles; ++g)
#pragma unroll
                    for (int c = 0; c < C::kChunks; ++c)
                        tma_load_3d(sQ + g * C::kOpBytes + c * C::kChunkBytes, &tm_q, q_full, c * 64, h,
                                    q0 + g * kTile, pol);
            }
        }
        const int br = p.box_rows;
        const int64_t tbase = static_cast<int64_t>(b) * p.max_blocks;
        const int my_i = lane * kIssueWarps + wsub;      // this lane's box of every tile
        const int box = my_i / C::kChunks, chunk = my_i % C::kChunks;
        auto nbox_of = [&](int j) { return (min(kTile, kv_len - j * kTile) + br - 1) / br; };
        auto read_id = [&](int j) -> int {               // raw table entry; checked at use
            return (j < je && box < nbox_of(j)) ? p.block_tables[tbase + (j * kTile + box * br) / p.bs] : 0;
        };
        int last = -1;                                   // last ring slot (local tile index) this warp filled
        int bid = read_id(jb);
        for (int j = jb; j < je; ++j) {
            const int i = j - jb;                        // ring position
            const int st = i & 1;
            const int nbox = nbox_of(j);
            const int bid_next = read_id(j + 1);
            const int n_mine = (nbox * C::kChunks - wsub + kIssueWarps - 1) / kIssueWarps;
            const uint32_t bytes = static_cast<uint32_t>(n_mine * br * 128);
            if (!mbar_wait(&empty[st], ((i >> 1) & 1) ^ 1, p.wait_ns)) { abort_now(); break; }
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
            last = i;
            bid = bid_next;
        }
        if (!is_k && wsub == 0 && !info[2] && je == n_tiles && n_loc > 0) {
            // the last V tile: rows past the sequence end become zero before any P V reads them
            const int jl = n_tiles - 1, il = jl - jb;
            if (mbar_wait(&v_full[il & 1], (il >> 1) & 1, p.wait_ns)) {
                const int valid = kv_len - jl * kTile;                 // 1 .. 128
                const int units = (kTile - valid) * C::kChunks * 8;   // 16-byte units to clear
                const uint32_t vbase = smem_u32(sV + (il & 1) * C::kOpBytes);
                for (int u = lane; u < units; u += 32) {
                    const int row = valid + u / (C::kChunks * 8);
                    const int rem = u % (C::kChunks * 8);
                    st_shared_zero16(vbase + (rem >> 3) * C::kChunkBytes + row * 128 + (rem & 7) * 16);
                }
                fence_proxy_async_smem();                  // the zeros reach the tensor core's view
                __syncwarp();
                if (lane == 0) mbar_arrive(v_tail);
            } else {
                abort_now();
            }
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
            const int n0 = n_g[0], n1 = n_g[1];
            // This thread sets the pace of the tensor core (the MMA queue in front of it is short), so it
            // waits on each ring barrier once per tile, right before the first MMA that needs it, and a wait
            // on a phase that has already completed returns in ~15 cycles (mbar_wait tries the phase first).
            // i: the tile's ring position (its index among this CTA's key tiles)
            auto issue_s = [&](int g, int i) {
                const uint32_t d = tmem + C::kColS + g * kTile;
                const uint64_t dQg = umma_desc_advance(dQ, g * C::kOpBytes);
                const uint64_t dKs = umma_desc_advance(dK, (i & 1) * C::kOpBytes);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
                    umma_f16_ss(d, umma_desc_advance(dQg, off), umma_desc_advance(dKs, off), idesc_qk, kk > 0);
                }
                umma_commit(&s_full[g]);
            };
            auto issue_pv = [&](int g, int i) {
                // P_g of keys 16kk .. 16kk+15 is fp16 in columns 8kk .. 8kk+7 of the tile's S buffer
                const uint32_t o = tmem + C::kColO + g * D;
                const uint32_t pbase = tmem + C::kColS + g * kTile;
                const uint64_t dVs = umma_desc_advance(dV, (i & 1) * C::kOpBytes);
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk)
                    umma_f16_ts(o, pbase + kk * 8, umma_desc_advance(dVs, kk * 16 * 128), idesc_pv, i > 0 || kk > 0);
                umma_commit(&pv_done[g]);
            };
            bool ok = n_loc == 0 || (mbar_wait(q_full, 0, p.wait_ns) && mbar_wait(&k_full[0], 0, p.wait_ns));
            if (ok && n_loc > 0) {
                tc_fence_after_sync();
                if (jb < n0) issue_s(0, 0);
                if (jb < n1) issue_s(1, 0);
                umma_commit(&k_empty[0]);
            }
            for (int i = 0; ok && i < n_loc; ++i) {
                const int j = jb + i;                       // the key tile
                const int st = i & 1;
                const bool next = i + 1 < n_loc;
                // each ring barrier is waited on once per tile, right before the first MMA that needs it
                bool k_ready = !next, v_ready = false, tail_ready = j != n_tiles - 1;
                if (info[2]) { ok = false; break; }
#pragma unroll
                for (int g = 0; g < kQTiles; ++g) {
                    if (j >= je_g[g]) continue;
                    if (!(ok = mbar_wait(&p_full[g], i & 1, p.wait_ns))) break;
                    if (!v_ready && !(ok = mbar_wait(&v_full[st], (i >> 1) & 1, p.wait_ns))) break;
                    v_ready = true;
                    if (!tail_ready && !(ok = mbar_wait(v_tail, 0, p.wait_ns))) break;
                    tail_ready = true;
                    tc_fence_after_sync();
                    issue_pv(g, i);
                    if (j + 1 < je_g[g]) {
                        if (!k_ready && !(ok = mbar_wait(&k_full[(i + 1) & 1], ((i + 1) >> 1) & 1, p.wait_ns)))
                            break;
                        k_ready = true;
                        issue_s(g, i + 1);
                    }
                }
                if (!ok) break;
                umma_commit(&v_empty[st]);                  // every P V of tile j issued
                if (next) umma_commit(&k_empty[(i + 1) & 1]);   // every S of tile j+1 issued
            }
            if (!ok) abort_now();
            // every MMA this thread issued has completed before TMEM can be released
            umma_commit(drain);
            (void)mbar_wait(drain, 0);
        }
        __syncwarp();
    } else {
        // ======================================================= softmax warpgroups
        // Thread (warpgroup g, row r): row r of query tile g = TMEM lane r, all 128 key columns of S_g,
        // and row r of O_g.
        const int g = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const int cnt = je_g[g] - jb;                    // this tile's key tiles in this CTA
        const bool row_valid = r < rows_g[g];
        const int pos_first = ctx + row0 + g * kTile;   // position of the tile's first row
        const int row_pos = min(pos_first + r, kv_len - 1);
        const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const uint32_t s_addr = lane_base + C::kColS + g * kTile;
        const uint32_t o_addr = lane_base + C::kColO + g * D;
        const float qs = p.qscale;
        float m = -INFINITY, l = 0.f;                    // log2-domain running max and sum of the row
        // the warp's lanes agree on every wait's outcome, so the .sync.aligned TMEM accesses after it
        // are never reached by part of a warp
        auto warp_wait = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, p.wait_ns));
        };
        // failure-detection test: the wait runs out and the softmax role stops; the MMA issuer and the
        // producers then run out of their own waits and unwind
        bool ok = !p.stall || warp_wait(never, 0);
        for (int t = 0; t < cnt && ok; ++t) {            // t: the tile's index among this CTA's tiles
            const int j = jb + t;
            if (!(ok = warp_wait(&s_full[g], t & 1))) break;
            tc_fence_after_sync();
            const int key0 = j * kTile;
            const bool diag = key0 + kTile - 1 > pos_first;     // some key of the tile is masked for some row
            const int lim = row_pos - key0;                       // columns c <= lim are visible
            // all 128 scores of the row in registers (one TMEM round trip), masked on diagonal tiles
            uint32_t sc[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld_32cols_nowait(s_addr + 32 * c, sc[c]);
            tmem_wait_ld();
            if (diag) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (32 * c + i > lim) sc[c][i] = __float_as_uint(-INFINITY);
            }
            // the row max of the raw scores (scale > 0 keeps the order), three operands per instruction
            auto sf = [&](int k) { return __uint_as_float(sc[k >> 5][k & 31]); };
            float mx8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) mx8[k] = fmax3(sf(k), sf(k + 8), sf(k + 16));
#pragma unroll
            for (int k = 24; k < 128; k += 2) mx8[(k >> 1) & 7] = fmax3(mx8[(k >> 1) & 7], sf(k), sf(k + 1));
            const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                                   fmaxf(mx8[6], mx8[7])) * qs;
            float alpha = 1.f;
            const bool raise = mx > m + kRescaleLog2;            // false while both are -inf
            if (raise) {
                alpha = exp2f(m - mx);                           // 0 when m is still -inf
                m = mx;
            }
            const float m_use = m == -INFINITY ? 0.f : m;
            // P = 2^(s*qs - m) as fp16 pairs, over the first 64 columns of the S buffer (all of it is in
            // registers already).  The scaling runs in packed f32x2 arithmetic and every exponential on the
            // special-function unit: moving a share of them to the FMA pipe measured slower, as this loop is
            // bound by its dependency latencies rather than by either unit.  The row sum adds the fp16 values
            // of P that the P V MMA multiplies, so numerator and denominator round alike.
            const uint64_t qs2 = f32x2_pack(qs, qs), nm2 = f32x2_pack(-m_use, -m_use);
            float rs4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint64_t x = fma_f32x2(
                        f32x2_pack(__uint_as_float(sc[c][2 * i]), __uint_as_float(sc[c][2 * i + 1])), qs2, nm2);
                    float x0, x1;
                    f32x2_unpack(x, x0, x1);
                    pk[i] = f2_to_h2(exp2f(x0), exp2f(x1));
                    rs4[i & 3] = add_h2_f32(rs4[i & 3], pk[i]);
                }
                tmem_st_16cols_u(s_addr + 16 * c, pk);
            }
            l = fmaf(l, alpha, (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]));
            if (t > 0 && __any_sync(0xffffffffu, raise)) {
                // O_g holds the sum up to tile j-1: wait for that P V, then rescale this warp's rows
                if (!(ok = warp_wait(&pv_done[g], (t - 1) & 1))) break;
                tc_fence_after_sync();
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    float v[32];
                    tmem_ld_32cols(o_addr + c * 32, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] *= alpha;
                    tmem_st_32cols(o_addr + c * 32, v);
                }
            }
            tmem_wait_st();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[g]);
            if (info[2]) ok = false;
        }
        if (ok && cnt > 0) ok = warp_wait(&pv_done[g], (cnt - 1) & 1);   // the last P V has landed
        if (ok && cnt > 0) {
            tc_fence_after_sync();
            const float inv = 1.f / l;
            __half* orow = p.out + (static_cast<int64_t>(q0 + g * kTile + r) * p.H + h) * D;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t a[32];
                tmem_ld_32cols_nowait(o_addr + c * 32, a);
                tmem_wait_ld();
                if (row_valid) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 o;
                        uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i = 8 * q + 2 * e;
                            ow[e] = f2_to_h2(__uint_as_float(a[i]) * inv, __uint_as_float(a[i + 1]) * inv);
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
                        unsigned grid, cudaStream_t stream) {
    using C = PCfg<D>;
    static std::atomic<uint64_t> smem_set{0};          // devices whose limit is raised
    const cudaError_t attr_err = ensure_dynamic_smem(reinterpret_cast<const void*>(prefill_kernel<D>),
                                                     static_cast<int>(C::kSmemBytes), &smem_set);
    if (attr_err != cudaSuccess) return attr_err;
    prefill_kernel<D><<<grid, kThreadsP, C::kSmemBytes, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace

bool prefill_supported(int32_t H, int32_t D, int32_t bs) {
    return (D == 64 || D == 128) && H > 0 && H <= 65535 && bs >= 8 && bs % 8 == 0;
}

cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t stream, const char** why) {
    const uint64_t stall_ns = take_injected_stall(kStallPrefill);
    const uint64_t wait_ns = stall_ns ? stall_ns : kWaitLimitNs;
    // Too few (256-row query block, head) pairs to fill the GPU: the one-query-tile kernel, twice the CTAs
    // (PAGEDKV_PREFILL_SPLIT=0 in the environment keeps this kernel, for comparisons and tests).
    static const bool small_allowed = [] {
        const char* e = std::getenv("PAGEDKV_PREFILL_SPLIT");
        return !(e && e[0] == '0');
    }();
    const int64_t pairs = static_cast<int64_t>((a.num_tokens + kRowsPerCta - 1) / kRowsPerCta) * a.num_heads;
    if (small_allowed && 2 * pairs <= device_sm_count()) return launch_prefill_q128(a, wait_ns, stall_ns != 0, stream, why);

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
    // an upper bound of the query blocks: sum over requests of ceil(L_b / 256)
    p.grid_blocks = (a.num_tokens + kRowsPerCta - 1) / kRowsPerCta + a.num_reqs;
    p.box_rows = br;
    p.qscale = a.scale * kLog2eP;
    p.err_flag = a.err_flag;
    p.wait_ns = wait_ns;
    p.stall = stall_ns != 0;
    const uint64_t grid = static_cast<uint64_t>(p.grid_blocks) * a.num_heads;
    if (grid > 0x7fffffffull) {
        if (why) *why = "too many query blocks x heads for one launch";
        return cudaErrorInvalidValue;
    }
    const unsigned g = static_cast<unsigned>(grid);
    return a.head_dim == 128 ? run_prefill<128>(tq, tk, tv, p, g, stream) : run_prefill<64>(tq, tk, tv, p, g, stream);
}

}  // namespace pagedkv
