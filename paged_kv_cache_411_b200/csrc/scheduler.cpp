// Iteration-level (continuous-batching) scheduler over the block allocator.
//
// The scheduler of the page "LLM 推理引擎 Continuous Batching 与
// PagedAttention" (§2.2 ContinuousBatchingScheduler.step / _build_batch),
// with chunked prefill (§4.3), block-watermark admission (§5.3) and
// preemption by recomputation (§5.4); [DB] §4.4 gives the same loop
// (accept -> allocate pages -> select prefill/decode -> run -> free).  One
// step, in this order:
//   1. requests that produced their last token are freed;
//   2. if the running decodes need more new blocks than are available, the
//      most recently admitted running request is preempted (its blocks freed,
//      it goes back to the FRONT of the waiting queue and will recompute its
//      prompt plus the tokens it generated), until they fit;
//   3. waiting requests are admitted in arrival order while the running set
//      is below max_num_seqs and the blocks of their whole prefill, plus the
//      decodes' needs, plus watermark_blocks, are available;
//   4. every fully prefilled running request decodes one token (its block is
//      guaranteed by 2); then, in running order, requests still prefilling get
//      a chunk of at most the remaining token budget (max_num_tokens); without
//      chunked prefill a prompt runs only whole.  A chunk that cannot get its
//      blocks waits for a later step.
// With a CPU pool attached (pa_sched_enable_swap), step 2 preempts by the
// page's second strategy instead (§5.4 "Swap to CPU" with §4.4's swap_out):
// the victim's blocks move to the CPU pool (pa_alloc_swap_out bookkeeping:
// CPU blocks allocated first, block i to block i, GPU blocks freed) and it
// waits, progress kept, in a swapped queue (most recently preempted first);
// a victim the CPU pool cannot take is recomputed.  Before admission,
// swapped requests come back in queue order while seats are free and the
// blocks of their table (plus one if their next decode opens a block), the
// decodes' needs and the watermark are available; no waiting request is
// admitted while one is still swapped.  The step reports the block moves
// (pa_sched_last_swaps), which the caller performs, swap-outs first, before
// the step's kernels.
// Requests added with their token ids (pa_sched_add_request_tokens) use the
// allocator's prefix cache (§4.2 inside the §2.2 loop): admission looks up
// the longest cached prefix of the ids known so far (prompt, then the
// generated ids pa_sched_complete_tokens reports), needs new blocks only for
// the rest (parked hits no longer count as available) and starts the request
// there with pa_alloc_begin_cached, so cached tokens are not prefilled again;
// the blocks its chunks and decodes fill are registered as they fill, and the
// generated ids go to the allocator as they are emitted, so decoded text
// becomes cacheable and a request recomputed after preemption finds its own
// blocks again.
// The step's slot mapping lists the prefill rows (in prefill order) and then
// the decode rows.  pa_sched_complete then applies the step: chunks become
// cached, a request whose prefill completed emits a token, each decode emits
// a token, and a request that has emitted max_new_tokens finishes.
#include <algorithm>
#include <cstdint>
#include <deque>
#include <new>
#include <unordered_map>
#include <vector>

#include "common.h"

using pagedkv::fail;

namespace {

enum : int32_t { kWaiting = 0, kRunning = 1, kFinished = 2, kSwapped = 3 };

struct Req {
    bool has_tokens = false;
    std::vector<int32_t> tokens;   // known ids: the prompt, then generated tokens as they are reported
    int32_t prompt_len = 0;
    int32_t max_new = 0;
    int32_t to_prefill = 0;        // tokens to prefill (prompt, plus generated tokens after a preemption)
    int32_t prefilled = 0;
    int32_t generated = 0;
    int32_t state = kWaiting;
    int64_t first_token_step = -1;
    int64_t finish_step = -1;
    int32_t preemptions = 0;
};

struct Entry {
    int64_t req;
    int32_t a, b;                  // prefill: (ctx_before, chunk); decode: (seq_len, 0)
};

}  // namespace

struct pa_sched {
    pa_alloc* alloc = nullptr;
    pa_alloc* cpu = nullptr;       // CPU pool for swap preemption (NULL: recompute)
    std::deque<int64_t> swapped;   // front = most recently preempted
    std::vector<int64_t> swap_out_pairs, swap_in_pairs;   // (src, dst) block pairs of the last step
    int64_t swap_outs = 0, swap_ins = 0;
    pa_sched_config_t cfg{};
    int32_t block_size = 0;
    std::unordered_map<int64_t, Req> reqs;
    std::deque<int64_t> waiting;
    std::vector<int64_t> running;  // admission order
    std::vector<Entry> last_prefill, last_decode;
    bool step_open = false;
    int64_t steps = 0, preemptions = 0, finished = 0, prefill_tokens = 0, decode_tokens = 0, cached_tokens = 0;

    int64_t available() const {
        int64_t n = 0;
        pa_alloc_available(alloc, &n);
        return n;
    }
    int32_t kv_len(int64_t r) const {
        int32_t n = 0;
        pa_alloc_seq_len(alloc, r, &n);
        return n;
    }
    bool decoding(const Req& q) const { return q.state == kRunning && q.prefilled == q.to_prefill && q.generated < q.max_new; }
    // the block table of r in allocator a (both pools hold ceil(seq_len / block_size) blocks)
    std::vector<int32_t> table(const pa_alloc* a, int64_t r) const {
        int32_t len = 0, n = 0;
        if (pa_alloc_seq_len(a, r, &len) != PA_OK) return {};
        std::vector<int32_t> t((len + block_size - 1) / block_size);
        if (pa_alloc_get_block_table(a, r, t.data(), static_cast<int32_t>(t.size()), &n) != PA_OK) return {};
        t.resize(n);
        return t;
    }
};

extern "C" {

pa_status pa_sched_create(pa_alloc* alloc, const pa_sched_config_t* cfg, pa_sched** out) {
    if (!out) return fail(PA_ERR_INVALID_ARG, "pa_sched_create: out is NULL");
    *out = nullptr;
    if (!alloc || !cfg || cfg->max_num_seqs <= 0 || cfg->max_num_tokens <= 0 || cfg->watermark_blocks < 0)
        return fail(PA_ERR_INVALID_ARG, "pa_sched_create: bad configuration");
    pa_alloc_stats_t s;
    pa_alloc_stats(alloc, &s);
    pa_sched* q = new (std::nothrow) pa_sched();
    if (!q) return fail(PA_ERR_OOM, "pa_sched_create: host allocation failed");
    q->alloc = alloc;
    q->cfg = *cfg;
    q->block_size = s.block_size;
    *out = q;
    return PA_OK;
}

void pa_sched_destroy(pa_sched* s) { delete s; }

pa_status pa_sched_enable_swap(pa_sched* s, pa_alloc* cpu) {
    if (!s) return fail(PA_ERR_INVALID_ARG, "pa_sched_enable_swap: NULL scheduler");
    if (s->step_open) return fail(PA_ERR_INVALID_ARG, "pa_sched_enable_swap: a step is open");
    if (!cpu) {
        if (!s->swapped.empty())
            return fail(PA_ERR_INVALID_ARG, "pa_sched_enable_swap: requests are still swapped out");
        s->cpu = nullptr;
        return PA_OK;
    }
    pa_alloc_stats_t st;
    pa_alloc_stats(cpu, &st);
    if (st.block_size != s->block_size)
        return fail(PA_ERR_INVALID_ARG, "pa_sched_enable_swap: CPU pool block size %d differs from %d",
                    st.block_size, s->block_size);
    s->cpu = cpu;
    return PA_OK;
}

pa_status pa_sched_last_swaps(const pa_sched* s, int64_t* out_pairs, int32_t out_cap, int32_t* n_out,
                              int64_t* in_pairs, int32_t in_cap, int32_t* n_in) {
    if (!s) return fail(PA_ERR_INVALID_ARG, "pa_sched_last_swaps: NULL scheduler");
    const int32_t no = static_cast<int32_t>(s->swap_out_pairs.size() / 2);
    const int32_t ni = static_cast<int32_t>(s->swap_in_pairs.size() / 2);
    if (n_out) *n_out = no;
    if (n_in) *n_in = ni;
    if ((out_pairs && out_cap < no) || (in_pairs && in_cap < ni))
        return fail(PA_ERR_INVALID_ARG, "pa_sched_last_swaps: capacity below %d / %d pairs", no, ni);
    for (size_t i = 0; out_pairs && i < s->swap_out_pairs.size(); ++i) out_pairs[i] = s->swap_out_pairs[i];
    for (size_t i = 0; in_pairs && i < s->swap_in_pairs.size(); ++i) in_pairs[i] = s->swap_in_pairs[i];
    return PA_OK;
}

static pa_status add_request(pa_sched* s, int64_t req, const int32_t* tokens, int32_t prompt_len,
                             int32_t max_new_tokens);

pa_status pa_sched_add_request(pa_sched* s, int64_t req, int32_t prompt_len, int32_t max_new_tokens) {
    return add_request(s, req, nullptr, prompt_len, max_new_tokens);
}

pa_status pa_sched_add_request_tokens(pa_sched* s, int64_t req, const int32_t* tokens, int32_t prompt_len,
                                      int32_t max_new_tokens) {
    if (!tokens) return fail(PA_ERR_INVALID_ARG, "pa_sched_add_request_tokens: tokens is NULL");
    return add_request(s, req, tokens, prompt_len, max_new_tokens);
}

static pa_status add_request(pa_sched* s, int64_t req, const int32_t* tokens, int32_t prompt_len,
                             int32_t max_new_tokens) {
    if (!s || prompt_len <= 0 || max_new_tokens <= 0)
        return fail(PA_ERR_INVALID_ARG, "pa_sched_add_request: prompt_len and max_new_tokens must be positive");
    if (s->reqs.count(req)) return fail(PA_ERR_EXISTS, "pa_sched_add_request: request %lld exists", (long long)req);
    int32_t dummy;
    if (pa_alloc_seq_len(s->alloc, req, &dummy) == PA_OK)
        return fail(PA_ERR_EXISTS, "pa_sched_add_request: request %lld already holds blocks", (long long)req);
    Req r;
    if (tokens) {
        r.has_tokens = true;
        r.tokens.assign(tokens, tokens + prompt_len);
    }
    r.prompt_len = prompt_len;
    r.max_new = max_new_tokens;
    r.to_prefill = prompt_len;
    s->reqs.emplace(req, r);
    s->waiting.push_back(req);
    return PA_OK;
}

pa_status pa_sched_step(pa_sched* s, pa_step_info_t* info, int64_t* prefill_reqs, int32_t* prefill_ctx,
                        int32_t* prefill_len, int64_t* decode_reqs, int32_t* decode_seq_lens,
                        int64_t* slot_mapping) {
    if (!s || !info) return fail(PA_ERR_INVALID_ARG, "pa_sched_step: NULL argument");
    if (s->step_open) return fail(PA_ERR_INVALID_ARG, "pa_sched_step: the previous step was not completed");
    pa_step_info_t inf{};
    const int32_t bs = s->block_size;
    s->swap_out_pairs.clear();
    s->swap_in_pairs.clear();
    // 1. free the requests that produced their last token
    std::vector<int64_t> keep;
    for (int64_t r : s->running) {
        Req& q = s->reqs[r];
        if (q.state == kFinished) {
            pa_alloc_free(s->alloc, r);
            inf.num_finished += 1;
        } else {
            keep.push_back(r);
        }
    }
    s->running.swap(keep);
    // 2. preempt the newest running requests until the decodes' new blocks fit
    auto decode_need = [&]() {
        int64_t need = 0;
        for (int64_t r : s->running)
            if (s->decoding(s->reqs[r]) && s->kv_len(r) % bs == 0) need += 1;
        return need;
    };
    int64_t need = decode_need();
    while (need > s->available() && !s->running.empty()) {
        const int64_t v = s->running.back();
        s->running.pop_back();
        Req& q = s->reqs[v];
        q.preemptions += 1;
        inf.num_preempted += 1;
        if (s->cpu) {
            const std::vector<int32_t> gt = s->table(s->alloc, v);
            if (pa_alloc_swap_out(s->alloc, s->cpu, v, nullptr, nullptr, nullptr, nullptr, 0, nullptr) == PA_OK) {
                const std::vector<int32_t> ct = s->table(s->cpu, v);
                for (size_t i = 0; i < gt.size(); ++i) {
                    s->swap_out_pairs.push_back(gt[i]);
                    s->swap_out_pairs.push_back(ct[i]);
                }
                q.state = kSwapped;
                s->swapped.push_front(v);
                s->swap_outs += 1;
                need = decode_need();
                continue;
            }
        }
        pa_alloc_free(s->alloc, v);
        q.to_prefill = q.prompt_len + q.generated;
        q.prefilled = 0;
        q.state = kWaiting;
        s->waiting.push_front(v);
        need = decode_need();
    }
    // swapped requests come back first, while seats and blocks last
    while (s->cpu && !s->swapped.empty() && static_cast<int32_t>(s->running.size()) < s->cfg.max_num_seqs) {
        const int64_t r = s->swapped.front();
        Req& q = s->reqs[r];
        const std::vector<int32_t> ct = s->table(s->cpu, r);
        int32_t len = 0;
        pa_alloc_seq_len(s->cpu, r, &len);
        const int64_t opens = (q.prefilled == q.to_prefill && q.generated < q.max_new && len % bs == 0) ? 1 : 0;
        if (s->available() - need - s->cfg.watermark_blocks < static_cast<int64_t>(ct.size()) + opens) break;
        s->swapped.pop_front();
        pa_status st = pa_alloc_swap_in(s->alloc, s->cpu, r, nullptr, nullptr, nullptr, nullptr, 0, nullptr);
        if (st != PA_OK) return st;
        const std::vector<int32_t> gt = s->table(s->alloc, r);
        for (size_t i = 0; i < ct.size(); ++i) {
            s->swap_in_pairs.push_back(ct[i]);
            s->swap_in_pairs.push_back(gt[i]);
        }
        q.state = kRunning;
        s->running.push_back(r);
        s->swap_ins += 1;
        need += opens;
    }
    // 3. admit in arrival order while the prefill's blocks fit beside the decodes and the watermark (not
    //    while a request is still swapped out)
    while (s->swapped.empty() && static_cast<int32_t>(s->running.size()) < s->cfg.max_num_seqs &&
           !s->waiting.empty()) {
        const int64_t r = s->waiting.front();
        Req& q = s->reqs[r];
        int32_t hits = 0, parked = 0;
        const int32_t known = q.has_tokens ? std::min<int32_t>(static_cast<int32_t>(q.tokens.size()), q.to_prefill) : 0;
        if (q.has_tokens) pa_alloc_cached_prefix(s->alloc, q.tokens.data(), known, &hits, &parked);
        const int64_t blocks = (static_cast<int64_t>(q.to_prefill) + bs - 1) / bs - hits;
        if (s->available() - parked - need - s->cfg.watermark_blocks < blocks) break;
        s->waiting.pop_front();
        q.prefilled = 0;
        pa_status st = q.has_tokens ? pa_alloc_begin_cached(s->alloc, r, q.tokens.data(), known, &q.prefilled)
                                    : pa_alloc_allocate(s->alloc, r, 0);
        if (st != PA_OK) return st;
        s->cached_tokens += q.prefilled;
        q.state = kRunning;
        s->running.push_back(r);
        inf.num_admitted += 1;
    }
    // 4. the batch: decodes (blocks guaranteed), then prefill chunks under the token budget
    s->last_prefill.clear();
    s->last_decode.clear();
    std::vector<int64_t> dec_slots, pre_slots;
    for (int64_t r : s->running) {
        if (!s->decoding(s->reqs[r])) continue;
        int64_t slot = -1;
        pa_status st = pa_alloc_append_token(s->alloc, r, &slot);
        if (st != PA_OK) return fail(PA_ERR_OOM, "pa_sched_step: decode append failed after preemption");
        dec_slots.push_back(slot);
        s->last_decode.push_back({r, s->kv_len(r), 0});
    }
    int32_t budget = s->cfg.max_num_tokens;
    for (int64_t r : s->running) {
        Req& q = s->reqs[r];
        if (q.state != kRunning || q.prefilled >= q.to_prefill) continue;
        const int32_t remaining = q.to_prefill - q.prefilled;
        int32_t chunk = s->cfg.chunked_prefill ? (remaining < budget ? remaining : budget)
                                               : (remaining <= budget ? remaining : 0);
        if (chunk <= 0) continue;
        const size_t at = pre_slots.size();
        pre_slots.resize(at + chunk);
        if (pa_alloc_append_tokens(s->alloc, r, chunk, pre_slots.data() + at) != PA_OK) {
            pre_slots.resize(at);           // no blocks for it this step
            continue;
        }
        s->last_prefill.push_back({r, q.prefilled, chunk});
        budget -= chunk;
    }
    inf.num_prefill = static_cast<int32_t>(s->last_prefill.size());
    inf.num_decode = static_cast<int32_t>(s->last_decode.size());
    inf.num_tokens = static_cast<int32_t>(pre_slots.size() + dec_slots.size());
    for (int32_t i = 0; i < inf.num_prefill; ++i) {
        if (prefill_reqs) prefill_reqs[i] = s->last_prefill[i].req;
        if (prefill_ctx) prefill_ctx[i] = s->last_prefill[i].a;
        if (prefill_len) prefill_len[i] = s->last_prefill[i].b;
    }
    for (int32_t i = 0; i < inf.num_decode; ++i) {
        if (decode_reqs) decode_reqs[i] = s->last_decode[i].req;
        if (decode_seq_lens) decode_seq_lens[i] = s->last_decode[i].a;
    }
    if (slot_mapping) {
        size_t k = 0;
        for (int64_t v : pre_slots) slot_mapping[k++] = v;
        for (int64_t v : dec_slots) slot_mapping[k++] = v;
    }
    inf.step = s->steps;
    s->step_open = true;
    *info = inf;
    return PA_OK;
}

static pa_status complete_step(pa_sched* s, bool with_ids, const int32_t* ids, int32_t n);

pa_status pa_sched_complete(pa_sched* s) { return complete_step(s, false, nullptr, 0); }

pa_status pa_sched_complete_tokens(pa_sched* s, const int32_t* ids, int32_t n) {
    if (n < 0 || (!ids && n > 0)) return fail(PA_ERR_INVALID_ARG, "pa_sched_complete_tokens: bad ids");
    return complete_step(s, true, ids, n);
}

static pa_status complete_step(pa_sched* s, bool with_ids, const int32_t* ids, int32_t n) {
    if (!s || !s->step_open) return fail(PA_ERR_INVALID_ARG, "pa_sched_complete: no step to complete");
    if (with_ids) {
        // one id per emitted token: requests whose prefill completes (prefill order), then the decodes
        std::vector<int64_t> emitting;
        for (const Entry& e : s->last_prefill)
            if (s->reqs[e.req].prefilled + e.b == s->reqs[e.req].to_prefill) emitting.push_back(e.req);
        for (const Entry& e : s->last_decode) emitting.push_back(e.req);
        if (static_cast<int32_t>(emitting.size()) != n)
            return fail(PA_ERR_INVALID_ARG, "pa_sched_complete_tokens: %d ids for %zu emitted tokens", n,
                        emitting.size());
        for (int32_t i = 0; i < n; ++i) {
            Req& q = s->reqs[emitting[i]];
            if (!q.has_tokens) continue;
            q.tokens.push_back(ids[i]);
            pa_alloc_extend_tokens(s->alloc, emitting[i], ids + i, 1);
        }
    }
    const int64_t now = s->steps;
    auto emit = [&](Req& q) {
        q.generated += 1;
        if (q.first_token_step < 0) q.first_token_step = now;
        if (q.generated >= q.max_new) {
            q.state = kFinished;
            q.finish_step = now;
            s->finished += 1;
        }
    };
    for (const Entry& e : s->last_prefill) {
        Req& q = s->reqs[e.req];
        q.prefilled += e.b;
        s->prefill_tokens += e.b;
        if (q.prefilled == q.to_prefill) emit(q);
    }
    for (const Entry& e : s->last_decode) {
        s->decode_tokens += 1;
        emit(s->reqs[e.req]);
    }
    s->steps += 1;
    s->step_open = false;
    return PA_OK;
}

pa_status pa_sched_request_info(const pa_sched* s, int64_t req, pa_request_info_t* out) {
    if (!s || !out) return fail(PA_ERR_INVALID_ARG, "pa_sched_request_info: NULL argument");
    auto it = s->reqs.find(req);
    if (it == s->reqs.end()) return fail(PA_ERR_NOT_FOUND, "pa_sched_request_info: request %lld not found", (long long)req);
    const Req& q = it->second;
    out->state = q.state;
    out->prompt_len = q.prompt_len;
    out->max_new_tokens = q.max_new;
    out->prefilled = q.prefilled;
    out->to_prefill = q.to_prefill;
    out->generated = q.generated;
    out->preemptions = q.preemptions;
    out->first_token_step = q.first_token_step;
    out->finish_step = q.finish_step;
    return PA_OK;
}

pa_status pa_sched_stats(const pa_sched* s, pa_sched_stats_t* out) {
    if (!s || !out) return fail(PA_ERR_INVALID_ARG, "pa_sched_stats: NULL argument");
    out->steps = s->steps;
    out->waiting = static_cast<int64_t>(s->waiting.size());
    out->running = static_cast<int64_t>(s->running.size());
    out->finished = s->finished;
    out->preemptions = 0;
    for (const auto& kv : s->reqs) out->preemptions += kv.second.preemptions;
    out->prefill_tokens = s->prefill_tokens;
    out->decode_tokens = s->decode_tokens;
    out->cached_tokens = s->cached_tokens;
    out->swapped = static_cast<int64_t>(s->swapped.size());
    out->swap_outs = s->swap_outs;
    out->swap_ins = s->swap_ins;
    return PA_OK;
}

}  // extern "C"
