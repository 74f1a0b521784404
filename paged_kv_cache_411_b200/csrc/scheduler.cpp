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
// The step's slot mapping lists the prefill rows (in prefill order) and then
// the decode rows.  pa_sched_complete then applies the step: chunks become
// cached, a request whose prefill completed emits a token, each decode emits
// a token, and a request that has emitted max_new_tokens finishes.
#include <cstdint>
#include <deque>
#include <new>
#include <unordered_map>
#include <vector>

#include "common.h"

using pagedkv::fail;

namespace {

enum : int32_t { kWaiting = 0, kRunning = 1, kFinished = 2 };

struct Req {
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
    pa_sched_config_t cfg{};
    int32_t block_size = 0;
    std::unordered_map<int64_t, Req> reqs;
    std::deque<int64_t> waiting;
    std::vector<int64_t> running;  // admission order
    std::vector<Entry> last_prefill, last_decode;
    bool step_open = false;
    int64_t steps = 0, preemptions = 0, finished = 0, prefill_tokens = 0, decode_tokens = 0;

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

pa_status pa_sched_add_request(pa_sched* s, int64_t req, int32_t prompt_len, int32_t max_new_tokens) {
    if (!s || prompt_len <= 0 || max_new_tokens <= 0)
        return fail(PA_ERR_INVALID_ARG, "pa_sched_add_request: prompt_len and max_new_tokens must be positive");
    if (s->reqs.count(req)) return fail(PA_ERR_EXISTS, "pa_sched_add_request: request %lld exists", (long long)req);
    int32_t dummy;
    if (pa_alloc_seq_len(s->alloc, req, &dummy) == PA_OK)
        return fail(PA_ERR_EXISTS, "pa_sched_add_request: request %lld already holds blocks", (long long)req);
    Req r;
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
        pa_alloc_free(s->alloc, v);
        q.to_prefill = q.prompt_len + q.generated;
        q.prefilled = 0;
        q.state = kWaiting;
        q.preemptions += 1;
        s->waiting.push_front(v);
        inf.num_preempted += 1;
        need = decode_need();
    }
    // 3. admit in arrival order while the prefill's blocks fit beside the decodes and the watermark
    while (static_cast<int32_t>(s->running.size()) < s->cfg.max_num_seqs && !s->waiting.empty()) {
        const int64_t r = s->waiting.front();
        Req& q = s->reqs[r];
        const int64_t blocks = (static_cast<int64_t>(q.to_prefill) + bs - 1) / bs;
        if (s->available() - need - s->cfg.watermark_blocks < blocks) break;
        s->waiting.pop_front();
        pa_status st = pa_alloc_allocate(s->alloc, r, 0);
        if (st != PA_OK) return st;
        q.state = kRunning;
        q.prefilled = 0;
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

pa_status pa_sched_complete(pa_sched* s) {
    if (!s || !s->step_open) return fail(PA_ERR_INVALID_ARG, "pa_sched_complete: no step to complete");
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
    return PA_OK;
}

}  // extern "C"
