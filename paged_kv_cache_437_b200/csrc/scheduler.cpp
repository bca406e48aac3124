// Iteration-level (continuous-batching) scheduler on top of the block
// allocator.  Host code only.
//
// "LLM Inference: KV Cache, Batching & Scheduling" (cariara.com):
//   * "Continuous batching (Orca)": every token step is batched across all
//     in-flight requests; finished requests leave and new ones join at any
//     step, so short requests return right away (no head-of-line blocking);
//   * "Chunked prefill": a long prompt is fed in fixed-size chunks (e.g. 512
//     tokens) interleaved with the other requests' decode steps;
//   * "The KV cache" (warning): running out of KV memory stalls new requests
//     or forces preemption of in-flight ones.
//
// Policy (the plainest reading): decode steps of running requests first (one
// token each, oldest first), then the next prefill chunk of requests still in
// their prompt, then new requests first-come-first-served, all within a token
// budget per step and a cap on the batch's sequences.  A request needing a
// new block when none is free preempts the most recently admitted running
// request (recompute: its blocks return to the pool and it goes back to the
// front of the queue; its prompt and the tokens it had generated are
// prefilled again when readmitted -- at the next step at the earliest, so
// that the blocks its preemption freed go to the request that needed them).  Every sequence's slots come from the
// allocator, so the block tables handed to the kernels are exactly its own.
#include <algorithm>
#include <cstdint>
#include <deque>
#include <new>
#include <vector>

#include "pkv.h"

namespace {

struct Request {
    int64_t id = 0;
    int32_t prompt_len = 0;
    int32_t max_new_tokens = 0;
    int32_t generated = 0;  // tokens produced so far
    int32_t seq = -1;       // allocator sequence while running
    int32_t prefilled = 0;  // tokens of (prompt + generated) already in the cache
    int64_t admit_order = 0;
    // tokens that must be in the cache before the next decode token
    int32_t target() const { return prompt_len + generated; }
};

struct Scheduler {
    void *alloc = nullptr;
    pkv_sched_config cfg{};
    std::deque<Request> waiting;
    std::vector<Request> running;
    std::vector<int64_t> finished_pending;
    int64_t admit_counter = 0;
};

Scheduler *as_sched(void *h) { return static_cast<Scheduler *>(h); }

// Blocks needed to grow a sequence of length len by n tokens.
int64_t blocks_needed(int64_t len, int64_t n, int64_t bs) {
    const int64_t have = (len + bs - 1) / bs;
    const int64_t want = (len + n + bs - 1) / bs;
    return want - have;
}

}  // namespace

extern "C" {

pkv_status pkv_sched_create(void *alloc, const pkv_sched_config *cfg, void **sched) {
    if (!alloc || !cfg || !sched || cfg->max_batch_tokens <= 0 || cfg->max_seqs <= 0 ||
        cfg->chunk_tokens <= 0 || cfg->block_size <= 0)
        return PKV_ERR_INVALID;
    Scheduler *s = new (std::nothrow) Scheduler();
    if (!s)
        return PKV_ERR_OOM;
    s->alloc = alloc;
    s->cfg = *cfg;
    *sched = s;
    return PKV_OK;
}

void pkv_sched_destroy(void *sched) {
    Scheduler *s = as_sched(sched);
    if (!s)
        return;
    for (Request &r : s->running)
        if (r.seq >= 0)
            pkv_seq_free(s->alloc, r.seq);
    delete s;
}

pkv_status pkv_sched_add(void *sched, int64_t request_id, int32_t prompt_len, int32_t max_new_tokens) {
    Scheduler *s = as_sched(sched);
    if (!s || prompt_len <= 0 || max_new_tokens <= 0)
        return PKV_ERR_INVALID;
    Request r;
    r.id = request_id;
    r.prompt_len = prompt_len;
    r.max_new_tokens = max_new_tokens;
    s->waiting.push_back(r);
    return PKV_OK;
}

int32_t pkv_sched_num_waiting(void *sched) {
    Scheduler *s = as_sched(sched);
    return s ? (int32_t)s->waiting.size() : -1;
}

int32_t pkv_sched_num_running(void *sched) {
    Scheduler *s = as_sched(sched);
    return s ? (int32_t)s->running.size() : -1;
}

pkv_status pkv_sched_step(void *sched, pkv_sched_batch *out) {
    Scheduler *s = as_sched(sched);
    if (!s || !out || !out->request_ids || !out->seq_ids || !out->query_lens || !out->context_lens ||
        !out->slots || !out->finished_ids || !out->preempted_ids)
        return PKV_ERR_INVALID;
    const int64_t bs = s->cfg.block_size;
    out->num_seqs = 0;
    out->num_tokens = 0;
    out->num_preempted = 0;
    out->num_finished = 0;

    // Requests that produced their last token in the previous step leave
    // now; their pages return to the pool at once.  (They stay valid until
    // this call: the previous step's kernels still read them.)
    for (int64_t id : s->finished_pending) {
        for (size_t i = 0; i < s->running.size(); ++i) {
            if (s->running[i].id == id) {
                pkv_seq_free(s->alloc, s->running[i].seq);
                s->running.erase(s->running.begin() + i);
                break;
            }
        }
        if (out->num_finished < s->cfg.max_seqs)
            out->finished_ids[out->num_finished++] = id;
    }
    s->finished_pending.clear();

    std::sort(s->running.begin(), s->running.end(),
              [](const Request &x, const Request &y) { return x.admit_order < y.admit_order; });

    struct Entry {
        size_t idx;
        int32_t n;
        int64_t need;  // blocks reserved
    };
    std::vector<Entry> plan;
    std::vector<char> in_plan(s->running.size(), 0);
    int64_t reserved = 0;
    int32_t budget = s->cfg.max_batch_tokens;
    auto free_avail = [&]() { return (int64_t)pkv_num_free(s->alloc) - reserved; };

    // preempt running request v (recompute): its blocks go back to the pool,
    // it goes back to the front of the queue
    bool preempted_now = false;  // the queue's front was preempted in this step
    auto preempt = [&](size_t v) {
        for (size_t e = 0; e < plan.size(); ++e) {
            if (plan[e].idx == v) {
                reserved -= plan[e].need;
                budget += plan[e].n;
                plan.erase(plan.begin() + e);
                break;
            }
        }
        for (Entry &e : plan)
            if (e.idx > v)
                --e.idx;
        Request r = s->running[v];
        pkv_seq_free(s->alloc, r.seq);
        r.seq = -1;
        r.prefilled = 0;
        s->running.erase(s->running.begin() + v);
        in_plan.erase(in_plan.begin() + v);
        s->waiting.push_front(r);
        preempted_now = true;
        if (out->num_preempted < s->cfg.max_seqs)
            out->preempted_ids[out->num_preempted++] = r.id;
    };

    // 1) one decode token per decoding request, then 2) the next prefill
    // chunk of requests still in their context, oldest first
    for (int phase = 0; phase < 2; ++phase) {
        for (size_t i = 0; i < s->running.size(); ++i) {
            if ((int32_t)plan.size() >= s->cfg.max_seqs || budget <= 0)
                break;
            const Request &r = s->running[i];
            const bool decoding = r.prefilled >= r.target();
            if ((phase == 0) != decoding || in_plan[i])
                continue;
            const int32_t n = decoding ? 1 : std::min({r.target() - r.prefilled, s->cfg.chunk_tokens, budget});
            const int64_t need = blocks_needed(pkv_seq_context_len(s->alloc, r.seq), n, bs);
            while (need > free_avail()) {
                // out of KV memory: preempt the newest other running request
                size_t v = s->running.size();
                for (size_t j = 0; j < s->running.size(); ++j)
                    if (j != i && (v == s->running.size() ||
                                   s->running[j].admit_order > s->running[v].admit_order))
                        v = j;
                if (v == s->running.size())
                    break;
                preempt(v);
                if (v < i)
                    --i;
            }
            if (need > free_avail())
                continue;  // nothing left to preempt: this request waits
            plan.push_back(Entry{i, n, need});
            in_plan[i] = 1;
            reserved += need;
            budget -= n;
        }
    }

    // 3) admit waiting requests, first come first served; KV memory that is
    // not there stalls them, and so does a request preempted in this step
    // (now at the front of the queue)
    while (!preempted_now && !s->waiting.empty() && budget > 0 && (int32_t)plan.size() < s->cfg.max_seqs &&
           (int32_t)s->running.size() < s->cfg.max_seqs) {
        Request a = s->waiting.front();
        const int32_t n = std::min({a.target(), s->cfg.chunk_tokens, budget});
        const int64_t need = blocks_needed(0, n, bs);
        if (need > free_avail())
            break;
        if (pkv_seq_create(s->alloc, &a.seq) != PKV_OK)
            return PKV_ERR_INVALID;
        s->waiting.pop_front();
        a.admit_order = ++s->admit_counter;
        a.prefilled = 0;
        s->running.push_back(a);
        in_plan.push_back(1);
        plan.push_back(Entry{s->running.size() - 1, n, need});
        reserved += need;
        budget -= n;
    }

    // emit the batch: per sequence its query tokens and, in the same order,
    // the slots of all new tokens
    int32_t k = 0, t = 0;
    for (const Entry &e : plan) {
        Request &r = s->running[e.idx];
        for (int32_t j = 0; j < e.n; ++j)
            if (pkv_seq_append_slot(s->alloc, r.seq, &out->slots[t + j]) != PKV_OK)
                return PKV_ERR_OOM;  // cannot happen: the blocks were reserved
        out->request_ids[k] = r.id;
        out->seq_ids[k] = r.seq;
        out->query_lens[k] = e.n;
        out->context_lens[k] = (int32_t)pkv_seq_context_len(s->alloc, r.seq);
        t += e.n;
        ++k;
        r.prefilled += e.n;
        if (r.prefilled >= r.target()) {
            // the step that completes the context produces the next token
            r.generated += 1;
            if (r.generated >= r.max_new_tokens)
                s->finished_pending.push_back(r.id);
        }
    }
    out->num_seqs = k;
    out->num_tokens = t;
    return PKV_OK;
}

}  // extern "C"
