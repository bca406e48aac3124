// Host block allocator for the paged KV pool.
//
// "LLM Inference: KV Cache, Batching & Scheduling" (cariara.com), section
// "PagedAttention and vLLM": KV is stored in fixed-size blocks, logical pages
// map to physical pages like OS virtual memory, pages are allocated on demand
// and a finished request's pages return to the pool at once.
// "LLM Inference Engineering: Overcoming the KV-Cache Bottleneck..."
// (adilsher.pro post, "The Elegant Fix: Paged Attention"): requests with the
// same prompt prefix share pages instead of duplicating them.
//
// Design: a LIFO free list of physical block ids, one reference count per
// block (0 = free), and per-sequence logical->physical tables.  Sharing a
// prefix is an incref of each shared block; a block returns to the free list
// when its count reaches 0.  pkv_seq_fork shares whole blocks only, and a
// plain append that would land in a shared block is refused
// (PKV_ERR_SHARED_WRITE); pkv_seq_fork_tokens may share a partly filled last
// block, and the copy-on-write appends give the writer a private copy (a
// fresh block plus a device block copy the caller makes).  Every operation
// either succeeds completely or leaves the state unchanged.
#include <cstdint>
#include <new>
#include <vector>

#include "pkv.h"

namespace {

struct Sequence {
    bool live = false;
    int64_t context_len = 0;
    std::vector<int32_t> blocks;  // logical order; size == ceil(len / bs)
};

struct Allocator {
    int32_t num_blocks = 0;
    int32_t block_size = 0;
    std::vector<int32_t> refcount;   // per physical block
    std::vector<int32_t> free_list;  // LIFO stack of free ids
    std::vector<Sequence> seqs;
    std::vector<int32_t> free_seq_ids;

    bool valid_block(int32_t b) const { return b >= 0 && b < num_blocks; }
    bool valid_seq(int32_t s) const {
        return s >= 0 && s < (int32_t)seqs.size() && seqs[s].live;
    }
    int32_t pop_block() {
        int32_t b = free_list.back();
        free_list.pop_back();
        refcount[b] = 1;
        return b;
    }
    void decref(int32_t b) {
        if (--refcount[b] == 0)
            free_list.push_back(b);
    }
    int32_t new_seq_id() {
        if (!free_seq_ids.empty()) {
            int32_t id = free_seq_ids.back();
            free_seq_ids.pop_back();
            return id;
        }
        seqs.emplace_back();
        return (int32_t)seqs.size() - 1;
    }
    // Does appending one token to seq s need a fresh block?  (len % bs == 0)
    bool needs_block(const Sequence &q) const { return q.context_len % block_size == 0; }
    // Would appending one token write into a shared block?
    bool writes_shared(const Sequence &q) const {
        if (needs_block(q))
            return false;
        int32_t b = q.blocks[q.context_len / block_size];
        return refcount[b] > 1;
    }
    int64_t append_one(Sequence &q) {
        int64_t logical = q.context_len / block_size;
        int64_t row = q.context_len % block_size;
        if (row == 0)
            q.blocks.push_back(pop_block());
        int64_t slot = (int64_t)q.blocks[logical] * block_size + row;
        q.context_len += 1;
        return slot;
    }
};

Allocator *as_alloc(void *h) { return static_cast<Allocator *>(h); }

}  // namespace

extern "C" {

pkv_status pkv_alloc_create(int32_t num_blocks, int32_t block_size, void **handle) {
    if (!handle || num_blocks <= 0 || block_size <= 0)
        return PKV_ERR_INVALID;
    Allocator *a = new (std::nothrow) Allocator();
    if (!a)
        return PKV_ERR_OOM;
    a->num_blocks = num_blocks;
    a->block_size = block_size;
    a->refcount.assign(num_blocks, 0);
    a->free_list.reserve(num_blocks);
    for (int32_t b = num_blocks - 1; b >= 0; --b)  // pops come out 0, 1, 2, ...
        a->free_list.push_back(b);
    *handle = a;
    return PKV_OK;
}

void pkv_alloc_destroy(void *handle) { delete as_alloc(handle); }

pkv_status pkv_block_alloc(void *h, int32_t *block_out) {
    Allocator *a = as_alloc(h);
    if (!a || !block_out)
        return PKV_ERR_INVALID;
    if (a->free_list.empty())
        return PKV_ERR_OOM;
    *block_out = a->pop_block();
    return PKV_OK;
}

pkv_status pkv_block_incref(void *h, int32_t block) {
    Allocator *a = as_alloc(h);
    if (!a || !a->valid_block(block) || a->refcount[block] <= 0)
        return PKV_ERR_INVALID;
    a->refcount[block] += 1;
    return PKV_OK;
}

pkv_status pkv_block_decref(void *h, int32_t block) {
    Allocator *a = as_alloc(h);
    if (!a || !a->valid_block(block) || a->refcount[block] <= 0)
        return PKV_ERR_INVALID;
    a->decref(block);
    return PKV_OK;
}

int32_t pkv_num_free(void *h) {
    Allocator *a = as_alloc(h);
    return a ? (int32_t)a->free_list.size() : -1;
}

int32_t pkv_refcount(void *h, int32_t block) {
    Allocator *a = as_alloc(h);
    if (!a || !a->valid_block(block))
        return -1;
    return a->refcount[block];
}

pkv_status pkv_seq_create(void *h, int32_t *seq_out) {
    Allocator *a = as_alloc(h);
    if (!a || !seq_out)
        return PKV_ERR_INVALID;
    int32_t id = a->new_seq_id();
    a->seqs[id] = Sequence();
    a->seqs[id].live = true;
    *seq_out = id;
    return PKV_OK;
}

pkv_status pkv_seq_fork(void *h, int32_t parent, int32_t num_full_blocks, int32_t *child_out) {
    Allocator *a = as_alloc(h);
    if (!a || !child_out || !a->valid_seq(parent) || num_full_blocks < 0)
        return PKV_ERR_INVALID;
    const Sequence &p = a->seqs[parent];
    if ((int64_t)num_full_blocks * a->block_size > p.context_len)
        return PKV_ERR_INVALID;
    std::vector<int32_t> shared(p.blocks.begin(), p.blocks.begin() + num_full_blocks);
    int32_t id = a->new_seq_id();  // may grow seqs: do not hold references into it
    Sequence &c = a->seqs[id];
    c = Sequence();
    c.live = true;
    c.blocks = shared;
    c.context_len = (int64_t)num_full_blocks * a->block_size;
    for (int32_t b : shared)
        a->refcount[b] += 1;
    *child_out = id;
    return PKV_OK;
}

pkv_status pkv_seq_append_slot(void *h, int32_t seq, int64_t *slot_out) {
    Allocator *a = as_alloc(h);
    if (!a || !slot_out || !a->valid_seq(seq))
        return PKV_ERR_INVALID;
    Sequence &q = a->seqs[seq];
    if (a->needs_block(q) && a->free_list.empty())
        return PKV_ERR_OOM;
    if (a->writes_shared(q))
        return PKV_ERR_SHARED_WRITE;
    *slot_out = a->append_one(q);
    return PKV_OK;
}

pkv_status pkv_seq_append_slots(void *h, const int32_t *seqs, int32_t n, int64_t *slots_out) {
    Allocator *a = as_alloc(h);
    if (!a || n < 0 || (n > 0 && (!seqs || !slots_out)))
        return PKV_ERR_INVALID;
    // validate everything first: all or nothing
    std::vector<char> seen(a->seqs.size(), 0);
    int64_t need = 0;
    for (int32_t i = 0; i < n; ++i) {
        int32_t s = seqs[i];
        if (!a->valid_seq(s) || seen[s])
            return PKV_ERR_INVALID;
        seen[s] = 1;
        const Sequence &q = a->seqs[s];
        if (a->needs_block(q))
            ++need;
        else if (a->writes_shared(q))
            return PKV_ERR_SHARED_WRITE;
    }
    if (need > (int64_t)a->free_list.size())
        return PKV_ERR_OOM;
    for (int32_t i = 0; i < n; ++i)
        slots_out[i] = a->append_one(a->seqs[seqs[i]]);
    return PKV_OK;
}

pkv_status pkv_seq_fork_tokens(void *h, int32_t parent, int64_t num_tokens, int32_t *child_out) {
    Allocator *a = as_alloc(h);
    if (!a || !child_out || !a->valid_seq(parent) || num_tokens < 0)
        return PKV_ERR_INVALID;
    const Sequence &p = a->seqs[parent];
    if (num_tokens > p.context_len)
        return PKV_ERR_INVALID;
    const int64_t nblk = (num_tokens + a->block_size - 1) / a->block_size;
    std::vector<int32_t> shared(p.blocks.begin(), p.blocks.begin() + nblk);
    int32_t id = a->new_seq_id();  // may grow seqs: do not hold references into it
    Sequence &c = a->seqs[id];
    c = Sequence();
    c.live = true;
    c.blocks = shared;
    c.context_len = num_tokens;
    for (int32_t b : shared)
        a->refcount[b] += 1;
    *child_out = id;
    return PKV_OK;
}

pkv_status pkv_seq_append_slot_cow(void *h, int32_t seq, int64_t *slot_out, int32_t *copy_src,
                                   int32_t *copy_dst) {
    Allocator *a = as_alloc(h);
    if (!a || !slot_out || !copy_src || !copy_dst || !a->valid_seq(seq))
        return PKV_ERR_INVALID;
    Sequence &q = a->seqs[seq];
    const bool shared = a->writes_shared(q);
    if ((a->needs_block(q) || shared) && a->free_list.empty())
        return PKV_ERR_OOM;
    *copy_src = *copy_dst = -1;
    if (shared) {
        // copy-on-write: a private block replaces the shared one
        const int64_t logical = q.context_len / a->block_size;
        const int32_t old = q.blocks[logical];
        const int32_t fresh = a->pop_block();
        a->decref(old);
        q.blocks[logical] = fresh;
        *copy_src = old;
        *copy_dst = fresh;
    }
    *slot_out = a->append_one(q);
    return PKV_OK;
}

pkv_status pkv_seq_append_slots_cow(void *h, const int32_t *seqs, int32_t n, int64_t *slots_out,
                                    int32_t *copies_out, int32_t *n_copies_out) {
    Allocator *a = as_alloc(h);
    if (!a || n < 0 || !n_copies_out || (n > 0 && (!seqs || !slots_out || !copies_out)))
        return PKV_ERR_INVALID;
    std::vector<char> seen(a->seqs.size(), 0);
    int64_t need = 0;
    for (int32_t i = 0; i < n; ++i) {
        int32_t s = seqs[i];
        if (!a->valid_seq(s) || seen[s])
            return PKV_ERR_INVALID;
        seen[s] = 1;
        const Sequence &q = a->seqs[s];
        if (a->needs_block(q) || a->writes_shared(q))
            ++need;
    }
    if (need > (int64_t)a->free_list.size())
        return PKV_ERR_OOM;
    int32_t nc = 0;
    for (int32_t i = 0; i < n; ++i) {
        int32_t src, dst;
        pkv_seq_append_slot_cow(h, seqs[i], &slots_out[i], &src, &dst);  // cannot fail now
        if (src >= 0) {
            copies_out[2 * nc] = src;
            copies_out[2 * nc + 1] = dst;
            ++nc;
        }
    }
    *n_copies_out = nc;
    return PKV_OK;
}

pkv_status pkv_seq_free(void *h, int32_t seq) {
    Allocator *a = as_alloc(h);
    if (!a || !a->valid_seq(seq))
        return PKV_ERR_INVALID;
    Sequence &q = a->seqs[seq];
    for (int32_t b : q.blocks)
        a->decref(b);
    q = Sequence();
    a->free_seq_ids.push_back(seq);
    return PKV_OK;
}

pkv_status pkv_seq_block_table(void *h, int32_t seq, int32_t *dst, int32_t cap, int32_t *n_out) {
    Allocator *a = as_alloc(h);
    if (!a || !a->valid_seq(seq) || cap < 0 || (cap > 0 && !dst))
        return PKV_ERR_INVALID;
    const Sequence &q = a->seqs[seq];
    int32_t n = (int32_t)q.blocks.size();
    for (int32_t i = 0; i < n && i < cap; ++i)
        dst[i] = q.blocks[i];
    if (n_out)
        *n_out = n;
    return PKV_OK;
}

int64_t pkv_seq_context_len(void *h, int32_t seq) {
    Allocator *a = as_alloc(h);
    if (!a || !a->valid_seq(seq))
        return -1;
    return a->seqs[seq].context_len;
}

pkv_status pkv_batch_tables(void *h, const int32_t *seqs, int32_t n, int32_t *dst, int32_t cap,
                            int32_t *context_lens) {
    Allocator *a = as_alloc(h);
    if (!a || n < 0 || cap <= 0 || (n > 0 && (!seqs || !dst || !context_lens)))
        return PKV_ERR_INVALID;
    for (int32_t i = 0; i < n; ++i) {
        if (!a->valid_seq(seqs[i]))
            return PKV_ERR_INVALID;
        if ((int64_t)a->seqs[seqs[i]].blocks.size() > cap)
            return PKV_ERR_INVALID;
    }
    for (int32_t i = 0; i < n; ++i) {
        const Sequence &q = a->seqs[seqs[i]];
        int32_t *row = dst + (int64_t)i * cap;
        int32_t k = 0;
        for (; k < (int32_t)q.blocks.size(); ++k)
            row[k] = q.blocks[k];
        for (; k < cap; ++k)
            row[k] = -1;
        context_lens[i] = (int32_t)q.context_len;
    }
    return PKV_OK;
}

pkv_status pkv_batch_prefix_groups(void *h, const int32_t *seqs, int32_t n, int32_t *group_start,
                                   int32_t *num_groups, int32_t *shared_lens) {
    Allocator *a = as_alloc(h);
    if (!a || n < 0 || !group_start || !num_groups || (n > 0 && (!seqs || !shared_lens)))
        return PKV_ERR_INVALID;
    for (int32_t i = 0; i < n; ++i)
        if (!a->valid_seq(seqs[i]))
            return PKV_ERR_INVALID;
    // A sequence that shares nothing joins the open group as a member with
    // claim 0 instead of splitting it: split groups would each read the
    // common prefix again.  A sequence whose first block is shared joins when
    // the open group has that first block, or none yet; otherwise it opens a
    // new group.
    int32_t ng = 0;
    int32_t group_first = -1;  // first block shared by the open group, -1: none yet
    for (int32_t i = 0; i < n; ++i) {
        const Sequence &q = a->seqs[seqs[i]];
        const int32_t first = q.blocks.empty() ? -1 : q.blocks[0];
        const bool shared_first = first >= 0 && a->refcount[first] > 1;
        if (i == 0 || (shared_first && group_first >= 0 && first != group_first)) {
            group_start[ng++] = i;
            group_first = -1;
        }
        if (shared_first)
            group_first = first;
        size_t k = 0;
        while (k < q.blocks.size() && a->refcount[q.blocks[k]] > 1)
            ++k;
        shared_lens[i] = (int32_t)(k * (size_t)a->block_size);
    }
    group_start[ng] = n;
    *num_groups = ng;
    return PKV_OK;
}

const char *pkv_status_string(pkv_status s) {
    switch (s) {
    case PKV_OK: return "ok";
    case PKV_ERR_INVALID: return "invalid argument";
    case PKV_ERR_OOM: return "out of KV blocks";
    case PKV_ERR_CUDA: return "CUDA error";
    case PKV_ERR_SHARED_WRITE: return "write into a shared block";
    case PKV_ERR_DEVICE_CHECK: return "device-side index check failed";
    case PKV_ERR_TIMEOUT: return "device wait timed out";
    case PKV_ERR_SCRATCH_TOO_SMALL: return "shape needs more than the static scratch";
    }
    return "unknown status";
}

}  // extern "C"
