"""Iteration-level scheduler (host only): continuous batching with chunked
prefill and preemption under a KV budget."""
import numpy as np
import pytest

import oracle

import paged_kv_cache_437_b200 as pkv  # a missing library fails here, never skips


def run_to_completion(sched, alloc, max_steps=10_000, check_slots=True, on_step=None):
    tokens_in_cache = {}
    finish_step = {}
    steps = 0
    while (sched.num_waiting or sched.num_running) and steps < max_steps:
        b = sched.step()
        steps += 1
        for rid in b["finished"]:
            finish_step[int(rid)] = steps
        assert b["query_lens"].sum() == len(b["slots"])
        assert len(b["slots"]) <= sched.cfg.max_batch_tokens
        assert len(b["seq_ids"]) <= sched.cfg.max_seqs
        assert (b["query_lens"] >= 1).all() and (b["query_lens"] <= sched.cfg.chunk_tokens).all()
        if check_slots and len(b["seq_ids"]):
            tables, lens = alloc.batch_tables(b["seq_ids"], 4096)
            assert (lens == b["context_lens"]).all()
            t = 0
            for k, n in enumerate(b["query_lens"]):
                want = [oracle.slot_of(tables[k], p, alloc.block_size)
                        for p in range(lens[k] - n, lens[k])]
                assert list(b["slots"][t:t + n]) == want
                t += n
        for rid, n in zip(b["request_ids"], b["query_lens"]):
            tokens_in_cache[int(rid)] = tokens_in_cache.get(int(rid), 0) + int(n)
        for rid in b["preempted"]:
            tokens_in_cache[int(rid)] = 0
        if on_step:
            on_step(b)
    b = sched.step()                     # report what finished in the last step
    for rid in b["finished"]:
        finish_step[int(rid)] = steps + 1
    return steps, tokens_in_cache, finish_step


def test_chunked_prefill_decode_and_early_return():
    alloc = pkv.BlockAllocator(512, 16)
    sched = pkv.Scheduler(alloc, max_batch_tokens=600, max_seqs=8, chunk_tokens=512)
    reqs = {1: (40, 3), 2: (1200, 2), 3: (10, 5)}
    for rid, (p, m) in reqs.items():
        sched.add(rid, p, m)
    first = sched.step()
    assert list(first["request_ids"]) == [1, 2, 3][:len(first["request_ids"])]
    assert first["query_lens"][0] == 40 and first["query_lens"][1] == 512   # chunked prompt
    steps, in_cache, fin = run_to_completion(sched, alloc)
    # every request ends with prompt + (max_new - 1) tokens in the cache (the
    # last generated token is never appended)
    in_cache[1] += 40
    in_cache[2] += 512
    if len(first["request_ids"]) > 2:
        in_cache[3] += int(first["query_lens"][2])
    for rid, (p, m) in reqs.items():
        assert in_cache[rid] == p + m - 1, rid
    # no head-of-line blocking: the short requests are served from the first
    # step on, alongside the long prompt's chunks, and request 1 returns first;
    # request 3 needs exactly its own 5 steps: finished in global step 5,
    # reported by step 6 (finish steps here count from the second step)
    assert 3 in first["request_ids"]
    assert fin[1] < fin[2]
    assert fin[3] + 1 == 6
    assert alloc.num_free() == 512


def test_requests_join_mid_run():
    alloc = pkv.BlockAllocator(256, 16)
    sched = pkv.Scheduler(alloc, max_batch_tokens=256, max_seqs=16, chunk_tokens=128)
    sched.add(0, 100, 50)
    for _ in range(5):
        sched.step()
    sched.add(1, 20, 3)
    b = sched.step()
    assert 1 in b["request_ids"] and 0 in b["request_ids"]      # joins at once
    _, _, fin = run_to_completion(sched, alloc)
    assert fin[1] < fin[0]
    assert alloc.num_free() == 256


def test_preemption_under_kv_budget_conserves_blocks_and_finishes():
    alloc = pkv.BlockAllocator(12, 16)           # 192 tokens of KV in total
    sched = pkv.Scheduler(alloc, max_batch_tokens=256, max_seqs=8, chunk_tokens=64)
    rng = np.random.default_rng(1)
    reqs = {i: (int(rng.integers(20, 90)), int(rng.integers(20, 60))) for i in range(6)}
    for rid, (p, m) in reqs.items():
        sched.add(rid, p, m)
    preempted = []

    def on_step(b):
        preempted.extend(int(x) for x in b["preempted"])
        # blocks are conserved: free + owned by running sequences == pool
        owned = sum(len(alloc.block_table(int(s))) for s in b["seq_ids"])
        assert alloc.num_free() + owned <= 12

    steps, _, fin = run_to_completion(sched, alloc, on_step=on_step)
    assert sorted(fin) == sorted(reqs)
    assert preempted, "the pool is too small for all requests at once: someone must be preempted"
    assert alloc.num_free() == 12


def test_scheduler_argument_checks():
    alloc = pkv.BlockAllocator(8, 16)
    with pytest.raises(pkv.PkvError):
        pkv.Scheduler(alloc, max_batch_tokens=0, max_seqs=4)
    sched = pkv.Scheduler(alloc, max_batch_tokens=64, max_seqs=4)
    with pytest.raises(pkv.PkvError):
        sched.add(1, 0, 4)
    with pytest.raises(pkv.PkvError):
        sched.add(1, 4, 0)


@pytest.mark.parametrize("seed", range(6))
def test_random_configurations_run_to_completion(seed):
    """Random pools, budgets, chunk sizes and request mixes (some joining
    mid-run): every step respects its budgets with slots that follow the
    allocator's tables, every request ends with its prompt and all but its
    last generated token in the cache, and the pool ends empty."""
    rng = np.random.default_rng(100 + seed)
    bs = int(rng.choice([16, 32]))
    nb = int(rng.integers(16, 96))
    cap = nb * bs
    alloc = pkv.BlockAllocator(nb, bs)
    sched = pkv.Scheduler(alloc, max_batch_tokens=int(rng.integers(64, 1024)), max_seqs=int(rng.integers(2, 24)),
                          chunk_tokens=int(rng.choice([32, 64, 128, 512])))
    reqs = {}
    for rid in range(int(rng.integers(4, 40))):
        p = int(rng.integers(1, max(2, cap // 3)))
        m = int(rng.integers(1, max(2, min(64, cap - p))))
        reqs[rid] = (p, m)
    late = {rid for rid in reqs if rng.random() < 0.3}
    for rid, (p, m) in reqs.items():
        if rid not in late:
            sched.add(rid, p, m)
    seen_late = [False]

    def on_step(b):
        ids = [int(x) for x in b["request_ids"]]
        assert len(ids) == len(set(ids)), "a request twice in one step"
        if not seen_late[0]:
            seen_late[0] = True
            for rid in sorted(late):
                sched.add(rid, *reqs[rid])

    _, in_cache, fin = run_to_completion(sched, alloc, max_steps=20_000, on_step=on_step)
    assert sorted(fin) == sorted(reqs), "every request finishes"
    for rid, (p, m) in reqs.items():
        assert in_cache[rid] == p + m - 1, rid
    assert alloc.num_free() == nb
