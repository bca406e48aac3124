"""Host block allocator (free list, refcounts, sequences), CPU only.

Slot addresses are checked against the oracle's slot function and against
brute-force enumeration of each sequence's blocks."""
import numpy as np
import pytest

import oracle

import paged_kv_cache_437_b200 as pkv  # a missing library fails here, never skips


def test_alloc_until_oom_and_return():
    a = pkv.BlockAllocator(8, 16)
    got = [a.alloc() for _ in range(8)]
    assert sorted(got) == list(range(8))
    assert a.num_free() == 0
    with pytest.raises(pkv.PkvError) as e:
        a.alloc()
    assert e.value.status == pkv.PKV_ERR_OOM
    for b in got:
        assert a.refcount(b) == 1
        a.decref(b)
        assert a.refcount(b) == 0
    assert a.num_free() == 8


def test_refcounts_and_double_free():
    a = pkv.BlockAllocator(4, 16)
    b = a.alloc()
    a.incref(b)
    a.incref(b)
    assert a.refcount(b) == 3
    a.decref(b)
    a.decref(b)
    assert a.num_free() == 3
    a.decref(b)
    assert a.num_free() == 4 and a.refcount(b) == 0
    with pytest.raises(pkv.PkvError) as e:
        a.decref(b)
    assert e.value.status == pkv.PKV_ERR_INVALID
    with pytest.raises(pkv.PkvError):
        a.incref(b)
    assert a.refcount(-1) == -1 and a.refcount(4) == -1
    with pytest.raises(pkv.PkvError):
        a.decref(99)


@pytest.mark.parametrize("bs", [16, 32])
def test_append_slots_match_oracle_and_bruteforce(orc, bs):
    rng = np.random.default_rng(0)
    a = pkv.BlockAllocator(64, bs)
    seqs = [a.seq_create() for _ in range(3)]
    lengths = [5, 40, 70]
    slots = {s: [] for s in seqs}
    for step in range(max(lengths)):
        for s, n in zip(seqs, lengths):
            if step < n:
                slots[s].append(a.append_slot(s))
    for s, n in zip(seqs, lengths):
        table = a.block_table(s)
        assert len(table) == -(-n // bs)
        assert a.context_len(s) == n
        enum = []
        for blk in table:  # brute force: block by block, row by row
            enum.extend(int(blk) * bs + r for r in range(bs))
        assert slots[s] == enum[:n]
        assert slots[s] == [oracle.slot_of(table, p, bs, lib=orc) for p in range(n)]
    all_blocks = np.concatenate([a.block_table(s) for s in seqs])
    assert len(set(all_blocks.tolist())) == len(all_blocks)  # no block owned twice
    del rng


def test_seq_free_returns_blocks_at_once():
    a = pkv.BlockAllocator(10, 16)
    s = a.seq_create()
    for _ in range(33):
        a.append_slot(s)
    assert a.num_free() == 7
    a.seq_free(s)
    assert a.num_free() == 10
    with pytest.raises(pkv.PkvError):
        a.append_slot(s)
    s2 = a.seq_create()       # id reuse is allowed
    assert a.context_len(s2) == 0


def test_fork_shares_full_prefix_blocks():
    a = pkv.BlockAllocator(16, 16)
    p = a.seq_create()
    for _ in range(40):       # blocks: 16 + 16 + 8
        a.append_slot(p)
    parent_table = a.block_table(p)
    c = a.seq_fork(p, 2)
    assert list(a.block_table(c)) == list(parent_table[:2])
    assert a.context_len(c) == 32
    for b in parent_table[:2]:
        assert a.refcount(int(b)) == 2
    assert a.refcount(int(parent_table[2])) == 1
    slot = a.append_slot(c)   # opens a private block
    assert slot // 16 not in parent_table.tolist()
    assert a.refcount(slot // 16) == 1
    a.seq_free(p)
    for b in parent_table[:2]:
        assert a.refcount(int(b)) == 1
    assert a.refcount(int(parent_table[2])) == 0
    a.seq_free(c)
    assert a.num_free() == 16


def test_write_into_shared_block_is_refused_without_change():
    a = pkv.BlockAllocator(8, 16)
    p = a.seq_create()
    for _ in range(20):
        a.append_slot(p)
    c = a.seq_fork(p, 1)
    # make the parent's second block shared too, then try to write into it
    b1 = int(a.block_table(p)[1])
    a.incref(b1)
    free_before = a.num_free()
    with pytest.raises(pkv.PkvError) as e:
        a.append_slot(p)
    assert e.value.status == pkv.PKV_ERR_SHARED_WRITE
    assert a.context_len(p) == 20 and a.num_free() == free_before
    a.decref(b1)
    a.append_slot(p)
    assert a.context_len(p) == 21
    del c


def test_fork_argument_checks():
    a = pkv.BlockAllocator(8, 16)
    p = a.seq_create()
    for _ in range(20):
        a.append_slot(p)
    with pytest.raises(pkv.PkvError):
        a.seq_fork(p, 2)      # 32 > 20 tokens
    with pytest.raises(pkv.PkvError):
        a.seq_fork(p, -1)
    with pytest.raises(pkv.PkvError):
        a.seq_fork(77, 0)


def test_batch_append_is_all_or_nothing():
    a = pkv.BlockAllocator(3, 16)
    s = [a.seq_create() for _ in range(3)]
    a.append_slots(s)                      # 3 blocks used
    assert a.num_free() == 0
    for _ in range(15):
        a.append_slots(s)                  # fills every block
    before = [a.context_len(x) for x in s]
    with pytest.raises(pkv.PkvError) as e:
        a.append_slots(s)                  # needs 3 new blocks, none free
    assert e.value.status == pkv.PKV_ERR_OOM
    assert [a.context_len(x) for x in s] == before
    with pytest.raises(pkv.PkvError) as e:
        a.append_slots([s[0], s[0]])
    assert e.value.status == pkv.PKV_ERR_INVALID


def test_batch_tables():
    a = pkv.BlockAllocator(32, 16)
    s = [a.seq_create() for _ in range(3)]
    for n, x in zip([1, 17, 40], s):
        for _ in range(n):
            a.append_slot(x)
    tables, lens = a.batch_tables(s, 4)
    assert lens.tolist() == [1, 17, 40]
    for i, x in enumerate(s):
        t = a.block_table(x)
        assert tables[i, :len(t)].tolist() == t.tolist()
        assert (tables[i, len(t):] == -1).all()
    with pytest.raises(pkv.PkvError):
        a.batch_tables(s, 2)               # row too short for 3 blocks


def test_shuffled_free_list_via_public_api():
    """Draining then returning blocks in a chosen order makes later pops come
    out in the reverse of that order (LIFO), so a seeded permutation of the
    pool can be reproduced through the allocator alone."""
    a = pkv.BlockAllocator(20, 16)
    got = [a.alloc() for _ in range(20)]
    perm = np.random.default_rng(3).permutation(20)
    for b in perm[::-1]:
        a.decref(int(got[b]))
    again = [a.alloc() for _ in range(20)]
    assert again == [int(got[b]) for b in perm]


def test_fork_tokens_and_copy_on_write():
    a = pkv.BlockAllocator(8, 16)
    p = a.seq_create()
    for _ in range(20):                    # b0 full, b1 holds 4 tokens
        a.append_slot(p)
    b0, b1 = (int(x) for x in a.block_table(p))
    c = a.seq_fork_tokens(p, 20)
    assert list(a.block_table(c)) == [b0, b1] and a.context_len(c) == 20
    assert a.refcount(b0) == 2 and a.refcount(b1) == 2
    with pytest.raises(pkv.PkvError) as e:
        a.append_slot(c)                   # plain append refuses the shared block
    assert e.value.status == pkv.PKV_ERR_SHARED_WRITE
    slot, src, dst = a.append_slot_cow(c)
    assert src == b1 and dst not in (b0, b1)
    assert list(a.block_table(c)) == [b0, dst] and slot == dst * 16 + 4
    assert a.refcount(b1) == 1 and a.refcount(dst) == 1 and a.refcount(b0) == 2
    slot_p, src_p, dst_p = a.append_slot_cow(p)   # parent's b1 is private again
    assert (src_p, dst_p) == (-1, -1) and slot_p == b1 * 16 + 4
    slot_c2, src2, _ = a.append_slot_cow(c)
    assert src2 == -1 and slot_c2 == dst * 16 + 5
    a.seq_free(p)
    assert a.refcount(b0) == 1 and a.refcount(b1) == 0
    a.seq_free(c)
    assert a.num_free() == 8


def test_copy_on_write_oom_changes_nothing():
    a = pkv.BlockAllocator(2, 16)
    p = a.seq_create()
    for _ in range(5):
        a.append_slot(p)
    c = a.seq_fork_tokens(p, 5)
    a.alloc()                              # the last free block
    with pytest.raises(pkv.PkvError) as e:
        a.append_slot_cow(c)
    assert e.value.status == pkv.PKV_ERR_OOM
    assert a.context_len(c) == 5 and a.refcount(int(a.block_table(c)[0])) == 2


def test_batch_copy_on_write():
    a = pkv.BlockAllocator(16, 16)
    p = a.seq_create()
    for _ in range(30):
        a.append_slot(p)
    kids = [a.seq_fork_tokens(p, n) for n in (30, 16, 7)]
    slots, copies = a.append_slots_cow(kids)
    # forks at 30 and 7 land in shared partial blocks; the fork at 16 opens a new block
    assert len(copies) == 2
    tables = [a.block_table(k) for k in kids]
    assert slots[0] == tables[0][1] * 16 + 14 and slots[2] == tables[2][0] * 16 + 7
    assert slots[1] == tables[1][1] * 16 + 0
    srcs = sorted(int(x) for x in copies[:, 0])
    assert srcs == sorted(int(x) for x in a.block_table(p)[:2][::-1])
    full = pkv.BlockAllocator(3, 16)
    q = full.seq_create()
    for _ in range(20):
        full.append_slot(q)
    k1 = full.seq_fork_tokens(q, 20)
    k2 = full.seq_fork_tokens(q, 20)
    with pytest.raises(pkv.PkvError) as e:
        full.append_slots_cow([k1, k2])    # needs two fresh blocks, one is free
    assert e.value.status == pkv.PKV_ERR_OOM
    assert full.context_len(k1) == 20 and full.context_len(k2) == 20


def test_batch_prefix_groups():
    bs = 16
    a = pkv.BlockAllocator(64, bs)
    p1 = a.seq_create()
    for _ in range(3 * bs + 5):
        a.append_slot(p1)
    m1 = a.seq_fork(p1, 3)
    m2 = a.seq_fork(p1, 2)
    for _ in range(bs + 1):
        a.append_slot(m1)
        a.append_slot(m2)
    lone = a.seq_create()
    for _ in range(2 * bs):
        a.append_slot(lone)
    p2 = a.seq_create()
    for _ in range(bs):
        a.append_slot(p2)
    m3 = a.seq_fork(p2, 1)
    a.append_slot(m3)
    # groups: runs of consecutive sequences whose shared first block is one
    # and the same; `lone` shares nothing and stays in the run around it
    starts, shared = a.prefix_groups([p1, m1, m2, lone, m3, p2])
    assert starts.tolist() == [0, 4, 6]
    # claims: leading blocks with refcount > 1, times bs (p1's third block is
    # shared with m1 only; its fourth is private)
    assert shared.tolist() == [3 * bs, 3 * bs, 2 * bs, 0, bs, bs]
    # a sequence sharing nothing does not split a group
    starts, _ = a.prefix_groups([m1, lone, m2])
    assert starts.tolist() == [0, 3]
    # ... and joins the group after it when it comes first
    starts, _ = a.prefix_groups([lone, m3, p2])
    assert starts.tolist() == [0, 3]
    # a different shared first block opens a new group
    starts, _ = a.prefix_groups([m1, m3, m2])
    assert starts.tolist() == [0, 1, 2, 3]
    starts, _ = a.prefix_groups([lone])
    assert starts.tolist() == [0, 1]
    starts, shared = a.prefix_groups([])
    assert starts.tolist() == [0] and shared.size == 0
    with pytest.raises(pkv.PkvError):
        a.prefix_groups([p1, 999])
    a.close()
