"""Model-based stress test of the host block allocator: long seeded random
sequences of create / fork / fork-at-token / append / copy-on-write append /
batch appends / free, each checked against a plain Python model of the
tables and lengths.  After every operation: every block's refcount equals
the number of tables holding it, the free count is the pool minus the
blocks in use, appended slots follow the table, and failed operations
(out of blocks, write into a shared block) change nothing."""
import numpy as np
import pytest

import paged_kv_cache_437_b200 as pkv


class Model:
    def __init__(self, nb, bs):
        self.nb, self.bs = nb, bs
        self.tables, self.lens = {}, {}

    def refcounts(self):
        rc = np.zeros(self.nb, dtype=np.int64)
        for t in self.tables.values():
            for b in t:
                rc[b] += 1
        return rc

    def used(self):
        return int(np.count_nonzero(self.refcounts()))


def check(a, m):
    rc = m.refcounts()
    for b in range(m.nb):
        assert a.refcount(b) == rc[b], f"block {b}"
    assert a.num_free() == m.nb - m.used()
    for s, t in m.tables.items():
        assert [int(x) for x in a.block_table(s)] == t
        assert a.context_len(s) == m.lens[s]


def expect_append(a, m, s, cow):
    """Apply one append to the model from the allocator's answer; return the
    (src, dst) copy or None."""
    bs, n, t = m.bs, m.lens[s], m.tables[s]
    rc = m.refcounts()
    opens = n % bs == 0
    shared_last = (not opens) and rc[t[-1]] > 1
    free = m.nb - m.used()
    if opens or (shared_last and cow):
        if free == 0:
            return "oom"
    if shared_last and not cow:
        return "shared"
    return "ok"


@pytest.mark.parametrize("bs,seed", [(16, 0), (32, 1), (16, 2)])
def test_random_operation_sequences(bs, seed):
    rng = np.random.default_rng(seed)
    nb = 96
    a = pkv.BlockAllocator(nb, bs)
    m = Model(nb, bs)
    for step in range(2500):
        live = sorted(m.tables)
        op = rng.choice(["create", "fork", "fork_tokens", "append", "append_cow", "batch", "batch_cow", "free"],
                        p=[0.06, 0.05, 0.1, 0.28, 0.24, 0.07, 0.07, 0.13])
        if op == "create" or not live:
            s = a.seq_create()
            assert s not in m.tables
            m.tables[s], m.lens[s] = [], 0
        elif op == "fork":
            p = int(rng.choice(live))
            nfull = int(rng.integers(0, m.lens[p] // bs + 1))
            c = a.seq_fork(p, nfull)
            m.tables[c], m.lens[c] = list(m.tables[p][:nfull]), nfull * bs
        elif op == "fork_tokens":
            p = int(rng.choice(live))
            n = int(rng.integers(0, m.lens[p] + 1))
            c = a.seq_fork_tokens(p, n)
            m.tables[c], m.lens[c] = list(m.tables[p][:-(-n // bs)]), n
        elif op in ("append", "append_cow"):
            s = int(rng.choice(live))
            cow = op == "append_cow"
            want = expect_append(a, m, s, cow)
            before = (list(m.tables[s]), m.lens[s])
            try:
                if cow:
                    slot, src, dst = a.append_slot_cow(s)
                else:
                    slot, src, dst = a.append_slot(s), -1, -1
            except pkv.PkvError as e:
                assert want == "oom" and e.status == pkv.PKV_ERR_OOM or \
                    want == "shared" and e.status == pkv.PKV_ERR_SHARED_WRITE, (want, e.status)
                check(a, m)
                continue
            assert want == "ok", want
            t = [int(x) for x in a.block_table(s)]
            n = before[1]
            if n % bs == 0:
                assert t[:-1] == before[0] and m.refcounts()[t[-1]] == 0   # a free block opened
                assert (src, dst) == (-1, -1)
            elif src >= 0:
                assert src == before[0][-1] and t[:-1] == before[0][:-1] and t[-1] == dst
                assert m.refcounts()[dst] == 0 and m.refcounts()[src] > 1
            else:
                assert t == before[0]
            assert slot == t[n // bs] * bs + n % bs
            m.tables[s], m.lens[s] = t, n + 1
        elif op in ("batch", "batch_cow"):
            k = int(rng.integers(1, min(4, len(live)) + 1))
            seqs = [int(x) for x in rng.choice(live, size=k, replace=False)]
            snap = {s: (list(m.tables[s]), m.lens[s]) for s in seqs}
            try:
                if op == "batch_cow":
                    slots, copies = a.append_slots_cow(seqs)
                else:
                    slots, copies = a.append_slots(seqs), np.zeros((0, 2), np.int32)
            except pkv.PkvError as e:
                assert e.status in (pkv.PKV_ERR_OOM, pkv.PKV_ERR_SHARED_WRITE)
                check(a, m)                                # all or nothing
                continue
            for i, s in enumerate(seqs):
                t = [int(x) for x in a.block_table(s)]
                n = snap[s][1]
                assert slots[i] == t[n // bs] * bs + n % bs
                m.tables[s], m.lens[s] = t, n + 1
            for src, dst in np.asarray(copies).reshape(-1, 2):
                assert m.refcounts()[int(dst)] >= 1
        else:
            s = int(rng.choice(live))
            a.seq_free(s)
            del m.tables[s], m.lens[s]
        check(a, m)
    for s in list(m.tables):
        a.seq_free(s)
    assert a.num_free() == nb
