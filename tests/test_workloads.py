"""The seeded input recipe: shapes, pool sizes and block structure of every
named workload, determinism, and the rounding of the N(0, 1) samples to
fp16 / bf16 bits.  (The generators hold no arithmetic of the method; this
pins that they produce the workloads the measurements describe.)"""
import collections

import numpy as np
import pytest
import torch

import workloads
from workloads import BF16, F16

SHAPES = {
    #            B    Hq  Hkv  D   bs  dtype  NB
    "tiny":     (4,   4,  4,  64, 16, F16,  64),
    "llama13b": (32, 40, 40, 128, 16, F16,  4096 + 32),
    "llama70b_gqa": (30, 64, 8, 128, 16, BF16, 7782),
    "long_split": (2, 64, 8, 128, 16, BF16, 8192 + 2),
}


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_named_shapes_and_pools(name):
    w = workloads.make(name, fill_pool=False)
    b, hq, hkv, d, bs, dt, nb = SHAPES[name]
    sp = w.spec
    assert (sp.num_seqs, sp.num_q_heads, sp.num_kv_heads, sp.head_dim, sp.block_size, sp.dtype) == \
        (b, hq, hkv, d, bs, dt)
    assert w.num_blocks == nb and w.k_cache.shape == (nb, hkv, bs, d)
    assert w.q.shape == (b, hq, d) and w.k_new.shape == (b, hkv, d)
    assert w.scale == float(np.float32(1) / np.sqrt(np.float32(d)))
    want_ctx = {"tiny": [17, 33, 64, 100], "llama13b": [2048] * 32, "llama70b_gqa": [4096] * 30,
                "long_split": [65536] * 2}[name]
    assert list(w.context_lens) == want_ctx


def _check_structure(w):
    bs, nb = w.spec.block_size, w.num_blocks
    owners = collections.defaultdict(set)
    for s, c in enumerate(w.context_lens):
        n = -(-int(c) // bs)
        row = w.block_tables[s]
        assert (row[:n] >= 0).all() and (row[:n] < nb).all() and (row[n:] == -1).all()
        for i, blk in enumerate(row[:n]):
            owners[int(blk)].add((s, i))
    for blk, uses in owners.items():
        if len(uses) > 1:
            # only a group's shared prefix blocks alias, always at the same
            # logical index, never the block that receives the new token
            grp = {s // max(1, w.spec.share_group) for s, _ in uses}
            idx = {i for _, i in uses}
            assert w.spec.share_group and len(grp) == 1 and len(idx) == 1, blk
            for s, i in uses:
                assert i < w.shared_blocks[s]
                assert i < (int(w.context_lens[s]) - 1) // bs
    return owners


@pytest.mark.parametrize("name", ["tiny", "llama13b", "llama70b_gqa", "long_split"])
def test_private_pools_have_no_aliasing(name):
    w = workloads.make(name, fill_pool=False)
    owners = _check_structure(w)
    assert all(len(u) == 1 for u in owners.values())


def test_continuous_batching_sharing_rule():
    w = workloads.make("cb_mixed", fill_pool=False)
    sp = w.spec
    assert (sp.num_seqs, sp.num_q_heads, sp.num_kv_heads, sp.block_size, sp.share_group) == (256, 32, 8, 32, 16)
    c = w.context_lens.astype(int)
    assert c.min() >= 16 and c.max() <= 8192
    # log-uniform: the median sits near the geometric mean of the range
    assert 200 < np.median(c) < 1500
    _check_structure(w)
    for s in range(sp.num_seqs):
        k = min(2048 // 32, (int(c[s]) - 1) // 32)
        assert w.shared_blocks[s] == k
        lead = s - s % 16                       # every member shares the group's prefix ids
        kk = min(k, w.shared_blocks[lead])
        assert (w.block_tables[s, :kk] == w.block_tables[lead, :kk]).all()


def test_seeded_and_deterministic():
    a = workloads.make("tiny")
    b = workloads.make("tiny")
    for f in ("context_lens", "block_tables", "q", "k_cache", "v_cache", "k_new", "v_new"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f
    c = workloads.make("tiny", seed=123)
    assert not np.array_equal(a.q, c.q)


@pytest.mark.parametrize("dtype", [F16, BF16])
def test_samples_are_normal_values_rounded_to_nearest_even(dtype):
    rng = np.random.default_rng(7)
    x = rng.standard_normal(1 << 16).astype(np.float32)
    bits = workloads.to_bits(x, dtype)
    td = torch.float16 if dtype == F16 else torch.bfloat16
    ref = torch.from_numpy(x).to(td).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, ref)
    w = workloads.make(workloads.custom("dist", 8, 8, 8, 128, 16, dtype, 3, [512] * 8))
    v = torch.from_numpy(w.k_cache.view(np.int16)).view(td).float().numpy().ravel()
    assert abs(v.mean()) < 0.01 and abs(v.std() - 1) < 0.01
