"""Decode steps whose sharing groups read their common prefix once
(pkv_append_decode_attention_shared_prefix) against the fp64 oracle.

The result must be the plain decode attention of every sequence over its
whole context: the oracle knows nothing about groups.  Every slot outside
the attended context is NaN-poisoned; the appended pool is compared bit for
bit.  Claims that overstate the sharing, groups whose members share nothing,
groups of one and zero groups must all give the same exact result."""
import numpy as np
import pytest
import torch

import gpu_harness as gh
import paged_kv_cache_437_b200 as pkv
import workloads
from workloads import BF16, F16, custom

pytestmark = pytest.mark.gpu

SPECS = [
    # groups of 8 sharing up to 512 tokens (16 blocks of 32); lengths around
    # every edge: one block, a block + 1, exactly the prefix, far past it
    custom("cas_f16", 24, 32, 8, 128, 32, F16, 61,
           [1, 31, 32, 33, 64, 500, 513, 514, 2000, 700, 96, 4000,
            513, 1, 2, 900, 1500, 33, 65, 512, 3000, 600, 300, 128],
           share_group=8, share_prefix_tokens=512),
    custom("cas_bf16", 12, 64, 8, 128, 16, BF16, 62,
           [300, 4096, 17, 257, 1024, 16, 2049, 129, 5000, 260, 258, 1],
           share_group=4, share_prefix_tokens=256),
    custom("cas_mha64", 9, 4, 4, 64, 16, F16, 63, [40, 41, 300, 7, 90, 200, 48, 49, 50],
           share_group=3, share_prefix_tokens=48),
    custom("cas_g16", 6, 32, 2, 128, 16, BF16, 64, [1000, 800, 300, 2000, 150, 40],
           share_group=6, share_prefix_tokens=1024),
]


def _groups_of(w):
    """group_start and claimed shared lengths straight from the workload's
    structure (groups of share_group consecutive sequences)."""
    sp = w.spec
    b = sp.num_seqs
    starts = np.arange(0, b, sp.share_group).tolist() + [b]
    claims = np.array(w.shared_blocks, dtype=np.int32) * sp.block_size
    return np.array(starts, dtype=np.int32), claims


def _run(w, kc, vc, slots, starts, claims, append=True):
    step = gh.GpuStep(w, kc, vc, slots)
    sp = w.spec
    n = pkv.pkv_shared_prefix_workspace_bytes(sp.num_seqs, sp.num_q_heads, sp.num_kv_heads, sp.head_dim,
                                              w.max_blocks_per_seq * sp.block_size, len(starts) - 1)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    step.out.fill_(float("nan"))
    gs = torch.from_numpy(np.ascontiguousarray(starts, dtype=np.int32)).cuda()
    cl = torch.from_numpy(np.ascontiguousarray(claims, dtype=np.int32)).cuda()
    if append:
        pkv.pkv_append_decode_attention_shared_prefix(step.kn, step.vn, step.slots, step.q, step.kc, step.vc,
                                                      step.tables, step.lens, gs, cl, w.scale, step.out, ws)
    else:
        step.append()
        pkv.pkv_append_decode_attention_shared_prefix(None, None, None, step.q, step.kc, step.vc, step.tables,
                                                      step.lens, gs, cl, w.scale, step.out, ws)
    torch.cuda.synchronize()
    st = pkv.pkv_get_last_error()
    assert st == pkv.PKV_OK, pkv.pkv_status_string(st)
    return step


@pytest.mark.parametrize("append", [True, False], ids=["fused_append", "append_first"])
@pytest.mark.parametrize("spec", SPECS, ids=lambda s: s.name)
def test_shared_prefix_matches_oracle(spec, append):
    w = workloads.make(spec)
    kc, vc, slots = gh.prepare(w)
    ref, k_ref, v_ref = gh.oracle_step(w, kc, vc, slots)
    starts, claims = _groups_of(w)
    step = _run(w, kc, vc, slots, starts, claims, append)
    assert np.array_equal(gh.host_bits(step.kc), k_ref) and np.array_equal(gh.host_bits(step.vc), v_ref)
    gh.assert_close(gh.to_f64(step.out), ref, spec.dtype, f"shared prefix {spec.name}")


def test_continuous_batching_step_full_size():
    # the continuous-batching workload at full size (256 sequences, groups of
    # 16 sharing a 2048-token prefix) through the shared-prefix call, as the
    # benchmark runs it: pools bit for bit, 256 sampled (sequence, head) rows
    w = workloads.make("cb_mixed")
    kc, vc, slots = gh.prepare(w)
    pairs = gh.sample_pairs(w, 256)
    ref, k_ref, v_ref = gh.oracle_step(w, kc, vc, slots, pairs=pairs)
    starts, claims = _groups_of(w)
    step = _run(w, kc, vc, slots, starts, claims, append=True)
    assert np.array_equal(gh.host_bits(step.kc), k_ref) and np.array_equal(gh.host_bits(step.vc), v_ref)
    got = gh.to_f64(step.out)
    assert np.all(np.isfinite(got))
    gh.assert_close(got[pairs[:, 0], pairs[:, 1]], ref, w.spec.dtype, "cb_mixed, shared-prefix call")


def test_groups_from_the_allocator():
    spec = SPECS[0]
    w = workloads.make(spec)
    kc, vc, slots = gh.prepare(w)
    ref, _, _ = gh.oracle_step(w, kc, vc, slots)
    sp = w.spec
    # rebuild the tables through the host allocator: holders own the group
    # prefixes, members fork them (refcounted sharing) and grow privately
    alloc = pkv.BlockAllocator(w.num_blocks + 64, sp.block_size)
    holders, seqs = {}, []
    for s in range(sp.num_seqs):
        g = s // sp.share_group
        holders[g] = max(holders.get(g, 0), w.shared_blocks[s])
    for g in sorted(holders):
        h = alloc.seq_create()
        for _ in range(holders[g] * sp.block_size):
            alloc.append_slot(h)
        holders[g] = h
    for s in range(sp.num_seqs):
        seq = alloc.seq_fork(holders[s // sp.share_group], w.shared_blocks[s])
        while alloc.context_len(seq) < int(w.context_lens[s]):
            alloc.append_slot(seq)
        seqs.append(seq)
    starts, claims = alloc.prefix_groups(seqs)
    tables, lens = alloc.batch_tables(seqs, w.max_blocks_per_seq)
    alloc.close()
    # the allocator's claims are the workload's; its groups are runs of one
    # shared first block, with sequences that share nothing kept inside them
    assert np.array_equal(lens, w.context_lens)
    assert starts[0] == 0 and starts[-1] == sp.num_seqs and np.all(np.diff(starts) > 0)
    for s in range(sp.num_seqs):
        assert claims[s] == w.shared_blocks[s] * sp.block_size
    # same attention on the allocator's own block ids: permute the pool into them
    k2 = np.zeros((alloc.num_blocks,) + kc.shape[1:], dtype=kc.dtype)
    v2 = np.zeros_like(k2)
    for s in range(sp.num_seqs):
        n = -(-int(w.context_lens[s]) // sp.block_size)
        k2[tables[s, :n]] = kc[w.block_tables[s, :n]]
        v2[tables[s, :n]] = vc[w.block_tables[s, :n]]
    w2 = workloads.Workload(sp, w.context_lens, tables, alloc.num_blocks, None, w.shared_blocks, w.q, k2, v2,
                            w.k_new, w.v_new, w.scale)
    slots2 = np.array([tables[s, (int(w.context_lens[s]) - 1) // sp.block_size] * sp.block_size +
                       (int(w.context_lens[s]) - 1) % sp.block_size for s in range(sp.num_seqs)], dtype=np.int64)
    step = _run(w2, k2, v2, slots2, starts, claims, append=True)
    gh.assert_close(gh.to_f64(step.out), ref, spec.dtype, "shared prefix, allocator groups")


def test_overstated_claims_and_unrelated_groups_stay_exact():
    spec = SPECS[1]
    w = workloads.make(spec)
    kc, vc, slots = gh.prepare(w)
    ref, _, _ = gh.oracle_step(w, kc, vc, slots)
    b = spec.num_seqs
    huge = np.full(b, 1 << 20, dtype=np.int32)
    # the right groups with claims far past what is shared
    starts, _ = _groups_of(w)
    gh.assert_close(gh.to_f64(_run(w, kc, vc, slots, starts, huge).out), ref, spec.dtype, "overstated claims")
    # groups that straddle the real ones (members of different prefixes)
    odd = np.array([0, 3, 5, 11, b], dtype=np.int32)
    gh.assert_close(gh.to_f64(_run(w, kc, vc, slots, odd, huge).out), ref, spec.dtype, "straddling groups")
    # every sequence a group of its own
    ones = np.arange(b + 1, dtype=np.int32)
    gh.assert_close(gh.to_f64(_run(w, kc, vc, slots, ones, huge).out), ref, spec.dtype, "groups of one")
    # no groups at all: the plain step
    none = np.zeros(1, dtype=np.int32)
    gh.assert_close(gh.to_f64(_run(w, kc, vc, slots, none, huge).out), ref, spec.dtype, "no groups")


def test_invalid_group_start_is_flagged_and_computed_unshared():
    spec = SPECS[2]
    w = workloads.make(spec)
    kc, vc, slots = gh.prepare(w)
    ref, _, _ = gh.oracle_step(w, kc, vc, slots)
    starts, claims = _groups_of(w)
    bad = starts.copy()
    bad[1] = spec.num_seqs + 5              # past the batch: that group is flagged
    step = gh.GpuStep(w, kc, vc, slots)
    n = pkv.pkv_shared_prefix_workspace_bytes(spec.num_seqs, spec.num_q_heads, spec.num_kv_heads, spec.head_dim,
                                              w.max_blocks_per_seq * spec.block_size, len(bad) - 1)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    pkv.pkv_append_decode_attention_shared_prefix(step.kn, step.vn, step.slots, step.q, step.kc, step.vc,
                                                  step.tables, step.lens, torch.from_numpy(bad).cuda(),
                                                  torch.from_numpy(claims).cuda(), w.scale, step.out, ws)
    assert pkv.pkv_get_last_error() == pkv.PKV_ERR_DEVICE_CHECK
    gh.assert_close(gh.to_f64(step.out), ref, spec.dtype, "invalid group entry")
