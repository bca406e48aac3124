"""The scheduler driving the hot path on the GPU: every step appends the
batch's new tokens at the scheduler's slots and runs chunked prefill /
decode attention over its mixed batch; pool and outputs match the oracle
replaying the same steps, including across a preemption."""
import numpy as np
import pytest
import torch

import gpu_harness as gh
import oracle
import paged_kv_cache_437_b200 as pkv
import workloads

pytestmark = pytest.mark.gpu


def test_scheduled_steps_match_oracle():
    dtype, nb, bs, hkv, hq, d = workloads.F16, 14, 16, 2, 8, 64
    rng = np.random.default_rng(90)
    alloc = pkv.BlockAllocator(nb, bs)
    sched = pkv.Scheduler(alloc, max_batch_tokens=96, max_seqs=4, chunk_tokens=48)
    for rid, (p, m) in enumerate([(70, 6), (20, 9), (100, 3), (33, 12)]):
        sched.add(rid, p, m)
    k_ref = np.zeros((nb, hkv, bs, d), np.uint16)
    v_ref = np.zeros((nb, hkv, bs, d), np.uint16)
    kc, vc = gh.dev(k_ref, dtype), gh.dev(v_ref, dtype)
    scale = 0.125
    steps = preempted = 0
    while (sched.num_waiting or sched.num_running) and steps < 200:
        b = sched.step()
        steps += 1
        preempted += len(b["preempted"])
        t = len(b["slots"])
        if t == 0:
            continue
        kn = workloads.to_bits(rng.standard_normal((t, hkv, d), dtype=np.float32), dtype)
        vn = workloads.to_bits(rng.standard_normal((t, hkv, d), dtype=np.float32), dtype)
        q = workloads.to_bits(rng.standard_normal((t, hq, d), dtype=np.float32), dtype)
        tables, lens = alloc.batch_tables(b["seq_ids"], nb)
        qs = np.concatenate([[0], np.cumsum(b["query_lens"])]).astype(np.int32)
        oracle.append(k_ref, kn, b["slots"])
        oracle.append(v_ref, vn, b["slots"])
        ref = oracle.prefill_attention(q, k_ref, v_ref, tables, qs, lens, scale, dtype)
        pkv.pkv_append(gh.dev(kn, dtype), gh.dev(vn, dtype), torch.from_numpy(b["slots"]).cuda(), kc, vc)
        qd = gh.dev(q, dtype)
        out = torch.empty_like(qd)
        ws = torch.empty(pkv.pkv_prefill_workspace_bytes(t, hq, hkv, d, nb * bs), dtype=torch.uint8,
                         device="cuda")
        pkv.pkv_prefill_attention(qd, kc, vc, torch.from_numpy(tables).cuda(), torch.from_numpy(qs).cuda(),
                                  torch.from_numpy(lens).cuda(), scale, out, ws)
        torch.cuda.synchronize()
        assert pkv.pkv_get_last_error() == pkv.PKV_OK
        gh.assert_close(gh.to_f64(out), ref, dtype, f"scheduled step {steps}")
        assert np.array_equal(gh.host_bits(kc), k_ref)
    assert sched.num_waiting == 0 and sched.num_running == 0
    assert preempted > 0           # 14 blocks cannot hold all four requests at once
    assert alloc.num_free() == nb
