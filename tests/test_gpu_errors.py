"""Device-side checks and the bounded waits: bad indices and an injected
wait time-out are reported through pkv_get_last_error(), nothing faults,
and the context stays usable for the next correct call."""
import numpy as np
import pytest
import torch

import gpu_harness as gh
import paged_kv_cache_437_b200 as pkv
import workloads
from workloads import F16, custom

pytestmark = pytest.mark.gpu


def _case():
    spec = custom("err", 3, 8, 2, 128, 16, F16, 31, [20, 50, 90])
    w = workloads.make(spec)
    kc, vc, slots = gh.prepare(w)
    return w, kc, vc, slots


def _good_call_still_works(w, kc, vc, slots):
    ref, _, _ = gh.oracle_step(w, kc, vc, slots)
    out = gh.GpuStep(w, kc, vc, slots).run(pkv.PKV_PARTITION_AUTO)
    gh.assert_close(gh.to_f64(out), ref, F16, "after error")


def test_table_entry_out_of_range_is_flagged():
    w, kc, vc, slots = _case()
    step = gh.GpuStep(w, kc, vc, slots)
    step.tables[1, 2] = w.num_blocks + 5
    step.append()
    step.decode(pkv.PKV_PARTITION_NONE)
    assert pkv.pkv_get_last_error() == pkv.PKV_ERR_DEVICE_CHECK
    assert pkv.pkv_get_last_error() == pkv.PKV_OK      # read-and-clear
    _good_call_still_works(w, kc, vc, slots)


def test_context_longer_than_table_is_flagged():
    w, kc, vc, slots = _case()
    step = gh.GpuStep(w, kc, vc, slots)
    step.lens[0] = w.max_blocks_per_seq * w.spec.block_size + 100
    step.decode(pkv.PKV_PARTITION_AUTO, gh.workspace_for(w, pkv.PKV_PARTITION_AUTO))
    assert pkv.pkv_get_last_error() == pkv.PKV_ERR_DEVICE_CHECK


def test_append_slot_outside_pool_is_flagged():
    w, kc, vc, slots = _case()
    step = gh.GpuStep(w, kc, vc, slots)
    step.slots[0] = w.num_blocks * w.spec.block_size + 3
    before = gh.host_bits(step.kc)
    step.append()
    assert pkv.pkv_get_last_error() == pkv.PKV_ERR_DEVICE_CHECK
    after = gh.host_bits(step.kc)
    assert np.count_nonzero(before != after) <= 2 * w.spec.num_kv_heads * w.spec.head_dim


def test_padding_slots_write_nothing():
    w, kc, vc, slots = _case()
    step = gh.GpuStep(w, kc, vc, slots)
    step.slots.fill_(-1)
    before = gh.host_bits(step.kc)
    step.append()
    torch.cuda.synchronize()
    assert pkv.pkv_get_last_error() == pkv.PKV_OK
    assert np.array_equal(gh.host_bits(step.kc), before)


def test_injected_wait_timeout_is_reported_and_recovers():
    w, kc, vc, slots = _case()
    step = gh.GpuStep(w, kc, vc, slots)
    pkv.pkv_test_inject_wait_timeout(True, 20_000_000)   # 20 ms
    try:
        step.decode(pkv.PKV_PARTITION_NONE)
        torch.cuda.synchronize()
    finally:
        pkv.pkv_test_inject_wait_timeout(False)
    assert pkv.pkv_get_last_error() == pkv.PKV_ERR_TIMEOUT
    _good_call_still_works(w, kc, vc, slots)
