"""The decode entry point for callers that cannot allocate device memory.

Such callers (a plugin / custom-operator interface that is handed device
pointers for its inputs and outputs but no allocator, or a serving loop that
bans cudaMalloc once running) use pkv_decode_attention_static_scratch, whose
split-context scratch is a fixed array inside the library.  This file checks,
through the C ABI, that two calls in a row give the same result as the
regular entry point with a caller-allocated workspace, within the parity
tolerance used everywhere else, and that a shape needing more scratch than
the fixed array is refused before anything runs.  It is named so that pytest
collects it last.
"""
import numpy as np
import pytest
import torch

import gpu_harness as gh
import paged_kv_cache_437_b200 as pkv
import workloads
from workloads import BF16, F16, custom

pytestmark = pytest.mark.gpu


def _call_static(step, partition):
    lib = pkv.lib
    st = lib.pkv_decode_attention_static_scratch(
        step.q.data_ptr(), step.q.shape[0], step.q.shape[1], pkv.cache_desc(step.kc), pkv.cache_desc(step.vc),
        step.tables.data_ptr(), step.tables.shape[1], step.lens.data_ptr(), float(step.w.scale),
        step.out.data_ptr(), int(partition), pkv._stream_ptr(None))
    assert st == pkv.PKV_OK, pkv.pkv_status_string(st)


@pytest.mark.parametrize("partition", [pkv.PKV_PARTITION_AUTO, 512, 64])
@pytest.mark.parametrize("spec", [
    custom("noalloc_gqa", 6, 32, 4, 128, 16, BF16, 41, [1, 17, 300, 1024, 2049, 5000]),
    custom("noalloc_mha", 5, 8, 8, 64, 32, F16, 42, [33, 64, 65, 700, 1500]),
], ids=lambda s: s.name)
def test_static_scratch_matches_workspace_entry_point(spec, partition):
    w = workloads.make(spec)
    kc, vc, slots = gh.prepare(w)
    step = gh.GpuStep(w, kc, vc, slots)
    step.append()
    ws = gh.workspace_for(w, partition)
    step.decode(partition, ws)
    torch.cuda.synchronize()
    expect = gh.to_f64(step.out)
    for _ in range(2):                    # two calls in a row share the array
        step.out.fill_(float("nan"))
        _call_static(step, partition)
        torch.cuda.synchronize()
        assert pkv.pkv_get_last_error() == pkv.PKV_OK
        gh.assert_close(gh.to_f64(step.out), expect, spec.dtype, f"static scratch {spec.name} {partition}")


def test_static_scratch_refuses_oversized_shapes():
    big_b = 4096
    need = pkv.pkv_decode_workspace_bytes(big_b, 64, 8, 128, 65536, 512)
    assert need > pkv.PKV_STATIC_SCRATCH_BYTES
    kc = torch.empty((8, 8, 16, 128), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((big_b, 64, 128), dtype=torch.bfloat16, device="cuda")
    tables = torch.zeros((big_b, 4096), dtype=torch.int32, device="cuda")
    lens = torch.zeros(big_b, dtype=torch.int32, device="cuda")
    with pytest.raises(pkv.PkvError) as e:
        pkv.pkv_decode_attention_static_scratch(q, kc, kc, tables, lens, 0.1, q, 512)
    assert e.value.status == pkv.PKV_ERR_SCRATCH_TOO_SMALL
