"""The decode entry point for callers that cannot allocate device memory.

Such callers (a plugin / custom-operator interface that is handed device
pointers for its inputs and outputs but no allocator, or a serving loop that
bans cudaMalloc once running) use pkv_decode_attention_static_scratch, whose
split-context scratch is a fixed array inside the library.  This file checks,
through the C ABI, that two calls in a row give the same result as the
regular entry point with a caller-allocated workspace and as the fp64 oracle,
within the parity tolerance used everywhere else -- after a call on another
workload has left different data in the array -- that a shape needing more
scratch than the fixed array is refused before anything runs, and that an
AUTO batch too large for the on-chip schedule still runs (with no scratch).
It is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import gpu_harness as gh
import oracle
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


# a different workload whose call fills the array with other partials first
_DIRTY = custom("noalloc_dirty", 7, 32, 4, 128, 16, BF16, 43, [4000, 9, 2500, 700, 1, 3333, 6000])


def _dirty_the_array(partition):
    w = workloads.make(_DIRTY)
    kc, vc, slots = gh.prepare(w, poison=False)
    step = gh.GpuStep(w, kc, vc, slots)
    step.append()
    _call_static(step, partition)
    torch.cuda.synchronize()
    assert pkv.pkv_get_last_error() == pkv.PKV_OK


@pytest.mark.parametrize("partition", [pkv.PKV_PARTITION_AUTO, 512, 64])
@pytest.mark.parametrize("spec", [
    custom("noalloc_gqa", 6, 32, 4, 128, 16, BF16, 41, [1, 17, 300, 1024, 2049, 5000]),
    custom("noalloc_mha", 5, 8, 8, 64, 32, F16, 42, [33, 64, 65, 700, 1500]),
], ids=lambda s: s.name)
def test_static_scratch_matches_workspace_entry_point_and_oracle(spec, partition):
    w = workloads.make(spec)
    kc, vc, slots = gh.prepare(w)
    ref, _, _ = gh.oracle_step(w, kc, vc, slots)
    step = gh.GpuStep(w, kc, vc, slots)
    step.append()
    ws = gh.workspace_for(w, partition)
    step.decode(partition, ws)
    torch.cuda.synchronize()
    expect = gh.to_f64(step.out)
    gh.assert_close(expect, ref, spec.dtype, f"workspace entry {spec.name} {partition}")
    _dirty_the_array(partition)
    for _ in range(2):                    # two calls in a row share the array
        step.out.fill_(float("nan"))
        _call_static(step, partition)
        torch.cuda.synchronize()
        assert pkv.pkv_get_last_error() == pkv.PKV_OK
        got = gh.to_f64(step.out)
        gh.assert_close(got, expect, spec.dtype, f"static scratch vs workspace {spec.name} {partition}")
        gh.assert_close(got, ref, spec.dtype, f"static scratch vs oracle {spec.name} {partition}")


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


def test_static_scratch_auto_batch_beyond_on_chip_schedule():
    # AUTO needs no scratch for a batch whose schedule does not fit on chip:
    # both entry points fall back to one pass per (sequence, head group)
    b, hkv, d, bs = 40000, 1, 64, 16
    assert pkv.pkv_decode_workspace_bytes(b, hkv, hkv, d, bs, pkv.PKV_PARTITION_AUTO) == 0
    rng = np.random.default_rng(5)
    lens = rng.integers(1, bs + 1, size=b).astype(np.int32)
    nb = b
    tables = rng.permutation(nb).astype(np.int32).reshape(b, 1)
    q = rng.standard_normal((b, hkv, d)).astype(np.float16)
    k = rng.standard_normal((nb, hkv, bs, d)).astype(np.float16)
    v = rng.standard_normal((nb, hkv, bs, d)).astype(np.float16)
    dq, dk, dv = (torch.from_numpy(x).cuda() for x in (q, k, v))
    dt, dl = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    out = torch.full_like(dq, float("nan"))
    pkv.pkv_decode_attention_static_scratch(dq, dk, dv, dt, dl, 0.125, out, pkv.PKV_PARTITION_AUTO)
    expect = torch.full_like(dq, float("nan"))
    pkv.pkv_decode_attention(dq, dk, dv, dt, dl, 0.125, expect, None, pkv.PKV_PARTITION_NONE)
    torch.cuda.synchronize()
    assert pkv.pkv_get_last_error() == pkv.PKV_OK
    assert torch.equal(out, expect)
    pick = np.array(sorted(set([0, b - 1] + rng.integers(0, b, 62).tolist())))
    bits = lambda x: x.view(np.uint16)
    ref = oracle.attention(bits(q[pick]), bits(k), bits(v), tables[pick], lens[pick], 0.125, F16)
    gh.assert_close(gh.to_f64(out[torch.from_numpy(pick).cuda()]), ref, F16, "static scratch AUTO, large batch")


def test_static_scratch_wrapper_checks_dtypes():
    kc = torch.zeros((4, 2, 16, 64), dtype=torch.float16, device="cuda")
    q = torch.zeros((2, 2, 64), dtype=torch.float16, device="cuda")
    tables = torch.zeros((2, 1), dtype=torch.int64, device="cuda")
    lens = torch.ones(2, dtype=torch.int32, device="cuda")
    with pytest.raises(TypeError):
        pkv.pkv_decode_attention_static_scratch(q, kc, kc, tables, lens, 0.1, q)
    with pytest.raises(TypeError):
        pkv.pkv_decode_attention_static_scratch(q.bfloat16(), kc, kc, tables.int(), lens, 0.1, q.bfloat16())
