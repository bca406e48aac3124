"""Invariants of the GPU path that hold bit for bit, and edge cases."""
import numpy as np
import pytest
import torch

import gpu_harness as gh
import oracle
import paged_kv_cache_437_b200 as pkv
import workloads
from workloads import BF16, F16, custom

pytestmark = pytest.mark.gpu

MODES = [pkv.PKV_PARTITION_NONE, pkv.PKV_PARTITION_AUTO, 64]


def _run(w, kc, vc, slots, mode):
    step = gh.GpuStep(w, kc, vc, slots)
    return step.run(mode).clone()


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype", [F16, BF16])
def test_physical_block_permutation_is_bit_identical(mode, dtype):
    spec = custom("perm", 5, 16, 4, 128, 16, dtype, 21, [3, 16, 77, 200, 333])
    w = workloads.make(spec)
    kc, vc, slots = gh.prepare(w)
    base = _run(w, kc, vc, slots, mode)
    perm = np.random.default_rng(5).permutation(w.num_blocks)
    k2, v2 = np.empty_like(kc), np.empty_like(vc)
    k2[perm], v2[perm] = kc, vc
    tables = np.where(w.block_tables >= 0, perm[np.maximum(w.block_tables, 0)], -1).astype(np.int32)
    w2 = workloads.Workload(w.spec, w.context_lens, tables, w.num_blocks, w.owned_blocks, w.shared_blocks,
                            w.q, k2, v2, w.k_new, w.v_new, w.scale)
    slots2 = oracle.slot_mapping(tables, w.context_lens.astype(np.int64) - 1, w.spec.block_size)
    moved = _run(w2, k2, v2, slots2, mode)
    assert torch.equal(moved.view(torch.int16), base.view(torch.int16))


@pytest.mark.parametrize("mode", MODES)
def test_shared_prefix_equals_duplicated_blocks(mode):
    spec = custom("share", 8, 8, 2, 128, 32, F16, 22, [40, 100, 129, 300, 64, 65, 200, 511],
                  share_group=4, share_prefix_tokens=128)
    w = workloads.make(spec)
    kc, vc, slots = gh.prepare(w)
    shared = _run(w, kc, vc, slots, mode)
    # give every sharer private copies of the shared blocks
    extra = sum(w.shared_blocks)
    nb2 = w.num_blocks + extra
    k2 = np.concatenate([kc, np.zeros((extra,) + kc.shape[1:], np.uint16)])
    v2 = np.concatenate([vc, np.zeros((extra,) + vc.shape[1:], np.uint16)])
    tables = w.block_tables.copy()
    nxt = w.num_blocks
    for s in range(spec.num_seqs):
        for i in range(w.shared_blocks[s]):
            src = tables[s, i]
            k2[nxt], v2[nxt] = kc[src], vc[src]
            tables[s, i] = nxt
            nxt += 1
    assert nxt == nb2 and extra > 0
    w2 = workloads.Workload(w.spec, w.context_lens, tables, nb2, w.owned_blocks, [0] * spec.num_seqs,
                            w.q, k2, v2, w.k_new, w.v_new, w.scale)
    dup = _run(w2, k2, v2, slots, mode)
    assert torch.equal(dup.view(torch.int16), shared.view(torch.int16))


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype", [F16, BF16])
def test_single_position_returns_v_exactly(mode, dtype):
    spec = custom("ctx1", 6, 16, 2, 128, 16, dtype, 23, [1] * 6)
    w = workloads.make(spec)
    kc, vc, slots = gh.prepare(w)
    out = _run(w, kc, vc, slots, mode)
    g = spec.num_q_heads // spec.num_kv_heads
    expect = np.repeat(w.v_new, g, axis=1)          # the appended token's V, per query head
    assert np.array_equal(gh.host_bits(out), expect)


@pytest.mark.parametrize("mode", MODES)
def test_scaling_v_by_two_doubles_output_exactly(mode):
    spec = custom("v2", 4, 8, 2, 64, 16, F16, 24, [17, 100, 250, 31])
    w = workloads.make(spec)
    kc, vc, slots = gh.prepare(w)
    base = _run(w, kc, vc, slots, mode)
    dbl = lambda bits: (bits.view(np.float16).astype(np.float32) * 2).astype(np.float16).view(np.uint16)
    vc2 = np.where(np.isnan(vc.view(np.float16)), vc, dbl(vc))
    w2 = workloads.Workload(w.spec, w.context_lens, w.block_tables, w.num_blocks, w.owned_blocks,
                            w.shared_blocks, w.q, kc, vc2, w.k_new, dbl(w.v_new), w.scale)
    out2 = _run(w2, kc, vc2, slots, mode)
    # exact wherever the output is a normal fp16 number; in the subnormal range
    # (|x| < 2^-14) rounding 2x and doubling round(x) can differ by one quantum
    b2 = (base.double() * 2).cpu()
    o2 = out2.double().cpu()
    normal = b2.abs() >= 2.0 ** -13
    assert torch.equal(o2[normal], b2[normal])
    assert float((o2 - b2).abs().max()) <= 2.0 ** -24


@pytest.mark.parametrize("mode", MODES + [512])
def test_zero_length_sequences_give_zero_rows(mode):
    spec = custom("zero", 5, 8, 2, 128, 16, BF16, 25, [0, 40, 0, 300, 1])
    w = workloads.make(spec)
    kc, vc, slots = gh.prepare(w)
    step = gh.GpuStep(w, kc, vc, slots)
    step.out.fill_(7.0)
    out = step.run(mode)
    ref, _, _ = gh.oracle_step(w, kc, vc, slots)
    assert torch.count_nonzero(out[0]) == 0 and torch.count_nonzero(out[2]) == 0
    gh.assert_close(gh.to_f64(out), ref, BF16, "zero-length")


def test_non_default_stream_and_repeat_calls():
    spec = custom("stream", 3, 16, 2, 128, 16, F16, 26, [100, 1000, 2000])
    w = workloads.make(spec)
    kc, vc, slots = gh.prepare(w)
    ref, _, _ = gh.oracle_step(w, kc, vc, slots)
    step = gh.GpuStep(w, kc, vc, slots)
    ws = gh.workspace_for(w, pkv.PKV_PARTITION_AUTO)
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        step.append(s)
        for _ in range(3):
            step.decode(pkv.PKV_PARTITION_AUTO, ws, s)
    s.synchronize()
    assert pkv.pkv_get_last_error() == pkv.PKV_OK
    gh.assert_close(gh.to_f64(step.out), ref, F16, "stream")
