"""GPU path vs the fp64 oracle on the same seeded inputs, through the C ABI.

Small shapes are compared element by element (they span several 16-token
tiles and ragged tails); the named full-size workloads are compared on
sampled (sequence, head) pairs with the same launch configuration the
benchmark times, plus a bit-exact check of the whole pool after the append.
Every slot outside the attended context is NaN-poisoned first.
"""
import numpy as np
import pytest

import gpu_harness as gh
import paged_kv_cache_437_b200 as pkv
import workloads
from workloads import BF16, F16, custom

pytestmark = pytest.mark.gpu

SMALL = [
    custom("mha_d64_f16", 4, 4, 4, 64, 16, F16, 10, [17, 33, 64, 100], num_blocks=64),
    custom("gqa8_d128_bf16", 7, 16, 2, 128, 16, BF16, 11, [1, 15, 16, 17, 100, 513, 1000]),
    custom("gqa4_d128_f16_bs32", 6, 16, 4, 128, 32, F16, 12, [31, 32, 33, 64, 300, 777]),
    custom("g16_d128_bf16", 3, 32, 2, 128, 16, BF16, 13, [5, 200, 1200]),
    custom("g32_d64_f16", 2, 64, 2, 64, 16, F16, 14, [40, 999]),
    custom("g2_d64_bf16_bs64", 5, 4, 2, 64, 64, BF16, 15, [1, 63, 64, 65, 500]),
    custom("g12_d128_f16", 3, 24, 2, 128, 16, F16, 16, [33, 48, 1500]),
    custom("shared_prefix_bs32", 12, 8, 2, 128, 32, F16, 17, [20, 64, 65, 100, 257, 300, 33, 40, 96, 97, 512, 700],
           share_group=4, share_prefix_tokens=256),
]
MODES = [pkv.PKV_PARTITION_NONE, pkv.PKV_PARTITION_AUTO, 512, 16, 48]


@pytest.fixture(scope="module", params=SMALL, ids=lambda s: s.name)
def small_case(request):
    w = workloads.make(request.param)
    kc, vc, slots = gh.prepare(w)
    ref, k_ref, v_ref = gh.oracle_step(w, kc, vc, slots)
    return w, kc, vc, slots, ref, k_ref, v_ref


@pytest.mark.parametrize("mode", MODES, ids=lambda m: f"part{m}")
def test_small_shapes_elementwise(small_case, mode):
    w, kc, vc, slots, ref, k_ref, v_ref = small_case
    step = gh.GpuStep(w, kc, vc, slots)
    out = step.run(mode)
    assert np.array_equal(gh.host_bits(step.kc), k_ref), "appended K pool differs"
    assert np.array_equal(gh.host_bits(step.vc), v_ref), "appended V pool differs"
    gh.assert_close(gh.to_f64(out), ref, w.spec.dtype, f"{w.spec.name} mode {mode}")


@pytest.mark.parametrize("mode", [pkv.PKV_PARTITION_NONE, pkv.PKV_PARTITION_AUTO, 512, 16], ids=lambda m: f"part{m}")
def test_fused_append_decode_small_shapes(small_case, mode):
    """pkv_append_decode_attention: same pool and the same output bits as
    pkv_append followed by pkv_decode_attention, and within tolerance of the oracle."""
    w, kc, vc, slots, ref, k_ref, v_ref = small_case
    fused = gh.GpuStep(w, kc, vc, slots)
    out_f = fused.run_fused(mode).clone()
    assert np.array_equal(gh.host_bits(fused.kc), k_ref), "fused: appended K pool differs"
    assert np.array_equal(gh.host_bits(fused.vc), v_ref), "fused: appended V pool differs"
    gh.assert_close(gh.to_f64(out_f), ref, w.spec.dtype, f"fused {w.spec.name} mode {mode}")
    sep = gh.GpuStep(w, kc, vc, slots)
    out_s = sep.run(mode)
    assert np.array_equal(gh.host_bits(out_f), gh.host_bits(out_s)), "fused and separate calls differ"


FULL_MODES = {
    "tiny": [pkv.PKV_PARTITION_AUTO, pkv.PKV_PARTITION_NONE, 512],
    "llama13b": [pkv.PKV_PARTITION_AUTO],
    "llama70b_gqa": [pkv.PKV_PARTITION_AUTO],
    "cb_mixed": [pkv.PKV_PARTITION_AUTO],
    "long_split": [512, pkv.PKV_PARTITION_AUTO],
}


@pytest.mark.parametrize("name", workloads.ORDER)
def test_named_workload_full_size(name):
    w = workloads.make(name)
    kc, vc, slots = gh.prepare(w)
    pairs = None if name == "tiny" else gh.sample_pairs(w, 256)
    ref, k_ref, v_ref = gh.oracle_step(w, kc, vc, slots, pairs=pairs)
    step = gh.GpuStep(w, kc, vc, slots)
    for mode, fused in [(m, f) for m in FULL_MODES[name] for f in (False, True)]:
        step.kc.copy_(gh.dev(kc, w.spec.dtype))
        step.vc.copy_(gh.dev(vc, w.spec.dtype))
        out = step.run_fused(mode) if fused else step.run(mode)
        assert np.array_equal(gh.host_bits(step.kc), k_ref), f"{name}: appended K pool differs"
        assert np.array_equal(gh.host_bits(step.vc), v_ref), f"{name}: appended V pool differs"
        got = gh.to_f64(out)
        assert np.all(np.isfinite(got)), f"{name}: non-finite output"
        if pairs is not None:
            got = got[pairs[:, 0], pairs[:, 1]]
        err = gh.assert_close(got, ref, w.spec.dtype, f"{name} mode {mode}")
        print(f"{name} mode {mode} fused {fused}: {len(ref) if pairs is not None else ref.size} compared, "
              f"max |err| {err:.3e}")


@pytest.mark.parametrize("unit_cost", ["0", "8"])
def test_balanced_schedule_unit_cost_extremes(small_case, unit_cost, monkeypatch):
    # the work-balanced order with no virtual tiles per (sequence, head group)
    # and with the most: ranges that start or end inside the virtual tails
    monkeypatch.setenv("PKV_UNIT_COST", unit_cost)
    w, kc, vc, slots, ref, k_ref, v_ref = small_case
    step = gh.GpuStep(w, kc, vc, slots)
    out = step.run_fused(pkv.PKV_PARTITION_AUTO)
    gh.assert_close(gh.to_f64(out), ref, w.spec.dtype, f"{w.spec.name} unit cost {unit_cost}")


def test_long_rows_merged_in_decode(monkeypatch):
    # rows split over many warps (more than the 16 pieces the whole-group
    # merge takes): the decode kernel's last piece merges them head by head
    monkeypatch.setenv("PKV_FOLD_MERGE", "1")
    spec = custom("long_fold_bf16", 2, 64, 8, 128, 16, BF16, 16, [20000, 12345])
    w = workloads.make(spec)
    kc, vc, slots = gh.prepare(w)
    ref, _, _ = gh.oracle_step(w, kc, vc, slots)
    for fused in (False, True):
        step = gh.GpuStep(w, kc, vc, slots)
        out = step.run_fused(pkv.PKV_PARTITION_AUTO) if fused else step.run(pkv.PKV_PARTITION_AUTO)
        gh.assert_close(gh.to_f64(out), ref, BF16, f"long rows, merge in decode, fused={fused}")


@pytest.mark.parametrize("fold", ["0", "1"], ids=["merge_kernel", "merge_in_decode"])
def test_split_rows_merged_either_way(small_case, fold, monkeypatch):
    # the work-balanced schedule's split rows, merged by the merge kernel or
    # by the decode kernel's last piece of each row (whichever the shape picks
    # by default, both must agree with the oracle), plain and fused step
    monkeypatch.setenv("PKV_FOLD_MERGE", fold)
    w, kc, vc, slots, ref, k_ref, v_ref = small_case
    for fused in (False, True):
        step = gh.GpuStep(w, kc, vc, slots)
        out = step.run_fused(pkv.PKV_PARTITION_AUTO) if fused else step.run(pkv.PKV_PARTITION_AUTO)
        gh.assert_close(gh.to_f64(out), ref, w.spec.dtype, f"{w.spec.name} fold={fold} fused={fused}")
