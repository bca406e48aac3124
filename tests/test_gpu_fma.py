"""The CUDA-core (FFMA) variant of the decode kernel against the fp64 oracle.

The variant exists to measure the choice of the tensor-core MMA for the two
small products (same pipeline, schedules and epilogue layout; FFMA
arithmetic); it is selected with PKV_FMA=1 and must meet the same
tolerances, fused append included.
"""
import numpy as np
import pytest

import gpu_harness as gh
import paged_kv_cache_437_b200 as pkv
import workloads
from test_gpu_parity import SMALL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", params=SMALL, ids=lambda s: s.name)
def fma_case(request):
    w = workloads.make(request.param)
    kc, vc, slots = gh.prepare(w)
    ref, k_ref, v_ref = gh.oracle_step(w, kc, vc, slots)
    return w, kc, vc, slots, ref, k_ref, v_ref


@pytest.mark.parametrize("mode", [pkv.PKV_PARTITION_NONE, pkv.PKV_PARTITION_AUTO, 512, 16],
                         ids=lambda m: f"part{m}")
def test_fma_variant_matches_oracle(fma_case, mode, monkeypatch):
    monkeypatch.setenv("PKV_FMA", "1")
    w, kc, vc, slots, ref, k_ref, v_ref = fma_case
    step = gh.GpuStep(w, kc, vc, slots)
    out = step.run(mode)
    assert np.array_equal(gh.host_bits(step.kc), k_ref)
    gh.assert_close(gh.to_f64(out), ref, w.spec.dtype, f"fma {w.spec.name} mode {mode}")
    fused = gh.GpuStep(w, kc, vc, slots)
    out_f = fused.run_fused(mode)
    assert np.array_equal(gh.host_bits(fused.vc), v_ref)
    gh.assert_close(gh.to_f64(out_f), ref, w.spec.dtype, f"fma fused {w.spec.name} mode {mode}")


@pytest.mark.parametrize("name", ["llama70b_gqa", "cb_mixed"])
def test_fma_variant_full_size_sampled(name, monkeypatch):
    monkeypatch.setenv("PKV_FMA", "1")
    w = workloads.make(name)
    kc, vc, slots = gh.prepare(w)
    pairs = gh.sample_pairs(w, 64)
    ref, _, _ = gh.oracle_step(w, kc, vc, slots, pairs=pairs)
    out = gh.to_f64(gh.GpuStep(w, kc, vc, slots).run(pkv.PKV_PARTITION_AUTO))
    gh.assert_close(out[pairs[:, 0], pairs[:, 1]], ref, w.spec.dtype, f"fma {name}")
