"""FP8 E4M3 KV cache on the GPU against the oracle: the quantizing append
must give the same codes and scales bit for bit; decode over oracle-quantized
pools must match the oracle's E4M3 attention within the usual tolerance.
Unused slots hold NaN codes and NaN scales."""
import numpy as np
import pytest
import torch

import gpu_harness as gh
import oracle
import paged_kv_cache_437_b200 as pkv
import workloads
from workloads import BF16, F16, custom

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [F16, BF16])
@pytest.mark.parametrize("d", [64, 128])
def test_e4m3_append_bit_exact(dtype, d):
    rng = np.random.default_rng(80 + d)
    nb, hkv, bs, t = 9, 3, 16, 40
    new_k = workloads.to_bits((rng.standard_normal((t, hkv, d)) * rng.uniform(0.01, 30, (t, hkv, 1)))
                              .astype(np.float32), dtype)
    new_v = workloads.to_bits(rng.standard_normal((t, hkv, d)).astype(np.float32) * 5, dtype)
    new_k[3, 1] = 0                                   # an all-zero row: scale 1, codes 0
    slots = rng.permutation(nb * bs)[:t].astype(np.int64)
    slots[7] = -1                                     # padding token
    k8 = np.full((nb, hkv, bs, d), 0x7f, np.uint8)
    v8 = np.full((nb, hkv, bs, d), 0x7f, np.uint8)
    ks = np.full((nb, hkv, bs), np.nan, np.float32)
    vs = np.full((nb, hkv, bs), np.nan, np.float32)
    kd8, vd8 = torch.from_numpy(k8).cuda(), torch.from_numpy(v8).cuda()
    kds, vds = torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda()
    pkv.pkv_append_e4m3(gh.dev(new_k, dtype), gh.dev(new_v, dtype), torch.from_numpy(slots).cuda(),
                        kd8, kds, vd8, vds)
    torch.cuda.synchronize()
    assert pkv.pkv_get_last_error() == pkv.PKV_OK
    oracle.append_e4m3(k8, ks, new_k, dtype, slots)
    oracle.append_e4m3(v8, vs, new_v, dtype, slots)
    assert np.array_equal(kd8.cpu().numpy(), k8) and np.array_equal(vd8.cpu().numpy(), v8)
    assert np.array_equal(kds.cpu().numpy().view(np.uint32), ks.view(np.uint32))
    assert np.array_equal(vds.cpu().numpy().view(np.uint32), vs.view(np.uint32))


SPECS = [
    custom("e4m3_gqa8", 5, 16, 2, 128, 16, BF16, 81, [1, 16, 17, 300, 1025]),
    custom("e4m3_gqa4_bs32", 4, 16, 4, 128, 32, F16, 82, [31, 64, 500, 2000]),
    custom("e4m3_mha_d64", 3, 4, 4, 64, 16, F16, 83, [5, 100, 260]),
    custom("e4m3_g16", 2, 32, 2, 128, 16, BF16, 84, [77, 900]),
]


@pytest.fixture(scope="module", params=SPECS, ids=lambda s: s.name)
def e4m3_case(request):
    spec = request.param
    w = workloads.make(spec)
    nb, hkv, bs, d = w.k_cache.shape
    # quantize every valid row of the 16-bit pools with the oracle; everything
    # else holds NaN codes and NaN scales
    lens = w.context_lens
    mask = oracle.slot_mask(w.block_tables, lens, bs, nb)
    slots = np.nonzero(mask)[0].astype(np.int64)
    rows_k = np.ascontiguousarray(w.k_cache.transpose(0, 2, 1, 3).reshape(nb * bs, hkv, d)[slots])
    rows_v = np.ascontiguousarray(w.v_cache.transpose(0, 2, 1, 3).reshape(nb * bs, hkv, d)[slots])
    k8 = np.full((nb, hkv, bs, d), 0x7f, np.uint8)
    v8 = np.full((nb, hkv, bs, d), 0x7f, np.uint8)
    ks = np.full((nb, hkv, bs), np.nan, np.float32)
    vs = np.full((nb, hkv, bs), np.nan, np.float32)
    oracle.append_e4m3(k8, ks, rows_k, spec.dtype, slots)
    oracle.append_e4m3(v8, vs, rows_v, spec.dtype, slots)
    ref = oracle.attention_e4m3(w.q, spec.dtype, k8, ks, v8, vs, w.block_tables, lens, w.scale)
    return w, k8, ks, v8, vs, ref


@pytest.mark.parametrize("mode", [pkv.PKV_PARTITION_NONE, pkv.PKV_PARTITION_AUTO, 512, 16], ids=lambda m: f"part{m}")
def test_e4m3_decode_matches_oracle(e4m3_case, mode):
    w, k8, ks, v8, vs, ref = e4m3_case
    dt = w.spec.dtype
    args = [torch.from_numpy(x).cuda() for x in (k8, ks, v8, vs)]
    q = gh.dev(w.q, dt)
    out = torch.empty_like(q)
    ws = gh.workspace_for(w, mode)
    pkv.pkv_decode_attention_e4m3(q, *args, torch.from_numpy(w.block_tables).cuda(),
                                  torch.from_numpy(w.context_lens).cuda(), w.scale, out, ws, mode)
    torch.cuda.synchronize()
    assert pkv.pkv_get_last_error() == pkv.PKV_OK
    gh.assert_close(gh.to_f64(out), ref, dt, f"e4m3 {w.spec.name} mode {mode}")


def test_e4m3_append_then_decode_pipeline():
    """Quantize a whole context with the GPU append and decode it: equals the
    oracle run on the oracle-quantized pools (same codes, so same answer)."""
    spec = custom("e4m3_pipe", 3, 16, 2, 128, 16, BF16, 85, [40, 333, 1000])
    w = workloads.make(spec)
    nb, hkv, bs, d = w.k_cache.shape
    lens = w.context_lens
    slots = np.nonzero(oracle.slot_mask(w.block_tables, lens, bs, nb))[0].astype(np.int64)
    rows_k = np.ascontiguousarray(w.k_cache.transpose(0, 2, 1, 3).reshape(nb * bs, hkv, d)[slots])
    rows_v = np.ascontiguousarray(w.v_cache.transpose(0, 2, 1, 3).reshape(nb * bs, hkv, d)[slots])
    k8 = torch.full((nb, hkv, bs, d), 0x7f, dtype=torch.uint8, device="cuda")
    v8 = torch.full_like(k8, 0x7f)
    ks = torch.full((nb, hkv, bs), float("nan"), device="cuda")
    vs = torch.full_like(ks, float("nan"))
    pkv.pkv_append_e4m3(gh.dev(rows_k, BF16), gh.dev(rows_v, BF16), torch.from_numpy(slots).cuda(), k8, ks, v8, vs)
    q = gh.dev(w.q, BF16)
    out = torch.empty_like(q)
    pkv.pkv_decode_attention_e4m3(q, k8, ks, v8, vs, torch.from_numpy(w.block_tables).cuda(),
                                  torch.from_numpy(lens).cuda(), w.scale, out, gh.workspace_for(w, 0), 0)
    torch.cuda.synchronize()
    assert pkv.pkv_get_last_error() == pkv.PKV_OK
    ok8 = np.full((nb, hkv, bs, d), 0x7f, np.uint8)
    ov8 = ok8.copy()
    oks = np.full((nb, hkv, bs), np.nan, np.float32)
    ovs = oks.copy()
    oracle.append_e4m3(ok8, oks, rows_k, BF16, slots)
    oracle.append_e4m3(ov8, ovs, rows_v, BF16, slots)
    assert np.array_equal(k8.cpu().numpy(), ok8)
    ref = oracle.attention_e4m3(w.q, BF16, ok8, oks, ov8, ovs, w.block_tables, lens, w.scale)
    gh.assert_close(gh.to_f64(out), ref, BF16, "e4m3 pipeline")
    # and within the expected quantization distance of the bf16 result
    ref16 = oracle.attention(w.q, w.k_cache, w.v_cache, w.block_tables, lens, w.scale, BF16)
    assert np.max(np.abs(ref - ref16)) < 0.1
