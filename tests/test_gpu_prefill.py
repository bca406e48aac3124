"""Chunked prefill on the GPU against the oracle: mixed batches of decode
tokens (chunks of one) and prefill chunks, the chunks' K/V appended with
pkv_append first, every slot outside the attended context NaN-poisoned."""
import numpy as np
import pytest
import torch

import gpu_harness as gh
import oracle
import paged_kv_cache_437_b200 as pkv
import workloads
from workloads import BF16, F16

pytestmark = pytest.mark.gpu

CASES = [
    # (dtype, Hq, Hkv, D, bs, [(context after the chunk, chunk length)])
    (BF16, 64, 8, 128, 16, [(2048 + 512, 512), (300, 1), (1000, 1), (33, 33)]),
    (F16, 32, 8, 128, 32, [(100, 17), (5, 5), (4097, 1), (640, 128)]),
    (F16, 8, 8, 64, 16, [(1, 1), (70, 64), (17, 2)]),
    (BF16, 32, 2, 128, 16, [(513, 500), (16, 16)]),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{workloads.DTYPE_NAMES[c[0]]}_{c[1]}_{c[2]}_{c[3]}_bs{c[4]}")
def test_prefill_matches_oracle(case):
    dtype, hq, hkv, d, bs, seqs = case
    rng = np.random.default_rng(70 + len(seqs))
    ctx = np.array([c for c, _ in seqs], dtype=np.int32)
    nq = np.array([n for _, n in seqs], dtype=np.int32)
    qs = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    t = int(qs[-1])
    nblk = -(-ctx // bs)
    mb = int(nblk.max())
    nb = int(nblk.sum()) + 3
    perm = rng.permutation(nb).astype(np.int32)
    tables = np.full((len(seqs), mb), -1, dtype=np.int32)
    cur = 0
    for s, k in enumerate(nblk):
        tables[s, :k] = perm[cur:cur + k]
        cur += k
    kc = workloads.to_bits(rng.standard_normal((nb, hkv, bs, d), dtype=np.float32), dtype)
    vc = workloads.to_bits(rng.standard_normal((nb, hkv, bs, d), dtype=np.float32), dtype)
    # poison everything but the prior context (positions < ctx - n)
    mask = oracle.slot_mask(tables, ctx - nq, bs, nb).reshape(nb, 1, bs, 1)
    nan = np.uint16(workloads.nan_bits(dtype))
    np.copyto(kc, nan, where=np.broadcast_to(~mask, kc.shape))
    np.copyto(vc, nan, where=np.broadcast_to(~mask, vc.shape))
    kn = workloads.to_bits(rng.standard_normal((t, hkv, d), dtype=np.float32), dtype)
    vn = workloads.to_bits(rng.standard_normal((t, hkv, d), dtype=np.float32), dtype)
    q = workloads.to_bits(rng.standard_normal((t, hq, d), dtype=np.float32), dtype)
    slots = np.concatenate([oracle.slot_mapping(np.repeat(tables[s:s + 1], nq[s], axis=0),
                                                np.arange(ctx[s] - nq[s], ctx[s]), bs)
                            for s in range(len(seqs))]).astype(np.int64)
    scale = float(np.float32(1.0) / np.sqrt(np.float32(d)))

    k_ref, v_ref = kc.copy(), vc.copy()
    oracle.append(k_ref, kn, slots)
    oracle.append(v_ref, vn, slots)
    ref = oracle.prefill_attention(q, k_ref, v_ref, tables, qs, ctx, scale, dtype)

    kd, vd = gh.dev(kc, dtype), gh.dev(vc, dtype)
    pkv.pkv_append(gh.dev(kn, dtype), gh.dev(vn, dtype), torch.from_numpy(slots).cuda(), kd, vd)
    qd = gh.dev(q, dtype)
    out = torch.empty_like(qd)
    ws = torch.empty(pkv.pkv_prefill_workspace_bytes(t, hq, hkv, d, mb * bs), dtype=torch.uint8, device="cuda")
    pkv.pkv_prefill_attention(qd, kd, vd, torch.from_numpy(tables).cuda(), torch.from_numpy(qs).cuda(),
                              torch.from_numpy(ctx).cuda(), scale, out, ws)
    torch.cuda.synchronize()
    assert pkv.pkv_get_last_error() == pkv.PKV_OK
    assert np.array_equal(gh.host_bits(kd), k_ref) and np.array_equal(gh.host_bits(vd), v_ref)
    gh.assert_close(gh.to_f64(out), ref, dtype, "prefill")


def test_prefill_flags_inconsistent_lengths():
    dtype, hq, hkv, d, bs = F16, 8, 8, 64, 16
    kc = torch.zeros((4, hkv, bs, d), dtype=torch.float16, device="cuda")
    tables = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
    qs = torch.tensor([0, 8], dtype=torch.int32, device="cuda")
    ctx = torch.tensor([5], dtype=torch.int32, device="cuda")    # chunk of 8 > context 5
    q = torch.zeros((8, hq, d), dtype=torch.float16, device="cuda")
    out = torch.ones_like(q)
    ws = torch.empty(pkv.pkv_prefill_workspace_bytes(8, hq, hkv, d, 2 * bs), dtype=torch.uint8, device="cuda")
    pkv.pkv_prefill_attention(q, kc, kc, tables, qs, ctx, 0.1, out, ws)
    assert pkv.pkv_get_last_error() == pkv.PKV_ERR_DEVICE_CHECK
    assert torch.count_nonzero(out) == 0
    del dtype
