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


def _run_case(case, seed=None, scale=None, expect=pkv.PKV_OK):
    """Build one mixed batch, run pkv_prefill_attention on it and the fp64
    oracle on the same inputs; returns (GPU out, oracle out, K/V pools after
    the append on both sides)."""
    dtype, hq, hkv, d, bs, seqs = case
    rng = np.random.default_rng(70 + len(seqs) if seed is None else seed)
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
    if scale is None:
        scale = float(np.float32(1.0) / np.sqrt(np.float32(d)))

    k_ref, v_ref = kc.copy(), vc.copy()
    oracle.append(k_ref, kn, slots)
    oracle.append(v_ref, vn, slots)
    ref = oracle.prefill_attention(q, k_ref, v_ref, tables, qs, ctx, scale, dtype)

    kd, vd = gh.dev(kc, dtype), gh.dev(vc, dtype)
    pkv.pkv_append(gh.dev(kn, dtype), gh.dev(vn, dtype), torch.from_numpy(slots).cuda(), kd, vd)
    qd = gh.dev(q, dtype)
    out = torch.full_like(qd, float("nan"))
    ws = torch.empty(pkv.pkv_prefill_workspace_bytes(t, hq, hkv, d, mb * bs), dtype=torch.uint8, device="cuda")
    pkv.pkv_prefill_attention(qd, kd, vd, torch.from_numpy(tables).cuda(), torch.from_numpy(qs).cuda(),
                              torch.from_numpy(ctx).cuda(), scale, out, ws)
    torch.cuda.synchronize()
    st = pkv.pkv_get_last_error()
    assert st == expect, pkv.pkv_status_string(st)
    return out, ref, (gh.host_bits(kd), gh.host_bits(vd)), (k_ref, v_ref)


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{workloads.DTYPE_NAMES[c[0]]}_{c[1]}_{c[2]}_{c[3]}_bs{c[4]}")
def test_prefill_matches_oracle(case):
    out, ref, pools, pools_ref = _run_case(case)
    assert np.array_equal(pools[0], pools_ref[0]) and np.array_equal(pools[1], pools_ref[1])
    gh.assert_close(gh.to_f64(out), ref, case[0], "prefill")


# the multi-query tensor-core kernel's edge cases: chunks that are not a
# multiple of the row block, tails whose last tile runs past the context
# (V rows there are poisoned), one-tile and many-tile ranges, several chunks
# in one call, a chunk that is the whole context, the largest GQA group
MQ_CASES = [
    (BF16, 64, 8, 128, 16, [(129, 129), (4000, 300), (1, 1), (257, 2)]),
    (F16, 16, 4, 128, 32, [(1000, 999), (77, 3), (128, 128), (129, 1)]),
    (BF16, 128, 1, 128, 16, [(300, 20), (16, 16)]),
    (F16, 4, 4, 64, 32, [(700, 256), (255, 255), (90, 7)]),
    (BF16, 24, 8, 64, 16, [(513, 64), (2048, 1), (40, 40)]),
]


@pytest.mark.parametrize("case", MQ_CASES, ids=lambda c: f"{workloads.DTYPE_NAMES[c[0]]}_{c[1]}_{c[2]}_{c[3]}_bs{c[4]}")
def test_multi_query_kernel_edge_cases(case):
    out, ref, _, _ = _run_case(case, seed=5)
    gh.assert_close(gh.to_f64(out), ref, case[0], "prefill (multi-query kernel)")


@pytest.mark.parametrize("poly", ["1", "2", "3"])
def test_multi_query_kernel_fma_pipe_exponentials(poly, monkeypatch):
    # PKV_MQ_POLY=n: n of every 8 probability pairs by the FMA-pipe exp2
    # (relative error < 8e-6): the same tolerance as the SFU path
    monkeypatch.setenv("PKV_MQ_POLY", poly)
    for case in (MQ_CASES[0], MQ_CASES[1]):
        out, ref, _, _ = _run_case(case, seed=9)
        gh.assert_close(gh.to_f64(out), ref, case[0], f"prefill, PKV_MQ_POLY={poly}")


def test_negative_scale():
    case = (F16, 32, 8, 128, 16, [(600, 200), (50, 1)])
    out, ref, _, _ = _run_case(case, seed=6, scale=-0.07)
    gh.assert_close(gh.to_f64(out), ref, F16, "prefill, negative scale")


def test_multi_query_kernel_matches_the_per_token_path(monkeypatch):
    case = (BF16, 64, 8, 128, 16, [(1500, 400), (300, 1)])
    out_mq, ref, _, _ = _run_case(case, seed=7)
    monkeypatch.setenv("PKV_PREFILL_MQ", "0")
    out_tok, _, _, _ = _run_case(case, seed=7)
    gh.assert_close(gh.to_f64(out_mq), ref, BF16, "multi-query kernel")
    gh.assert_close(gh.to_f64(out_tok), ref, BF16, "per-token decode path")


def test_multi_query_wait_timeout_is_reported_and_recovers():
    case = (BF16, 64, 8, 128, 16, [(700, 300)])
    pkv.pkv_test_inject_wait_timeout(True, 20_000_000)   # 20 ms
    try:
        _run_case(case, seed=8, expect=pkv.PKV_ERR_TIMEOUT)
    finally:
        pkv.pkv_test_inject_wait_timeout(False)
    assert pkv.pkv_get_last_error() == pkv.PKV_OK  # read and cleared above
    out, ref, _, _ = _run_case(case, seed=8)
    gh.assert_close(gh.to_f64(out), ref, BF16, "prefill after a time-out")


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
