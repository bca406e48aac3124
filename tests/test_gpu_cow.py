"""Copy-on-write on the GPU: a child forked in the middle of a block shares
the parent's blocks; appends through the copy-on-write allocator calls plus
pkv_copy_blocks + pkv_append, then decode of both sequences, against the
oracle replaying the same block copies and appends on host pools."""
import numpy as np
import pytest
import torch

import gpu_harness as gh
import oracle
import paged_kv_cache_437_b200 as pkv
import workloads

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [workloads.F16, workloads.BF16])
@pytest.mark.parametrize("fork_at", [37, 32, 1])
def test_fork_cow_append_decode(dtype, fork_at):
    rng = np.random.default_rng(50 + fork_at)
    nb, hkv, hq, bs, d = 24, 2, 8, 16, 128
    alloc = pkv.BlockAllocator(nb, bs)
    k_host = workloads.to_bits(rng.standard_normal((nb, hkv, bs, d), dtype=np.float32), dtype)
    v_host = workloads.to_bits(rng.standard_normal((nb, hkv, bs, d), dtype=np.float32), dtype)
    kc, vc = gh.dev(k_host, dtype), gh.dev(v_host, dtype)
    k_ref, v_ref = k_host.copy(), v_host.copy()

    def new_tokens(n):
        kn = workloads.to_bits(rng.standard_normal((n, hkv, d), dtype=np.float32), dtype)
        vn = workloads.to_bits(rng.standard_normal((n, hkv, d), dtype=np.float32), dtype)
        return kn, vn

    def append_step(seqs):
        slots, copies = alloc.append_slots_cow(seqs)
        if len(copies):
            pkv.pkv_copy_blocks(kc, vc, torch.from_numpy(copies).cuda())
            oracle.copy_blocks(k_ref, copies)
            oracle.copy_blocks(v_ref, copies)
        kn, vn = new_tokens(len(seqs))
        pkv.pkv_append(gh.dev(kn, dtype), gh.dev(vn, dtype), torch.from_numpy(slots).cuda(), kc, vc)
        oracle.append(k_ref, kn, slots)
        oracle.append(v_ref, vn, slots)
        return len(copies)

    parent = alloc.seq_create()
    for _ in range(40):
        append_step([parent])
    child = alloc.seq_fork_tokens(parent, fork_at)
    n_copies = 0
    for step in range(3):
        n_copies += append_step([child, parent] if step < 2 else [child])
    assert n_copies == (1 if fork_at % bs else 0)
    seqs = [parent, child]
    tables, lens = alloc.batch_tables(seqs, 4)
    q_bits = workloads.to_bits(rng.standard_normal((2, hq, d), dtype=np.float32), dtype)
    out = torch.empty((2, hq, d), dtype=gh.tdtype(dtype), device="cuda")
    pkv.pkv_decode_attention(gh.dev(q_bits, dtype), kc, vc, torch.from_numpy(tables).cuda(),
                             torch.from_numpy(lens).cuda(), 0.088, out, None, pkv.PKV_PARTITION_NONE)
    torch.cuda.synchronize()
    assert pkv.pkv_get_last_error() == pkv.PKV_OK
    assert np.array_equal(gh.host_bits(kc), k_ref) and np.array_equal(gh.host_bits(vc), v_ref)
    ref = oracle.attention(q_bits, k_ref, v_ref, tables, lens, 0.088, dtype)
    gh.assert_close(gh.to_f64(out), ref, dtype, f"cow fork_at={fork_at}")
    # the parent's shared prefix was never written by the child
    assert lens.tolist() == [42, fork_at + 3]


def test_copy_blocks_bit_exact_and_checked():
    rng = np.random.default_rng(60)
    nb, hkv, bs, d = 12, 4, 32, 64
    k_host = rng.integers(0, 65535, size=(nb, hkv, bs, d), dtype=np.uint16)
    v_host = rng.integers(0, 65535, size=(nb, hkv, bs, d), dtype=np.uint16)
    kc, vc = gh.dev(k_host, workloads.F16), gh.dev(v_host, workloads.F16)
    pairs = np.array([[0, 5], [7, 2], [3, 11]], dtype=np.int32)
    pkv.pkv_copy_blocks(kc, vc, torch.from_numpy(pairs).cuda())
    torch.cuda.synchronize()
    oracle.copy_blocks(k_host, pairs)
    oracle.copy_blocks(v_host, pairs)
    assert np.array_equal(gh.host_bits(kc), k_host) and np.array_equal(gh.host_bits(vc), v_host)
    assert pkv.pkv_get_last_error() == pkv.PKV_OK
    bad = torch.tensor([[1, nb + 3]], dtype=torch.int32, device="cuda")
    pkv.pkv_copy_blocks(kc, vc, bad)
    assert pkv.pkv_get_last_error() == pkv.PKV_ERR_DEVICE_CHECK
    assert np.array_equal(gh.host_bits(kc), k_host)
