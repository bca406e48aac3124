"""Shared helpers of the GPU parity tests: run one decode step through the
C ABI (append + attention) and the same step through the fp64 oracle on the
same seeded inputs, then compare.

Tolerances (fp32 accumulation against fp64): max |err| <= 2e-3 for fp16 and
<= 1.5e-2 for bf16; where the output's own rounding step is larger than that
(|out| >= 4 in fp16, >= 2 in bf16 -- only at tiny contexts) one unit in the
last place of the output type at the oracle's value is allowed instead.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import paged_kv_cache_437_b200 as pkv
import workloads

TOL = {workloads.F16: 2e-3, workloads.BF16: 1.5e-2}
MANTISSA = {workloads.F16: 10, workloads.BF16: 7}


def tdtype(dtype: int):
    return torch.float16 if dtype == workloads.F16 else torch.bfloat16


def dev(bits: np.ndarray, dtype: int) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(tdtype(dtype)).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def allowed_error(ref: np.ndarray, dtype: int) -> np.ndarray:
    mag = np.abs(ref)
    ulp = np.where(mag > 0, np.exp2(np.floor(np.log2(np.maximum(mag, 1e-300))) - MANTISSA[dtype]), 0.0)
    return np.maximum(TOL[dtype], ulp)


def assert_close(got: np.ndarray, ref: np.ndarray, dtype: int, what: str = "") -> float:
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite GPU output"
    err = np.abs(got - ref)
    bad = err > allowed_error(ref, dtype)
    assert not bad.any(), f"{what}: {bad.sum()} elements out of tolerance, max |err| {err.max():.3e}"
    return float(err.max())


def prepare(w: workloads.Workload, poison: bool = True):
    """Host copies of the pools with every slot outside the prior context
    (positions < ctx-1 of some sequence) set to NaN, and the slot of each
    sequence's new token (position ctx-1; -1 when ctx == 0)."""
    bs, nb = w.spec.block_size, w.num_blocks
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    prior = np.maximum(w.context_lens - 1, 0)
    if poison:
        mask = oracle.slot_mask(w.block_tables, prior, bs, nb).reshape(nb, 1, bs, 1)
        where = np.broadcast_to(~mask, kc.shape)
        nan = np.uint16(workloads.nan_bits(w.spec.dtype))
        np.copyto(kc, nan, where=where)
        np.copyto(vc, nan, where=where)
    slots = oracle.slot_mapping(w.block_tables, w.context_lens.astype(np.int64) - 1, bs)
    return kc, vc, slots


def workspace_for(w: workloads.Workload, partition: int):
    if partition == pkv.PKV_PARTITION_NONE:
        return None
    n = pkv.pkv_decode_workspace_bytes(w.spec.num_seqs, w.spec.num_q_heads, w.spec.num_kv_heads,
                                       w.spec.head_dim, w.max_blocks_per_seq * w.spec.block_size, partition)
    assert n > 0
    return torch.empty(n, dtype=torch.uint8, device="cuda")


class GpuStep:
    """Device copies of one workload and the calls of one decode step."""

    def __init__(self, w: workloads.Workload, kc: np.ndarray, vc: np.ndarray, slots: np.ndarray):
        dt = w.spec.dtype
        self.w = w
        self.q = dev(w.q, dt)
        self.kc, self.vc = dev(kc, dt), dev(vc, dt)
        self.kn, self.vn = dev(w.k_new, dt), dev(w.v_new, dt)
        self.slots = torch.from_numpy(np.ascontiguousarray(slots, dtype=np.int64)).cuda()
        self.tables = torch.from_numpy(np.ascontiguousarray(w.block_tables)).cuda()
        self.lens = torch.from_numpy(np.ascontiguousarray(w.context_lens)).cuda()
        self.out = torch.empty_like(self.q)

    def append(self, stream=None):
        pkv.pkv_append(self.kn, self.vn, self.slots, self.kc, self.vc, stream)

    def decode(self, partition: int = pkv.PKV_PARTITION_AUTO, workspace=None, stream=None):
        pkv.pkv_decode_attention(self.q, self.kc, self.vc, self.tables, self.lens, self.w.scale, self.out,
                                 workspace, partition, stream)

    def run_fused(self, partition: int = pkv.PKV_PARTITION_AUTO):
        ws = workspace_for(self.w, partition)
        pkv.pkv_append_decode_attention(self.kn, self.vn, self.slots, self.q, self.kc, self.vc, self.tables,
                                        self.lens, self.w.scale, self.out, ws, partition)
        torch.cuda.synchronize()
        st = pkv.pkv_get_last_error()
        assert st == pkv.PKV_OK, pkv.pkv_status_string(st)
        return self.out

    def run(self, partition: int = pkv.PKV_PARTITION_AUTO):
        ws = workspace_for(self.w, partition)
        self.append()
        self.decode(partition, ws)
        torch.cuda.synchronize()
        st = pkv.pkv_get_last_error()
        assert st == pkv.PKV_OK, pkv.pkv_status_string(st)
        return self.out


def oracle_step(w: workloads.Workload, kc: np.ndarray, vc: np.ndarray, slots: np.ndarray, pairs=None):
    k2, v2 = kc.copy(), vc.copy()
    oracle.append(k2, w.k_new, slots)
    oracle.append(v2, w.v_new, slots)
    ref = oracle.attention(w.q, k2, v2, w.block_tables, w.context_lens, w.scale, w.spec.dtype, pairs=pairs)
    return ref, k2, v2


def sample_pairs(w: workloads.Workload, n: int = 64, seed: int = 0) -> np.ndarray:
    """>= n distinct (seq, head) pairs, always including the longest and the
    shortest sequence (every head group of each) and the last head."""
    rng = np.random.default_rng(seed)
    b, hq = w.spec.num_seqs, w.spec.num_q_heads
    chosen = set()
    for s in (int(np.argmax(w.context_lens)), int(np.argmin(w.context_lens))):
        for h in range(0, hq, max(1, hq // 8)):
            chosen.add((s, h))
        chosen.add((s, hq - 1))
    while len(chosen) < min(n, b * hq):
        chosen.add((int(rng.integers(b)), int(rng.integers(hq))))
    return np.array(sorted(chosen), dtype=np.int64)
