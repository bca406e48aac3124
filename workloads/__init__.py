"""Seeded synthetic inputs for paged-KV decode attention.

This module is the only thing the CUDA path and the fp64 oracle both consume.
It draws random numbers and builds structure (context lengths, which physical
blocks each sequence owns, which blocks a group shares); it holds none of the
method's arithmetic -- no position-to-slot address, no attention.

Every float tensor is returned as raw 16-bit patterns (``np.uint16``): values
are drawn as N(0, 1) fp32 with ``numpy.random.default_rng(seed)`` and rounded
to fp16 / bf16 with round-to-nearest-even.  Both pools are filled with random
values everywhere; tests that want unused slots poisoned do so themselves.

Named workloads (shapes from the pages' own examples):

* ``tiny``          -- 4 sequences, context {17, 33, 64, 100}, 4/4 heads, D 64,
                       block 16, 64-block pool, fp16.
* ``llama13b``      -- 13B-shaped layer: 32 x 2048 context, 40/40 heads, D 128,
                       block 16, fp16 ("13B parameter model with a 2048-token
                       context window and a batch size of 32", adilsher.pro post,
                       "The Problem Nobody Mentions: KV-Cache Isn't Free").
* ``llama70b_gqa``  -- 70B-shaped GQA layer: 30 x 4096, 64/8 heads, D 128,
                       block 16, bf16, pool of 38 GiB / 80 layers = 7782 blocks
                       (cariara.com page, "The KV cache" worked table).
* ``cb_mixed``      -- continuous-batching step: 256 sequences, context
                       log-uniform in [16, 8192], 32/8 heads, D 128, block 32,
                       fp16; groups of 16 share a 2048-token prefix's blocks.
* ``long_split``    -- 2 x 65536 context, 64/8 heads, D 128, block 16, bf16,
                       512-token partitions.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

F16, BF16 = 0, 1
DTYPE_NAMES = {F16: "f16", BF16: "bf16"}


@dataclasses.dataclass(frozen=True)
class Spec:
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: int
    seed: int
    # context lengths: a fixed list, a single value, or log-uniform bounds
    context_lens: Optional[tuple] = None
    context_len: Optional[int] = None
    log_uniform: Optional[tuple] = None
    # pool: explicit block count, or "used + spare_per_seq * num_seqs"
    num_blocks: Optional[int] = None
    spare_per_seq: int = 1
    # prefix sharing: groups of `share_group` sequences share up to
    # `share_prefix_tokens` tokens of full blocks
    share_group: int = 0
    share_prefix_tokens: int = 0
    # partition size (tokens) the workload is specified with, 0 = none
    partition_tokens: int = 0
    description: str = ""


CONFIGS = {
    "tiny": Spec("tiny", 4, 4, 4, 64, 16, F16, seed=0, context_lens=(17, 33, 64, 100),
                 num_blocks=64,
                 description="tiny single layer: 4 seqs ctx {17,33,64,100}, MHA 4/4, D64, bs16, 64-block pool, fp16"),
    "llama13b": Spec("llama13b", 32, 40, 40, 128, 16, F16, seed=1, context_len=2048,
                     description="Llama-2-13B-shaped decode layer: 32 seqs x ctx 2048, 40/40 heads, D128, bs16, fp16"),
    "llama70b_gqa": Spec("llama70b_gqa", 30, 64, 8, 128, 16, BF16, seed=2, context_len=4096,
                         num_blocks=7782,
                         description="70B-shaped GQA decode layer: 30 seqs x ctx 4096, 64/8 heads, D128, bs16, bf16, 7782-block pool"),
    "cb_mixed": Spec("cb_mixed", 256, 32, 8, 128, 32, F16, seed=3, log_uniform=(16, 8192),
                     share_group=16, share_prefix_tokens=2048,
                     description="continuous-batching step: 256 seqs, ctx log-uniform [16,8192], 32/8 heads, D128, bs32, fp16, groups of 16 share a 2048-token prefix"),
    "long_split": Spec("long_split", 2, 64, 8, 128, 16, BF16, seed=4, context_len=65536,
                       partition_tokens=512,
                       description="long-context split-KV: 2 seqs x ctx 65536, 64/8 heads, D128, bs16, bf16, 512-token partitions"),
}

ORDER = ["tiny", "llama13b", "llama70b_gqa", "cb_mixed", "long_split"]


def to_bits(x: np.ndarray, dtype: int) -> np.ndarray:
    """Round fp32 values to fp16 / bf16 (round-to-nearest-even) and return the bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == F16:
        return x.astype(np.float16).view(np.uint16)
    import torch  # CPU cast only; torch rounds fp32 -> bf16 to nearest even

    return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def nan_bits(dtype: int) -> int:
    """A quiet-NaN bit pattern of the 16-bit type."""
    return 0x7E00 if dtype == F16 else 0x7FC0


def _randn_bits(rng, shape, dtype, chunk=1 << 26) -> np.ndarray:
    """N(0,1) fp32 draws rounded to 16 bits, generated in chunks to bound host memory."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        out[s:e] = to_bits(rng.standard_normal(e - s, dtype=np.float32), dtype)
    return out.reshape(shape)


@dataclasses.dataclass
class Workload:
    spec: Spec
    context_lens: np.ndarray      # int32 [B]  (after this step's append)
    block_tables: np.ndarray      # int32 [B][MB], unused entries -1
    num_blocks: int
    owned_blocks: list            # per sequence: list of physical ids, logical order
    shared_blocks: list           # per sequence: how many leading entries are shared
    q: np.ndarray                 # uint16 [B][Hq][D]
    k_cache: np.ndarray           # uint16 [NB][Hkv][bs][D]
    v_cache: np.ndarray           # uint16 [NB][Hkv][bs][D]
    k_new: np.ndarray             # uint16 [B][Hkv][D]
    v_new: np.ndarray             # uint16 [B][Hkv][D]
    scale: float                  # fp32 value 1/sqrt(D)

    @property
    def max_blocks_per_seq(self) -> int:
        return self.block_tables.shape[1]


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def context_lengths(spec: Spec, rng) -> np.ndarray:
    if spec.context_lens is not None:
        return np.array(spec.context_lens, dtype=np.int32)
    if spec.context_len is not None:
        return np.full(spec.num_seqs, spec.context_len, dtype=np.int32)
    lo, hi = spec.log_uniform
    u = rng.uniform(math.log(lo), math.log(hi), size=spec.num_seqs)
    return np.clip(np.floor(np.exp(u)), lo, hi).astype(np.int32)


def assign_blocks(spec: Spec, ctx: np.ndarray, rng):
    """Decide which physical blocks each sequence owns (logical order).

    A sequence with context c owns ceil(c / bs) blocks.  With sharing, the
    sequences of a group share the leading min(P, floor((c-1)/bs)) full blocks
    of one prefix (P = prefix tokens / bs); only full blocks are shared, so the
    block that receives this step's token is always private.  Physical ids are
    drawn in order from a seeded random permutation of the pool."""
    bs = spec.block_size
    nblk = [_ceil_div(int(c), bs) for c in ctx]
    nshared = [0] * len(ctx)
    group_prefix = {}
    if spec.share_group:
        pmax = spec.share_prefix_tokens // bs
        for s, c in enumerate(ctx):
            nshared[s] = min(pmax, (int(c) - 1) // bs)
        for s in range(len(ctx)):
            g = s // spec.share_group
            group_prefix[g] = max(group_prefix.get(g, 0), nshared[s])
    used = sum(group_prefix.values()) + sum(n - k for n, k in zip(nblk, nshared))
    nb = spec.num_blocks if spec.num_blocks is not None else used + spec.spare_per_seq * len(ctx)
    if nb < used:
        raise ValueError(f"{spec.name}: pool of {nb} blocks < {used} needed")
    perm = rng.permutation(nb).astype(np.int32)
    cursor = 0
    prefix_ids = {}
    for g in sorted(group_prefix):
        prefix_ids[g] = perm[cursor:cursor + group_prefix[g]].tolist()
        cursor += group_prefix[g]
    owned = []
    for s in range(len(ctx)):
        ids = []
        if spec.share_group:
            ids = prefix_ids[s // spec.share_group][:nshared[s]]
        k = nblk[s] - nshared[s]
        ids = list(ids) + perm[cursor:cursor + k].tolist()
        cursor += k
        owned.append(ids)
    return nb, owned, nshared


def make(spec_or_name, seed: Optional[int] = None, fill_pool: bool = True) -> Workload:
    """Build the seeded workload.  Draw order: context lengths, block
    permutation, q, K pool, V pool, k_new, v_new."""
    spec = CONFIGS[spec_or_name] if isinstance(spec_or_name, str) else spec_or_name
    rng = np.random.default_rng(spec.seed if seed is None else seed)
    ctx = context_lengths(spec, rng)
    nb, owned, nshared = assign_blocks(spec, ctx, rng)
    mb = max(1, max(len(o) for o in owned))
    tables = np.full((spec.num_seqs, mb), -1, dtype=np.int32)
    for s, ids in enumerate(owned):
        tables[s, :len(ids)] = ids
    b, hq, hkv, d, bs = spec.num_seqs, spec.num_q_heads, spec.num_kv_heads, spec.head_dim, spec.block_size
    q = _randn_bits(rng, (b, hq, d), spec.dtype)
    if fill_pool:
        kc = _randn_bits(rng, (nb, hkv, bs, d), spec.dtype)
        vc = _randn_bits(rng, (nb, hkv, bs, d), spec.dtype)
    else:
        kc = np.zeros((nb, hkv, bs, d), dtype=np.uint16)
        vc = np.zeros((nb, hkv, bs, d), dtype=np.uint16)
    kn = _randn_bits(rng, (b, hkv, d), spec.dtype)
    vn = _randn_bits(rng, (b, hkv, d), spec.dtype)
    scale = float(np.float32(1.0) / np.sqrt(np.float32(d)))
    return Workload(spec, ctx, tables, nb, owned, nshared, q, kc, vc, kn, vn, scale)


def custom(name: str, num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
           block_size: int, dtype: int, seed: int, context_lens, **kw) -> Spec:
    """A small spec for parity tests (explicit per-sequence context lengths)."""
    return Spec(name, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, dtype, seed,
                context_lens=tuple(int(c) for c in context_lens), **kw)
