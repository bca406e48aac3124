"""Pins of the fp64 oracle against things other than itself.

Each ``check_*`` function takes an oracle library handle (the real one, or a
deliberately mutated build in ``test_oracle_mutations.py``) and raises
``AssertionError`` when the oracle disagrees with:

* library routines (numpy's float16 and torch's bfloat16 decoders,
  ``scipy.special.softmax`` on an unpaged contiguous cache),
* closed forms (one position returns V; equal scores average V; scores 0 and
  ln 3 weigh 1:3; a constant V per KV head pins the query-head -> KV-head map),
* brute force on tiny inputs (slot addresses enumerated block by block),
* invariants (physical block permutation, shared vs duplicated prefix blocks,
  NaN-poisoned unused slots, V scaled by 2, split + log-sum-exp merge),
* the pages' worked sizing example (``tests/golden/kv_sizing_worked_example.txt``).
"""
from __future__ import annotations

import math
import os

import numpy as np
import scipy.special

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_golden(name: str) -> dict:
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = line.split()
                vals[k] = int(v)
    return vals


# ---------------------------------------------------------------- helpers

def f16_bits(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def bf16_bits(x) -> np.ndarray:
    import torch

    t = torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(bits: np.ndarray, dtype: int) -> np.ndarray:
    """Library decode (numpy / torch), independent of the oracle's decoder."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    if dtype == oracle.F16:
        return bits.view(np.float16).astype(np.float64)
    import torch

    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()


def contiguous_to_pool(k_seq: np.ndarray, block_size: int) -> np.ndarray:
    """Unpaged per-sequence caches [B][Hkv][n][D] -> pool [B*n/bs][Hkv][bs][D]
    with sequence s owning blocks s*n/bs ... (s+1)*n/bs - 1 in order.
    Built with reshape / transpose only, not with a position -> slot formula."""
    b, hkv, n, d = k_seq.shape
    nb = n // block_size
    return np.ascontiguousarray(
        k_seq.reshape(b, hkv, nb, block_size, d).transpose(0, 2, 1, 3, 4).reshape(b * nb, hkv, block_size, d))


def textbook(qd, kd, vd, scale, ctx):
    """scipy softmax(scale * K q) V on unpaged caches; qd [B][Hq][D], kd/vd [B][Hkv][n][D]."""
    b, hq, d = qd.shape
    hkv = kd.shape[1]
    grp = hq // hkv
    out = np.zeros((b, hq, d))
    for s in range(b):
        for h in range(hq):
            kk = kd[s, h // grp, :ctx[s]]
            vv = vd[s, h // grp, :ctx[s]]
            p = scipy.special.softmax(scale * (kk @ qd[s, h]))
            out[s, h] = p @ vv
    return out


def _rand_case(rng, b, hq, hkv, d, n, dtype):
    mk = f16_bits if dtype == oracle.F16 else bf16_bits
    q = mk(rng.standard_normal((b, hq, d)))
    k = mk(rng.standard_normal((b, hkv, n, d)))
    v = mk(rng.standard_normal((b, hkv, n, d)))
    return q, k, v


# ---------------------------------------------------------------- checks

def check_decoders(lib):
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    for dtype, f in ((oracle.F16, lib.oracle_half_to_double), (oracle.BF16, lib.oracle_bf16_to_double)):
        ref = bits_to_f64(allbits, dtype)
        got = np.array([f(int(x)) for x in allbits])
        nan = np.isnan(ref)
        assert np.array_equal(np.isnan(got), nan), "NaN set differs"
        assert np.array_equal(got[~nan], ref[~nan]), f"decoder {dtype} differs from library"


def check_sizing_golden(lib):
    g = read_golden("kv_sizing_worked_example.txt")
    per_tok = lib.oracle_kv_bytes_per_layer(1, g["kv_heads"], g["head_dim"], g["dtype_bytes"])
    assert per_tok == g["per_layer_bytes_per_token"]
    for seq_len in (1, 7, 2048, 4096):
        assert lib.oracle_kv_bytes_per_layer(seq_len, g["kv_heads"], g["head_dim"], g["dtype_bytes"]) == \
            g["per_layer_bytes_per_token"] * seq_len
    assert per_tok * g["layers"] == g["per_token_all_layers_bytes"]
    req = lib.oracle_kv_bytes_per_layer(g["request_tokens"], g["kv_heads"], g["head_dim"], g["dtype_bytes"]) * g["layers"]
    assert req == g["request_bytes"]
    assert req == g["request_mib"] * 2 ** 20
    assert g["hbm_total_gb"] - g["weights_gb"] == g["kv_budget_gib"]
    budget = g["kv_budget_gib"] * 2 ** 30
    assert budget // req == g["concurrent_requests"]
    blk = lib.oracle_kv_bytes_per_layer(g["block_size"], g["kv_heads"], g["head_dim"], g["dtype_bytes"])
    blocks = budget // g["layers"] // blk
    assert blocks == g["pool_blocks_per_layer"]
    assert blocks >= g["concurrent_requests"] * g["request_tokens"] // g["block_size"]


def check_textbook(lib, dtype=oracle.F16):
    """Oracle on a paged pool equals scipy softmax on the unpaged caches."""
    rng = np.random.default_rng(11)
    b, hq, hkv, d, bs, n = 3, 8, 2, 16, 4, 12
    q, k, v = _rand_case(rng, b, hq, hkv, d, n, dtype)
    ctx = np.array([12, 5, 1], dtype=np.int32)
    scale = 0.3
    kd, vd, qd = bits_to_f64(k, dtype), bits_to_f64(v, dtype), bits_to_f64(q, dtype)
    ref = textbook(qd, kd, vd, scale, ctx)
    tables = np.arange(b * n // bs, dtype=np.int32).reshape(b, n // bs)
    got = oracle.attention(q, contiguous_to_pool(k, bs), contiguous_to_pool(v, bs), tables, ctx,
                           scale, dtype, lib=lib)
    assert np.max(np.abs(got - ref)) < 1e-12, np.max(np.abs(got - ref))
    # one block per sequence (block size = whole context)
    got1 = oracle.attention(q, contiguous_to_pool(k, n), contiguous_to_pool(v, n),
                            np.arange(b, dtype=np.int32).reshape(b, 1), ctx, scale, dtype, lib=lib)
    assert np.max(np.abs(got1 - ref)) < 1e-12


def check_closed_forms(lib):
    d = 4
    # one position: output is V exactly
    rng = np.random.default_rng(3)
    q = f16_bits(rng.standard_normal((1, 1, d)))
    k = f16_bits(rng.standard_normal((1, 1, 1, d)))
    v = f16_bits(rng.standard_normal((1, 1, 1, d)))
    out = oracle.attention(q, k, v, np.zeros((1, 1), np.int32), np.array([1], np.int32), 0.5, oracle.F16, lib=lib)
    assert np.array_equal(out[0, 0], bits_to_f64(v[0, 0, 0], oracle.F16))
    # equal scores: the mean of V
    kk = f16_bits(np.tile([[0.5, -1.0, 2.0, 0.25]], (3, 1))).reshape(1, 1, 3, d)
    vv = f16_bits([[1.0, 2.0, 3.0, 4.0], [-1.0, 0.0, 5.0, 8.0], [3.0, 1.0, -2.0, 0.0]]).reshape(1, 1, 3, d)
    out = oracle.attention(q, kk, vv, np.zeros((1, 1), np.int32), np.array([3], np.int32), 0.7, oracle.F16, lib=lib)
    assert np.allclose(out[0, 0], [1.0, 1.0, 2.0, 4.0], atol=1e-15, rtol=0)
    # zero query: the mean of V whatever the keys
    q0 = f16_bits(np.zeros((1, 1, d)))
    kr = f16_bits(rng.standard_normal((1, 1, 3, d)))
    out = oracle.attention(q0, kr, vv, np.zeros((1, 1), np.int32), np.array([3], np.int32), 1.0, oracle.F16, lib=lib)
    assert np.allclose(out[0, 0], [1.0, 1.0, 2.0, 4.0], atol=1e-15, rtol=0)
    # scores 0 and ln 3: weights 1/4 and 3/4
    qe = f16_bits([[[1.0, 0.0, 0.0, 0.0]]])
    k2 = f16_bits([[0.0, 0.0, 0.0, 0.0], [1.0, 0.0, 0.0, 0.0]]).reshape(1, 1, 2, d)
    v2 = f16_bits([[4.0, 0.0, -8.0, 1.0], [0.0, 4.0, 8.0, 1.0]]).reshape(1, 1, 2, d)
    sc = float(np.float32(math.log(3.0)))
    out = oracle.attention(qe, k2, v2, np.zeros((1, 1), np.int32), np.array([2], np.int32), sc, oracle.F16, lib=lib)
    assert np.allclose(out[0, 0], [1.0, 3.0, 4.0, 1.0], atol=1e-6, rtol=0), out
    # scores 0, ln 2, 2 ln 2: weights 1/7, 2/7, 4/7
    k3 = f16_bits([[0, 0, 0, 0], [1, 0, 0, 0], [2, 0, 0, 0]]).reshape(1, 1, 3, d)
    v3 = f16_bits([[7, 0, 0, 0], [0, 7, 0, 0], [0, 0, 7, 0]]).reshape(1, 1, 3, d)
    s2 = float(np.float32(math.log(2.0)))
    out = oracle.attention(qe, k3, v3, np.zeros((1, 1), np.int32), np.array([3], np.int32), s2, oracle.F16, lib=lib)
    assert np.allclose(out[0, 0], [1.0, 2.0, 4.0, 0.0], atol=1e-6, rtol=0), out
    # hand dot products: q = (1,2,3,4), k0 = e1 -> 1, k1 = e4 -> 4, scale 1
    qh = f16_bits([[[1.0, 2.0, 3.0, 4.0]]])
    kh = f16_bits([[1, 0, 0, 0], [0, 0, 0, 1]]).reshape(1, 1, 2, d)
    vh = f16_bits([[1, 0, 0, 0], [0, 1, 0, 0]]).reshape(1, 1, 2, d)
    out = oracle.attention(qh, kh, vh, np.zeros((1, 1), np.int32), np.array([2], np.int32), 1.0, oracle.F16, lib=lib)
    w1 = 1.0 / (1.0 + math.exp(-3.0))
    assert np.allclose(out[0, 0], [1.0 - w1, w1, 0.0, 0.0], atol=1e-15, rtol=0)
    # a dominant score selects its V
    kd = f16_bits([[0, 0, 0, 0], [60.0, 0, 0, 0], [0, 0, 0, 0]]).reshape(1, 1, 3, d)
    out = oracle.attention(qe, kd, v3, np.zeros((1, 1), np.int32), np.array([3], np.int32), 1.0, oracle.F16, lib=lib)
    assert np.allclose(out[0, 0], [0.0, 7.0, 0.0, 0.0], atol=1e-20, rtol=1e-20)


def check_gqa_map(lib):
    """Constant V per KV head: query head h must return KV head h / G's constant."""
    b, hq, hkv, d, bs, n = 2, 12, 3, 8, 4, 8
    grp = hq // hkv
    rng = np.random.default_rng(5)
    q = f16_bits(rng.standard_normal((b, hq, d)))
    k = f16_bits(rng.standard_normal((b, hkv, n, d)))
    vconst = np.zeros((b, hkv, n, d))
    for g in range(hkv):
        vconst[:, g] = g + 1
    v = f16_bits(vconst)
    tables = np.arange(b * n // bs, dtype=np.int32).reshape(b, n // bs)
    out = oracle.attention(q, contiguous_to_pool(k, bs), contiguous_to_pool(v, bs), tables,
                           np.array([n, 5], np.int32), 0.4, oracle.F16, lib=lib)
    for h in range(hq):
        assert np.allclose(out[:, h], h // grp + 1, atol=1e-13, rtol=0), (h, out[:, h, 0])


def check_slot_bruteforce(lib):
    rng = np.random.default_rng(8)
    bs, mb, b = 4, 5, 3
    tables = rng.permutation(40)[:b * mb].astype(np.int32).reshape(b, mb)
    for s in range(b):
        expected = {}
        pos = 0
        for blk in tables[s]:            # enumerate block by block, row by row
            for r in range(bs):
                expected[pos] = int(blk) * bs + r
                pos += 1
        for p, slot in expected.items():
            assert oracle.slot_of(tables[s], p, bs, lib=lib) == slot


def check_slot_mask(lib):
    """The attended-slot mask (which slots every GPU test leaves un-poisoned)
    against a brute-force enumeration: walk each sequence's table block by
    block and row by row, counting positions, and keep the first lens[s].
    Lengths 0, 1, bs, bs + 1 and a full table; two sequences share blocks."""
    rng = np.random.default_rng(11)
    bs, mb, nb = 4, 5, 40
    lens = np.array([0, 1, bs, bs + 1, mb * bs, 7, 13], np.int32)
    b = lens.size
    tables = np.full((b, mb), -1, np.int32)
    free = list(rng.permutation(nb))
    for s in range(b):
        need = -(-int(lens[s]) // bs)
        for j in range(need):
            tables[s, j] = free.pop()
    tables[6, :2] = tables[4, :2]          # a shared two-block prefix
    expected = np.zeros(nb * bs, bool)
    for s in range(b):
        pos = 0
        for blk in tables[s]:
            for r in range(bs):
                if pos < lens[s]:
                    expected[int(blk) * bs + r] = True
                pos += 1
    got = oracle.slot_mask(tables, lens, bs, nb, lib=lib)
    assert got.shape == expected.shape and np.array_equal(got, expected)
    # the mask of the lengths before one append leaves exactly the new slots out
    prior = np.maximum(lens - 1, 0)
    got_prior = oracle.slot_mask(tables, prior, bs, nb, lib=lib)
    new_slots = {int(tables[s, (lens[s] - 1) // bs]) * bs + int(lens[s] - 1) % bs for s in range(b) if lens[s] > 0}
    assert set(np.nonzero(got & ~got_prior)[0].tolist()) == new_slots - set(np.nonzero(got_prior)[0].tolist())


def check_append(lib, dtype=oracle.F16):
    rng = np.random.default_rng(9)
    nb, hkv, bs, d, t = 6, 3, 4, 8, 7
    pool = rng.integers(0, 65535, size=(nb, hkv, bs, d), dtype=np.uint16)
    before = pool.copy()
    new = rng.integers(0, 65535, size=(t, hkv, d), dtype=np.uint16)
    slots = np.array([0, 23, -1, 5, 17, -7, 9], dtype=np.int64)
    oracle.append(pool, new, slots, lib=lib)
    # expected via a slot-major view of the pool: [NB*bs][Hkv][D]
    exp = np.ascontiguousarray(before.transpose(0, 2, 1, 3)).reshape(nb * bs, hkv, d)
    for i, sl in enumerate(slots):
        if sl >= 0:
            exp[sl] = new[i]
    exp = exp.reshape(nb, bs, hkv, d).transpose(0, 2, 1, 3)
    assert np.array_equal(pool, exp)


def check_permutation_and_sharing(lib):
    rng = np.random.default_rng(12)
    b, hq, hkv, d, bs, n = 4, 4, 2, 8, 4, 16
    q, k, v = _rand_case(rng, b, hq, hkv, d, n, oracle.F16)
    ctx = np.array([16, 13, 9, 2], dtype=np.int32)
    kp, vp = contiguous_to_pool(k, bs), contiguous_to_pool(v, bs)
    tables = np.arange(b * n // bs, dtype=np.int32).reshape(b, n // bs)
    base = oracle.attention(q, kp, vp, tables, ctx, 0.35, oracle.F16, lib=lib)
    # move every physical block to perm[i] and remap the tables
    perm = rng.permutation(kp.shape[0])
    kq, vq = np.empty_like(kp), np.empty_like(vp)
    kq[perm], vq[perm] = kp, vp
    out = oracle.attention(q, kq, vq, perm[tables].astype(np.int32), ctx, 0.35, oracle.F16, lib=lib)
    assert np.array_equal(out, base)
    # sequence 1 shares sequence 0's first two blocks instead of holding copies
    k2, v2 = k.copy(), v.copy()
    k2[1, :, :8], v2[1, :, :8] = k[0, :, :8], v[0, :, :8]
    kp2, vp2 = contiguous_to_pool(k2, bs), contiguous_to_pool(v2, bs)
    dup = oracle.attention(q, kp2, vp2, tables, ctx, 0.35, oracle.F16, lib=lib)
    shared_tables = tables.copy()
    shared_tables[1, :2] = tables[0, :2]
    shr = oracle.attention(q, kp2, vp2, shared_tables, ctx, 0.35, oracle.F16, lib=lib)
    assert np.array_equal(shr, dup)
    assert not np.array_equal(dup[1], base[1])


def check_poison_and_scaling(lib):
    rng = np.random.default_rng(13)
    b, hq, hkv, d, bs, n = 2, 2, 1, 8, 4, 12
    q, k, v = _rand_case(rng, b, hq, hkv, d, n, oracle.F16)
    ctx = np.array([10, 3], dtype=np.int32)
    kp, vp = contiguous_to_pool(k, bs), contiguous_to_pool(v, bs)
    nb = kp.shape[0]
    # two extra free blocks at the end of the pool
    kp = np.concatenate([kp, np.zeros((2, hkv, bs, d), np.uint16)])
    vp = np.concatenate([vp, np.zeros((2, hkv, bs, d), np.uint16)])
    tables = np.arange(b * n // bs, dtype=np.int32).reshape(b, n // bs)
    base = oracle.attention(q, kp, vp, tables, ctx, 0.5, oracle.F16, lib=lib)
    # poison every slot a sequence does not attend, and the free blocks
    kpo, vpo = kp.copy(), vp.copy()
    mask = np.ones((b, hkv, n, d), bool)
    for s in range(b):
        mask[s, :, :ctx[s]] = False
    pm = contiguous_to_pool(mask.astype(np.uint16), bs).astype(bool)
    kpo[:nb][pm] = 0x7E00
    vpo[:nb][pm] = 0x7E00
    kpo[nb:] = 0x7E00
    vpo[nb:] = 0x7E00
    out = oracle.attention(q, kpo, vpo, tables, ctx, 0.5, oracle.F16, lib=lib)
    assert np.all(np.isfinite(out)) and np.array_equal(out, base)
    # V scaled by 2 (exact in fp16 here) scales the output by exactly 2
    v2 = f16_bits(bits_to_f64(v, oracle.F16) * 2.0)
    out2 = oracle.attention(q, kp, np.concatenate([contiguous_to_pool(v2, bs), vp[nb:]]), tables, ctx,
                            0.5, oracle.F16, lib=lib)
    assert np.array_equal(out2, 2.0 * base)


def check_split_merge(lib):
    rng = np.random.default_rng(14)
    b, hq, hkv, d, bs, n = 1, 4, 2, 16, 8, 64
    q, k, v = _rand_case(rng, b, hq, hkv, d, n, oracle.BF16)
    ctx = np.array([61], dtype=np.int32)
    kp, vp = contiguous_to_pool(k, bs), contiguous_to_pool(v, bs)
    tables = np.arange(n // bs, dtype=np.int32).reshape(1, -1)
    full = oracle.attention(q, kp, vp, tables, ctx, 0.25, oracle.BF16, lib=lib)
    for part in (8, 16, 24, 61, 100):
        for h in range(hq):
            ms, ls, os_ = [], [], []
            for lo in range(0, 128, part):          # trailing parts are empty
                m, l, o = oracle.attention_range(q, kp, vp, tables, 0.25, oracle.BF16, 0, h,
                                                 min(lo, 61), min(lo + part, 61), lib=lib)
                ms.append(m)
                ls.append(l)
                os_.append(o)
            merged = oracle.lse_merge(ms, ls, np.array(os_), lib=lib)
            assert np.max(np.abs(merged - full[0, h])) < 1e-12, (part, h)


def check_copy_blocks(lib):
    """Block copies against numpy fancy indexing, applied pair by pair."""
    rng = np.random.default_rng(15)
    pool = rng.integers(0, 65535, size=(7, 2, 4, 8), dtype=np.uint16)
    exp = pool.copy()
    pairs = np.array([[0, 3], [3, 5], [6, 0]], dtype=np.int32)
    oracle.copy_blocks(pool, pairs, lib=lib)
    for src, dst in pairs:
        exp[dst] = exp[src]
    assert np.array_equal(pool, exp)


def check_prefill(lib):
    """Chunked prefill: scipy softmax over each query's causal window on the
    unpaged caches, and a chunk of one equals the decode oracle."""
    rng = np.random.default_rng(16)
    b, hq, hkv, d, bs, n = 3, 4, 2, 8, 4, 16
    q_all, k, v = _rand_case(rng, 6, hq, hkv, d, n, oracle.BF16)
    k, v = k[:b], v[:b]
    ctx = np.array([16, 9, 5], dtype=np.int32)
    nq = [5, 1, 0]                                    # chunk lengths
    qs = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    q = q_all[:qs[-1]]
    kp, vp = contiguous_to_pool(k, bs), contiguous_to_pool(v, bs)
    tables = np.arange(b * n // bs, dtype=np.int32).reshape(b, n // bs)
    got = oracle.prefill_attention(q, kp, vp, tables, qs, ctx, 0.4, oracle.BF16, lib=lib)
    kd, vd, qd = bits_to_f64(k, oracle.BF16), bits_to_f64(v, oracle.BF16), bits_to_f64(q, oracle.BF16)
    grp = hq // hkv
    for s in range(b):
        for i in range(nq[s]):
            tok = qs[s] + i
            win = ctx[s] - nq[s] + i + 1
            for h in range(hq):
                p = scipy.special.softmax(0.4 * (kd[s, h // grp, :win] @ qd[tok, h]))
                assert np.max(np.abs(got[tok, h] - p @ vd[s, h // grp, :win])) < 1e-12
    # the one-token chunk of sequence 1 is a decode over its whole context
    dec = oracle.attention(q[qs[1]:qs[1] + 1], kp, vp, tables[1:2], ctx[1:2], 0.4, oracle.BF16, lib=lib)
    assert np.array_equal(dec[0], got[qs[1]])


def check_e4m3(lib):
    """E4M3 decode table and quantizer against torch.float8_e4m3fn; append
    scales and round trips; attention over E4M3 pools against scipy softmax
    on the dequantized values."""
    import torch

    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([lib.oracle_e4m3_value(int(c)) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and np.array_equal(got[~nan], ref[~nan])
    rng = np.random.default_rng(17)
    ys = np.concatenate([rng.uniform(-448, 448, 400), rng.standard_normal(400) * 3,
                         (ref[~nan][:120] + ref[~nan][1:121]) / 2]).astype(np.float32)   # incl. midpoints (ties)
    ys = ys[np.abs(ys) <= 448]
    want = torch.from_numpy(ys).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([lib.oracle_e4m3_quantize(float(y)) for y in ys], dtype=np.uint8)
    assert np.array_equal(mine, want)
    assert lib.oracle_e4m3_quantize(1000.0) == 0x7e and lib.oracle_e4m3_quantize(-449.0) == 0xfe
    # append: the largest element becomes +-448, every element within half a step
    nb, hkv, bs, d = 3, 2, 4, 16
    pool8 = np.zeros((nb, hkv, bs, d), np.uint8)
    scales = np.zeros((nb, hkv, bs), np.float32)
    x = rng.standard_normal((2, hkv, d)).astype(np.float32) * 3
    bits = f16_bits(x)
    oracle.append_e4m3(pool8, scales, bits, oracle.F16, np.array([5, 9]), lib=lib)
    xd = bits_to_f64(bits, oracle.F16)
    for t, slot in enumerate([5, 9]):
        blk, row = divmod(slot, bs)
        for h in range(hkv):
            sc = np.float32(np.abs(xd[t, h]).max()) / np.float32(448.0)
            assert scales[blk, h, row] == sc
            deq = np.array([lib.oracle_e4m3_value(int(c)) for c in pool8[blk, h, row]]) * float(sc)
            assert np.all(np.abs(deq - xd[t, h]) <= np.abs(xd[t, h]) / 16 + float(sc) * 2 ** -10)
            assert np.abs(deq).max() == 448.0 * float(sc)
    # attention over E4M3 pools == scipy softmax on the dequantized rows
    b, hq, n = 2, 4, 8
    tables = np.arange(b * n // bs, dtype=np.int32).reshape(b, n // bs)
    k8 = rng.integers(0, 0x7e, size=(b * n // bs, hkv, bs, d)).astype(np.uint8)
    v8 = rng.integers(0, 0x7e, size=(b * n // bs, hkv, bs, d)).astype(np.uint8) | 0x80 * (rng.random((b * n // bs, hkv, bs, d)) < 0.5).astype(np.uint8)
    ks = rng.uniform(0.001, 0.01, size=(b * n // bs, hkv, bs)).astype(np.float32)
    vs = rng.uniform(0.001, 0.01, size=(b * n // bs, hkv, bs)).astype(np.float32)
    q = bf16_bits(rng.standard_normal((b, hq, d)))
    ctx = np.array([8, 5], np.int32)
    out = oracle.attention_e4m3(q, oracle.BF16, k8, ks, v8, vs, tables, ctx, 0.3, lib=lib)
    val = np.vectorize(lambda c: lib.oracle_e4m3_value(int(c)))
    kd = val(k8) * ks[..., None]
    vd = val(v8) * vs[..., None]
    qd = bits_to_f64(q, oracle.BF16)
    for s_ in range(b):
        for h in range(hq):
            blocks = tables[s_]
            kk = np.concatenate([kd[bl, h // 2] for bl in blocks])[:ctx[s_]]
            vv = np.concatenate([vd[bl, h // 2] for bl in blocks])[:ctx[s_]]
            p = scipy.special.softmax(0.3 * (kk @ qd[s_, h]))
            assert np.max(np.abs(out[s_, h] - p @ vv)) < 1e-12


ALL_CHECKS = [check_decoders, check_sizing_golden, check_textbook, check_closed_forms, check_gqa_map,
              check_slot_bruteforce, check_slot_mask, check_append, check_permutation_and_sharing,
              check_poison_and_scaling, check_split_merge, check_copy_blocks, check_prefill,
              check_e4m3]
