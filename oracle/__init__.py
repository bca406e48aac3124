"""fp64 CPU oracle for paged-KV decode attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
path (``paged_kv_cache_437_b200``) never imports it, and this package never
imports the product: the two share no code.  The only thing both sides consume
is the seeded inputs from the ``workloads`` package, which holds none of the
method's arithmetic.

The arithmetic lives in ``pkv_oracle.c`` (plain C, fp64); each function there
cites the page and section it follows.  This module only compiles it with gcc
and marshals numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pkv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

F16, BF16 = 0, 1

_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle into a shared library (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", src, "-o", out, "-lm"]
        subprocess.run(cmd, check=True)
    return out


def _bind(lib):
    i64, i32, dbl, vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_double, ctypes.c_void_p
    lib.oracle_half_to_double.restype = dbl
    lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_double.restype = dbl
    lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_kv_bytes_per_layer.restype = i64
    lib.oracle_kv_bytes_per_layer.argtypes = [i64, i64, i64, i64]
    lib.oracle_slot_of.restype = i64
    lib.oracle_slot_of.argtypes = [vp, i64, i64]
    lib.oracle_append.restype = ctypes.c_int
    lib.oracle_append.argtypes = [vp, i64, i64, i64, i64, vp, vp, i64]
    lib.oracle_attention_range.restype = ctypes.c_int
    lib.oracle_attention_range.argtypes = [
        ctypes.c_int, vp, i64, vp, vp, i64, i64, i64, i64, vp, i64, dbl,
        i64, i64, i64, i64, vp, vp, vp]
    lib.oracle_paged_attention.restype = ctypes.c_int
    lib.oracle_paged_attention.argtypes = [
        ctypes.c_int, vp, i64, i64, vp, vp, i64, i64, i64, i64, vp, i64, vp, dbl,
        vp, i64, vp]
    lib.oracle_lse_merge.restype = ctypes.c_int
    lib.oracle_lse_merge.argtypes = [i64, vp, vp, vp, i64, vp]
    lib.oracle_prefill_attention.restype = ctypes.c_int
    lib.oracle_prefill_attention.argtypes = [ctypes.c_int, vp, i64, i64, i64, vp, vp, i64, i64, i64, i64, vp, i64,
                                             vp, vp, dbl, vp]
    lib.oracle_e4m3_value.restype = dbl
    lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_quantize.restype = ctypes.c_uint8
    lib.oracle_e4m3_quantize.argtypes = [ctypes.c_float]
    lib.oracle_e4m3_row_scale.restype = ctypes.c_float
    lib.oracle_e4m3_row_scale.argtypes = [vp, i64, ctypes.c_int]
    lib.oracle_append_e4m3.restype = ctypes.c_int
    lib.oracle_append_e4m3.argtypes = [vp, vp, i64, i64, i64, i64, vp, ctypes.c_int, vp, i64]
    lib.oracle_paged_attention_e4m3.restype = ctypes.c_int
    lib.oracle_paged_attention_e4m3.argtypes = [ctypes.c_int, vp, i64, i64, vp, vp, vp, vp, i64, i64, i64, i64, vp,
                                                i64, vp, dbl, vp]
    lib.oracle_copy_blocks.restype = ctypes.c_int
    lib.oracle_copy_blocks.argtypes = [vp, i64, i64, vp, i64]
    lib.oracle_mark_slots.restype = ctypes.c_int
    lib.oracle_mark_slots.argtypes = [vp, i64, i64, vp, i64, i64, vp]
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
    del i32
    return lib


def load(path: str | None = None):
    """Load (building if needed) the oracle library.  ``path`` loads another
    build of it, e.g. a deliberately mutated copy in a test."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        a = a.view(np.uint16)
    return a


def half_to_double(bits: int, lib=None) -> float:
    return (lib or load()).oracle_half_to_double(bits)


def bf16_to_double(bits: int, lib=None) -> float:
    return (lib or load()).oracle_bf16_to_double(bits)


def decode16(bits: np.ndarray, dtype: int, lib=None) -> np.ndarray:
    """Decode an array of 16-bit float bit patterns to fp64, element by element."""
    lib = lib or load()
    f = lib.oracle_half_to_double if dtype == F16 else lib.oracle_bf16_to_double
    flat = _u16(bits).reshape(-1)
    return np.array([f(int(x)) for x in flat], dtype=np.float64).reshape(np.shape(bits))


def kv_bytes_per_layer(seq_len: int, kv_heads: int, head_dim: int, dtype_bytes: int, lib=None) -> int:
    return int((lib or load()).oracle_kv_bytes_per_layer(seq_len, kv_heads, head_dim, dtype_bytes))


def slot_of(table_row: np.ndarray, pos: int, block_size: int, lib=None) -> int:
    row = np.ascontiguousarray(table_row, dtype=np.int32)
    return int((lib or load()).oracle_slot_of(_p(row), pos, block_size))


def slot_mapping(block_tables: np.ndarray, positions: np.ndarray, block_size: int, lib=None) -> np.ndarray:
    """Slot of position ``positions[s]`` for every sequence s (-1 where the position is < 0)."""
    lib = lib or load()
    out = np.empty(len(positions), dtype=np.int64)
    for s, p in enumerate(positions):
        out[s] = -1 if p < 0 else slot_of(block_tables[s], int(p), block_size, lib)
    return out


def append(cache: np.ndarray, new_kv: np.ndarray, slots: np.ndarray, lib=None) -> None:
    """In-place byte copy of ``new_kv[t]`` into ``cache`` at ``slots[t]`` (skip slot < 0).

    ``cache`` is [NB][Hkv][bs][D] of 16-bit values, ``new_kv`` [T][Hkv][D]."""
    lib = lib or load()
    assert cache.flags.c_contiguous
    nb, hkv, bs, d = cache.shape
    new = _u16(new_kv)
    sl = np.ascontiguousarray(slots, dtype=np.int64)
    rc = lib.oracle_append(_p(cache.view(np.uint16)), nb, hkv, bs, d, _p(new), _p(sl), len(sl))
    if rc != 0:
        raise ValueError("oracle_append: slot out of range")


def attention(q, k_cache, v_cache, block_tables, context_lens, scale, dtype,
              pairs=None, lib=None) -> np.ndarray:
    """Exact fp64 paged decode attention.

    Returns [B][Hq][D] fp64, or [len(pairs)][D] when ``pairs`` (an int array of
    (seq, head) rows) is given."""
    lib = lib or load()
    q16 = _u16(q)
    b, hq, d = q16.shape
    k16, v16 = _u16(k_cache), _u16(v_cache)
    nb, hkv, bs, d2 = k16.shape
    assert d2 == d and v16.shape == k16.shape
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    if pairs is None:
        out = np.zeros((b, hq, d), dtype=np.float64)
        pp, npairs = None, 0
    else:
        pr = np.ascontiguousarray(pairs, dtype=np.int64).reshape(-1, 2)
        out = np.zeros((len(pr), d), dtype=np.float64)
        pp, npairs = _p(pr), len(pr)
    rc = lib.oracle_paged_attention(dtype, _p(q16), b, hq, _p(k16), _p(v16), nb, bs, hkv, d,
                                    _p(bt), bt.shape[1], _p(cl), float(scale), pp, npairs, _p(out))
    if rc != 0:
        raise ValueError("oracle_paged_attention: invalid arguments or table entry out of range")
    return out


def attention_range(q, k_cache, v_cache, block_tables, scale, dtype, seq, head, p_begin, p_end, lib=None):
    """Unnormalised (m, l, o) of one (seq, head) over positions [p_begin, p_end)."""
    lib = lib or load()
    q16 = _u16(q)
    b, hq, d = q16.shape
    k16, v16 = _u16(k_cache), _u16(v_cache)
    nb, hkv, bs, _ = k16.shape
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    m = np.zeros(1)
    l = np.zeros(1)
    o = np.zeros(d)
    rc = lib.oracle_attention_range(dtype, _p(q16), hq, _p(k16), _p(v16), nb, bs, hkv, d,
                                    _p(bt), bt.shape[1], float(scale), seq, head, p_begin, p_end,
                                    _p(m), _p(l), _p(o))
    if rc != 0:
        raise ValueError("oracle_attention_range: invalid arguments")
    return float(m[0]), float(l[0]), o


def lse_merge(m, l, o, lib=None) -> np.ndarray:
    lib = lib or load()
    m = np.ascontiguousarray(m, dtype=np.float64)
    l = np.ascontiguousarray(l, dtype=np.float64)
    o = np.ascontiguousarray(o, dtype=np.float64)
    n, d = o.shape
    out = np.zeros(d)
    lib.oracle_lse_merge(n, _p(m), _p(l), _p(o), d, _p(out))
    return out


def slot_mask(block_tables, lens, block_size: int, num_blocks: int, lib=None) -> np.ndarray:
    """bool [num_blocks * block_size]: True where a slot holds a position < lens[s] of some sequence."""
    lib = lib or load()
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    ln = np.ascontiguousarray(lens, dtype=np.int32)
    mask = np.zeros(num_blocks * block_size, dtype=np.uint8)
    rc = lib.oracle_mark_slots(_p(bt), bt.shape[0], bt.shape[1], _p(ln), block_size, num_blocks, _p(mask))
    if rc != 0:
        raise ValueError("oracle_mark_slots: table entry out of range")
    return mask.astype(bool)


def prefill_attention(q, k_cache, v_cache, block_tables, query_start, context_lens, scale, dtype,
                      lib=None) -> np.ndarray:
    """Causal chunked-prefill attention, fp64 [T][Hq][D] (see the C source)."""
    lib = lib or load()
    q16 = _u16(q)
    t, hq, d = q16.shape
    k16, v16 = _u16(k_cache), _u16(v_cache)
    nb, hkv, bs, _ = k16.shape
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    qs = np.ascontiguousarray(query_start, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    out = np.zeros((t, hq, d), dtype=np.float64)
    rc = lib.oracle_prefill_attention(dtype, _p(q16), t, len(cl), hq, _p(k16), _p(v16), nb, bs, hkv, d, _p(bt),
                                      bt.shape[1], _p(qs), _p(cl), float(scale), _p(out))
    if rc != 0:
        raise ValueError("oracle_prefill_attention: inconsistent lengths or table entry out of range")
    return out


def e4m3_value(code: int, lib=None) -> float:
    return float((lib or load()).oracle_e4m3_value(code))


def e4m3_quantize(y: float, lib=None) -> int:
    return int((lib or load()).oracle_e4m3_quantize(float(y)))


def append_e4m3(cache8: np.ndarray, scales: np.ndarray, new_kv, new_dtype: int, slots, lib=None) -> None:
    """Quantize rows of new_kv [T][Hkv][D] (16-bit bits) into an E4M3 pool
    [NB][Hkv][bs][D] (uint8) and its scales [NB][Hkv][bs] (float32), in place."""
    lib = lib or load()
    assert cache8.dtype == np.uint8 and scales.dtype == np.float32
    nb, hkv, bs, d = cache8.shape
    new = _u16(new_kv)
    sl = np.ascontiguousarray(slots, dtype=np.int64)
    rc = lib.oracle_append_e4m3(_p(cache8), _p(scales), nb, hkv, bs, d, _p(new), new_dtype, _p(sl), len(sl))
    if rc != 0:
        raise ValueError("oracle_append_e4m3: slot out of range")


def attention_e4m3(q, q_dtype, k8, k_scales, v8, v_scales, block_tables, context_lens, scale, lib=None):
    lib = lib or load()
    q16 = _u16(q)
    b, hq, d = q16.shape
    nb, hkv, bs, _ = k8.shape
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    out = np.zeros((b, hq, d), dtype=np.float64)
    args = [np.ascontiguousarray(x) for x in (k8, k_scales, v8, v_scales)]
    rc = lib.oracle_paged_attention_e4m3(q_dtype, _p(q16), b, hq, *(_p(x) for x in args), nb, bs, hkv, d, _p(bt),
                                         bt.shape[1], _p(cl), float(scale), _p(out))
    if rc != 0:
        raise ValueError("oracle_paged_attention_e4m3: invalid arguments")
    return out


def copy_blocks(cache: np.ndarray, pairs, lib=None) -> None:
    """In-place whole-block copies src -> dst of a [NB][Hkv][bs][D] pool, in order."""
    lib = lib or load()
    assert cache.flags.c_contiguous
    nb = cache.shape[0]
    pr = np.ascontiguousarray(pairs, dtype=np.int32).reshape(-1, 2)
    rc = lib.oracle_copy_blocks(_p(cache.view(np.uint16)), nb, int(np.prod(cache.shape[1:])), _p(pr), len(pr))
    if rc != 0:
        raise ValueError("oracle_copy_blocks: block id out of range")


def num_threads(lib=None) -> int:
    return int((lib or load()).oracle_num_threads())


def set_num_threads(n: int, lib=None) -> None:
    (lib or load()).oracle_set_num_threads(int(n))
