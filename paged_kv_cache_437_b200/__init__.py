"""Python binding of ``libpkv.so`` -- paged KV-cache decode attention on B200.

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels (sm_100a) or its C++ host allocator.  There is no fallback: if the
shared library is missing, importing this package raises ``ImportError``.
Build it with ``python paged_kv_cache_437_b200/build.py``.

Names follow the C ABI in ``include/pkv.h``.  Device buffers are passed as
torch CUDA tensors (torch is used for device memory and streams only).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpkv.so")

PKV_OK = 0
PKV_ERR_INVALID = -1
PKV_ERR_OOM = -2
PKV_ERR_CUDA = -3
PKV_ERR_SHARED_WRITE = -4
PKV_ERR_DEVICE_CHECK = -5
PKV_ERR_TIMEOUT = -6
PKV_ERR_SCRATCH_TOO_SMALL = -7
PKV_STATIC_SCRATCH_BYTES = 32 << 20

PKV_F16 = 0
PKV_BF16 = 1
PKV_E4M3 = 2

PKV_PARTITION_NONE = -1
PKV_PARTITION_AUTO = 0

_c_i32, _c_i64, _c_vp, _c_sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t


class pkv_cache(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int), ("num_blocks", ctypes.c_int64),
                ("block_size", ctypes.c_int64), ("num_kv_heads", ctypes.c_int64),
                ("head_dim", ctypes.c_int64), ("scales", ctypes.c_void_p)]


class pkv_sched_config(ctypes.Structure):
    _fields_ = [("max_batch_tokens", ctypes.c_int32), ("max_seqs", ctypes.c_int32),
                ("chunk_tokens", ctypes.c_int32), ("block_size", ctypes.c_int32)]


class pkv_sched_batch(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("num_tokens", ctypes.c_int32), ("num_preempted", ctypes.c_int32),
                ("num_finished", ctypes.c_int32), ("request_ids", ctypes.c_void_p), ("seq_ids", ctypes.c_void_p),
                ("query_lens", ctypes.c_void_p), ("context_lens", ctypes.c_void_p), ("slots", ctypes.c_void_p),
                ("finished_ids", ctypes.c_void_p), ("preempted_ids", ctypes.c_void_p)]


class PkvError(RuntimeError):
    def __init__(self, status: int, what: str):
        detail = f" [{lib.pkv_last_cuda_error().decode()}]" if status == PKV_ERR_CUDA else ""
        super().__init__(f"{what}: {pkv_status_string(status)} ({status}){detail}")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python paged_kv_cache_437_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    sig = {
        "pkv_append": (ctypes.c_int, [_c_vp, _c_vp, _c_vp, _c_i64, pkv_cache, pkv_cache, _c_vp]),
        "pkv_decode_attention": (ctypes.c_int, [_c_vp, _c_i64, _c_i64, pkv_cache, pkv_cache, _c_vp, _c_i64,
                                                _c_vp, ctypes.c_float, _c_vp, _c_vp, _c_sz, _c_i32, _c_vp]),
        "pkv_decode_workspace_bytes": (_c_sz, [_c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_i32]),
        "pkv_append_decode_attention": (ctypes.c_int, [_c_vp, _c_vp, _c_vp, _c_vp, _c_i64, _c_i64, pkv_cache,
                                                       pkv_cache, _c_vp, _c_i64, _c_vp, ctypes.c_float, _c_vp,
                                                       _c_vp, _c_sz, _c_i32, _c_vp]),
        "pkv_alloc_create": (ctypes.c_int, [_c_i32, _c_i32, ctypes.POINTER(_c_vp)]),
        "pkv_alloc_destroy": (None, [_c_vp]),
        "pkv_block_alloc": (ctypes.c_int, [_c_vp, ctypes.POINTER(_c_i32)]),
        "pkv_block_incref": (ctypes.c_int, [_c_vp, _c_i32]),
        "pkv_block_decref": (ctypes.c_int, [_c_vp, _c_i32]),
        "pkv_num_free": (_c_i32, [_c_vp]),
        "pkv_refcount": (_c_i32, [_c_vp, _c_i32]),
        "pkv_seq_create": (ctypes.c_int, [_c_vp, ctypes.POINTER(_c_i32)]),
        "pkv_seq_fork": (ctypes.c_int, [_c_vp, _c_i32, _c_i32, ctypes.POINTER(_c_i32)]),
        "pkv_seq_append_slot": (ctypes.c_int, [_c_vp, _c_i32, ctypes.POINTER(_c_i64)]),
        "pkv_seq_append_slots": (ctypes.c_int, [_c_vp, _c_vp, _c_i32, _c_vp]),
        "pkv_seq_free": (ctypes.c_int, [_c_vp, _c_i32]),
        "pkv_seq_fork_tokens": (ctypes.c_int, [_c_vp, _c_i32, _c_i64, ctypes.POINTER(_c_i32)]),
        "pkv_seq_append_slot_cow": (ctypes.c_int, [_c_vp, _c_i32, ctypes.POINTER(_c_i64), ctypes.POINTER(_c_i32),
                                                   ctypes.POINTER(_c_i32)]),
        "pkv_seq_append_slots_cow": (ctypes.c_int, [_c_vp, _c_vp, _c_i32, _c_vp, _c_vp, ctypes.POINTER(_c_i32)]),
        "pkv_copy_blocks": (ctypes.c_int, [pkv_cache, pkv_cache, _c_vp, _c_i64, _c_vp]),
        "pkv_append_e4m3": (ctypes.c_int, [_c_vp, _c_vp, ctypes.c_int, _c_vp, _c_i64, pkv_cache, pkv_cache, _c_vp]),
        "pkv_decode_attention_e4m3": (ctypes.c_int, [_c_vp, ctypes.c_int, _c_i64, _c_i64, pkv_cache, pkv_cache,
                                                     _c_vp, _c_i64, _c_vp, ctypes.c_float, _c_vp, _c_vp, _c_sz,
                                                     _c_i32, _c_vp]),
        "pkv_sched_create": (ctypes.c_int, [_c_vp, ctypes.POINTER(pkv_sched_config), ctypes.POINTER(_c_vp)]),
        "pkv_sched_destroy": (None, [_c_vp]),
        "pkv_sched_add": (ctypes.c_int, [_c_vp, _c_i64, _c_i32, _c_i32]),
        "pkv_sched_step": (ctypes.c_int, [_c_vp, ctypes.POINTER(pkv_sched_batch)]),
        "pkv_sched_num_waiting": (_c_i32, [_c_vp]),
        "pkv_sched_num_running": (_c_i32, [_c_vp]),
        "pkv_prefill_attention": (ctypes.c_int, [_c_vp, _c_i64, _c_i64, _c_i64, pkv_cache, pkv_cache, _c_vp,
                                                 _c_i64, _c_vp, _c_vp, ctypes.c_float, _c_vp, _c_vp, _c_sz,
                                                 _c_vp]),
        "pkv_prefill_workspace_bytes": (_c_sz, [_c_i64, _c_i64, _c_i64, _c_i64, _c_i64]),
        "pkv_seq_block_table": (ctypes.c_int, [_c_vp, _c_i32, _c_vp, _c_i32, ctypes.POINTER(_c_i32)]),
        "pkv_seq_context_len": (_c_i64, [_c_vp, _c_i32]),
        "pkv_batch_tables": (ctypes.c_int, [_c_vp, _c_vp, _c_i32, _c_vp, _c_i32, _c_vp]),
        "pkv_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "pkv_last_cuda_error": (ctypes.c_char_p, []),
        "pkv_get_last_error": (ctypes.c_int, []),
        "pkv_test_inject_wait_timeout": (ctypes.c_int, [_c_i32, _c_i64]),
        "pkv_decode_attention_static_scratch": (ctypes.c_int, [_c_vp, _c_i64, _c_i64, pkv_cache, pkv_cache,
                                                               _c_vp, _c_i64, _c_vp, ctypes.c_float, _c_vp,
                                                               _c_i32, _c_vp]),
        "pkv_append_decode_attention_shared_prefix": (ctypes.c_int, [_c_vp, _c_vp, _c_vp, _c_vp, _c_i64, _c_i64,
                                                                     pkv_cache, pkv_cache, _c_vp, _c_i64, _c_vp,
                                                                     _c_vp, _c_i64, _c_vp, ctypes.c_float, _c_vp,
                                                                     _c_vp, _c_sz, _c_vp]),
        "pkv_shared_prefix_workspace_bytes": (_c_sz, [_c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _c_i64]),
        "pkv_batch_prefix_groups": (ctypes.c_int, [_c_vp, _c_vp, _c_i32, _c_vp, ctypes.POINTER(_c_i32), _c_vp]),
        "pkv_test_exp2_poly": (ctypes.c_int, [_c_vp, _c_vp, _c_i64, _c_vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def pkv_status_string(status: int) -> str:
    return lib.pkv_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != PKV_OK:
        raise PkvError(status, what)


# ------------------------------------------------------------------ device calls

def _dtype_code(t) -> int:
    import torch

    if t.dtype == torch.float16:
        return PKV_F16
    if t.dtype == torch.bfloat16:
        return PKV_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; use float16 or bfloat16")


def _stream_ptr(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _require(t, name, ndim=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")


def cache_desc(cache) -> pkv_cache:
    """Describe a [NB][Hkv][bs][D] fp16/bf16 CUDA tensor as a ``pkv_cache``."""
    _require(cache, "cache", 4)
    nb, hkv, bs, d = cache.shape
    return pkv_cache(cache.data_ptr(), _dtype_code(cache), nb, bs, hkv, d, None)


def cache_desc_e4m3(codes, scales) -> pkv_cache:
    """Describe an E4M3 pool: codes uint8 [NB][Hkv][bs][D], scales float32 [NB][Hkv][bs]."""
    import torch

    _require(codes, "codes", 4)
    _require(scales, "scales", 3)
    if codes.dtype != torch.uint8 or scales.dtype != torch.float32 or tuple(scales.shape) != tuple(codes.shape[:3]):
        raise TypeError("E4M3 pool: uint8 codes [NB][Hkv][bs][D] and float32 scales [NB][Hkv][bs]")
    nb, hkv, bs, d = codes.shape
    return pkv_cache(codes.data_ptr(), PKV_E4M3, nb, bs, hkv, d, scales.data_ptr())


def pkv_append(k_new, v_new, slot_mapping, k_cache, v_cache, stream=None) -> None:
    """Write k_new/v_new [T][Hkv][D] into the caches at slot_mapping[T] (int64, <0 = skip)."""
    import torch

    for t, n in ((k_new, "k_new"), (v_new, "v_new"), (slot_mapping, "slot_mapping")):
        _require(t, n)
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    if k_new.dtype != k_cache.dtype or v_new.dtype != v_cache.dtype:
        raise TypeError("new K/V must have the caches' dtype")
    if k_new.shape != v_new.shape or k_new.dim() != 3 or k_new.shape[0] != slot_mapping.numel() or \
            k_new.shape[1] != k_cache.shape[1] or k_new.shape[2] != k_cache.shape[3]:
        raise ValueError("k_new / v_new must be [T][Hkv][D] with T = len(slot_mapping)")
    st = lib.pkv_append(k_new.data_ptr(), v_new.data_ptr(), slot_mapping.data_ptr(), slot_mapping.numel(),
                        cache_desc(k_cache), cache_desc(v_cache), _stream_ptr(stream))
    _check(st, "pkv_append")


def pkv_decode_workspace_bytes(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                               max_context_len: int, partition_tokens: int = PKV_PARTITION_AUTO) -> int:
    return int(lib.pkv_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                              max_context_len, partition_tokens))


def _check_decode_args(q, k_cache, block_tables, context_lens, out) -> None:
    """Dtype and shape checks shared by the decode wrappers."""
    import torch

    for t, n in ((q, "q"), (out, "out"), (block_tables, "block_tables"), (context_lens, "context_lens")):
        _require(t, n)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    if q.dtype != k_cache.dtype or out.dtype != q.dtype:
        raise TypeError("q, out and the caches must share one dtype")
    if q.dim() != 3 or out.shape != q.shape or block_tables.dim() != 2 or \
            block_tables.shape[0] != q.shape[0] or context_lens.numel() != q.shape[0]:
        raise ValueError("shapes: q/out [B][Hq][D], block_tables [B][MB], context_lens [B]")


def pkv_decode_attention(q, k_cache, v_cache, block_tables, context_lens, scale: float, out,
                         workspace=None, partition_tokens: int = PKV_PARTITION_AUTO, stream=None) -> None:
    """out[B][Hq][D] = paged decode attention of q[B][Hq][D] over the caches."""
    _check_decode_args(q, k_cache, block_tables, context_lens, out)
    ws_ptr, ws_bytes = 0, 0
    if workspace is not None:
        _require(workspace, "workspace")
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    st = lib.pkv_decode_attention(q.data_ptr(), q.shape[0], q.shape[1], cache_desc(k_cache),
                                  cache_desc(v_cache), block_tables.data_ptr(), block_tables.shape[1],
                                  context_lens.data_ptr(), float(scale), out.data_ptr(), ws_ptr or None,
                                  ws_bytes, int(partition_tokens), _stream_ptr(stream))
    _check(st, "pkv_decode_attention")


def pkv_test_inject_wait_timeout(enable: bool, wait_limit_ns: int = 50_000_000) -> None:
    _check(lib.pkv_test_inject_wait_timeout(1 if enable else 0, int(wait_limit_ns)),
           "pkv_test_inject_wait_timeout")


def pkv_decode_attention_static_scratch(q, k_cache, v_cache, block_tables, context_lens, scale: float, out,
                                        partition_tokens: int = PKV_PARTITION_AUTO, stream=None) -> None:
    """pkv_decode_attention for callers that cannot allocate device memory:
    the split scratch is the library's fixed device array (see include/pkv.h).
    Calls that overlap on the GPU share that array and must be serialised."""
    _check_decode_args(q, k_cache, block_tables, context_lens, out)
    st = lib.pkv_decode_attention_static_scratch(q.data_ptr(), q.shape[0], q.shape[1], cache_desc(k_cache),
                                                 cache_desc(v_cache), block_tables.data_ptr(),
                                                 block_tables.shape[1], context_lens.data_ptr(), float(scale),
                                                 out.data_ptr(), int(partition_tokens), _stream_ptr(stream))
    _check(st, "pkv_decode_attention_static_scratch")


def pkv_append_decode_attention(k_new, v_new, slot_mapping, q, k_cache, v_cache, block_tables, context_lens,
                                scale: float, out, workspace=None, partition_tokens: int = PKV_PARTITION_AUTO,
                                stream=None) -> None:
    """Append (one new token per sequence, at position ctx-1) and decode in one launch."""
    import torch

    for t, n in ((k_new, "k_new"), (v_new, "v_new"), (slot_mapping, "slot_mapping"), (q, "q"), (out, "out"),
                 (block_tables, "block_tables"), (context_lens, "context_lens")):
        _require(t, n)
    if slot_mapping.dtype != torch.int64 or block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("slot_mapping int64, block_tables / context_lens int32")
    if q.dtype != k_cache.dtype or out.dtype != q.dtype or k_new.dtype != q.dtype or v_new.dtype != q.dtype:
        raise TypeError("q, out, k_new, v_new and the caches must share one dtype")
    b = q.shape[0]
    if k_new.shape != (b, k_cache.shape[1], k_cache.shape[3]) or v_new.shape != k_new.shape or \
            slot_mapping.numel() != b or out.shape != q.shape or block_tables.shape[0] != b or \
            context_lens.numel() != b:
        raise ValueError("shapes: k_new/v_new [B][Hkv][D], slot_mapping [B], q/out [B][Hq][D]")
    ws_ptr, ws_bytes = 0, 0
    if workspace is not None:
        _require(workspace, "workspace")
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    st = lib.pkv_append_decode_attention(k_new.data_ptr(), v_new.data_ptr(), slot_mapping.data_ptr(), q.data_ptr(),
                                         b, q.shape[1], cache_desc(k_cache), cache_desc(v_cache),
                                         block_tables.data_ptr(), block_tables.shape[1], context_lens.data_ptr(),
                                         float(scale), out.data_ptr(), ws_ptr or None, ws_bytes,
                                         int(partition_tokens), _stream_ptr(stream))
    _check(st, "pkv_append_decode_attention")


def pkv_prefill_workspace_bytes(num_tokens: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                                max_context_len: int) -> int:
    return int(lib.pkv_prefill_workspace_bytes(num_tokens, num_q_heads, num_kv_heads, head_dim, max_context_len))


def pkv_prefill_attention(q, k_cache, v_cache, block_tables, query_start, context_lens, scale: float, out,
                          workspace, stream=None) -> None:
    """Causal chunked-prefill attention: q/out [T][Hq][D], query_start [B+1], context_lens [B]."""
    import torch

    for t, n in ((q, "q"), (out, "out"), (block_tables, "block_tables"), (query_start, "query_start"),
                 (context_lens, "context_lens"), (workspace, "workspace")):
        _require(t, n)
    if query_start.dtype != torch.int32 or context_lens.dtype != torch.int32 or block_tables.dtype != torch.int32:
        raise TypeError("query_start, context_lens and block_tables must be int32")
    b = context_lens.numel()
    if query_start.numel() != b + 1 or block_tables.shape[0] != b or out.shape != q.shape or q.dim() != 3:
        raise ValueError("shapes: q/out [T][Hq][D], query_start [B+1], context_lens [B], block_tables [B][MB]")
    st = lib.pkv_prefill_attention(q.data_ptr(), q.shape[0], b, q.shape[1], cache_desc(k_cache), cache_desc(v_cache),
                                   block_tables.data_ptr(), block_tables.shape[1], query_start.data_ptr(),
                                   context_lens.data_ptr(), float(scale), out.data_ptr(), workspace.data_ptr(),
                                   workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    _check(st, "pkv_prefill_attention")


def pkv_append_e4m3(k_new, v_new, slot_mapping, k_codes, k_scales, v_codes, v_scales, stream=None) -> None:
    """Quantize k_new / v_new [T][Hkv][D] (f16 / bf16) into E4M3 pools at the slots."""
    for t, n in ((k_new, "k_new"), (v_new, "v_new"), (slot_mapping, "slot_mapping")):
        _require(t, n)
    st = lib.pkv_append_e4m3(k_new.data_ptr(), v_new.data_ptr(), _dtype_code(k_new), slot_mapping.data_ptr(),
                             slot_mapping.numel(), cache_desc_e4m3(k_codes, k_scales),
                             cache_desc_e4m3(v_codes, v_scales), _stream_ptr(stream))
    _check(st, "pkv_append_e4m3")


def pkv_decode_attention_e4m3(q, k_codes, k_scales, v_codes, v_scales, block_tables, context_lens, scale: float,
                              out, workspace=None, partition_tokens: int = PKV_PARTITION_AUTO, stream=None) -> None:
    """pkv_decode_attention over E4M3 pools; q / out f16 or bf16."""
    for t, n in ((q, "q"), (out, "out"), (block_tables, "block_tables"), (context_lens, "context_lens")):
        _require(t, n)
    ws_ptr, ws_bytes = 0, 0
    if workspace is not None:
        _require(workspace, "workspace")
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    st = lib.pkv_decode_attention_e4m3(q.data_ptr(), _dtype_code(q), q.shape[0], q.shape[1],
                                       cache_desc_e4m3(k_codes, k_scales), cache_desc_e4m3(v_codes, v_scales),
                                       block_tables.data_ptr(), block_tables.shape[1], context_lens.data_ptr(),
                                       float(scale), out.data_ptr(), ws_ptr or None, ws_bytes,
                                       int(partition_tokens), _stream_ptr(stream))
    _check(st, "pkv_decode_attention_e4m3")


def pkv_get_last_error() -> int:
    """Read-and-clear the device check word (synchronises the device)."""
    return int(lib.pkv_get_last_error())


# ------------------------------------------------------------------ host allocator

def pkv_alloc_create(num_blocks: int, block_size: int):
    h = ctypes.c_void_p()
    _check(lib.pkv_alloc_create(num_blocks, block_size, ctypes.byref(h)), "pkv_alloc_create")
    return h


def pkv_alloc_destroy(h) -> None:
    lib.pkv_alloc_destroy(h)


def pkv_block_alloc(h) -> int:
    b = ctypes.c_int32()
    _check(lib.pkv_block_alloc(h, ctypes.byref(b)), "pkv_block_alloc")
    return b.value


def pkv_block_incref(h, block: int) -> None:
    _check(lib.pkv_block_incref(h, block), "pkv_block_incref")


def pkv_block_decref(h, block: int) -> None:
    _check(lib.pkv_block_decref(h, block), "pkv_block_decref")


def pkv_num_free(h) -> int:
    return int(lib.pkv_num_free(h))


def pkv_refcount(h, block: int) -> int:
    return int(lib.pkv_refcount(h, block))


def pkv_seq_create(h) -> int:
    s = ctypes.c_int32()
    _check(lib.pkv_seq_create(h, ctypes.byref(s)), "pkv_seq_create")
    return s.value


def pkv_seq_fork(h, parent: int, num_full_blocks: int) -> int:
    s = ctypes.c_int32()
    _check(lib.pkv_seq_fork(h, parent, num_full_blocks, ctypes.byref(s)), "pkv_seq_fork")
    return s.value


def pkv_seq_append_slot(h, seq: int) -> int:
    slot = ctypes.c_int64()
    _check(lib.pkv_seq_append_slot(h, seq, ctypes.byref(slot)), "pkv_seq_append_slot")
    return slot.value


def pkv_seq_append_slots(h, seqs):
    """Slots (numpy int64) for one new token of each sequence; all or nothing."""
    import numpy as np

    s = np.ascontiguousarray(seqs, dtype=np.int32)
    out = np.empty(len(s), dtype=np.int64)
    _check(lib.pkv_seq_append_slots(h, s.ctypes.data, len(s), out.ctypes.data), "pkv_seq_append_slots")
    return out


def pkv_seq_fork_tokens(h, parent: int, num_tokens: int) -> int:
    s = ctypes.c_int32()
    _check(lib.pkv_seq_fork_tokens(h, parent, num_tokens, ctypes.byref(s)), "pkv_seq_fork_tokens")
    return s.value


def pkv_seq_append_slot_cow(h, seq: int):
    """(slot, copy_src, copy_dst); copy_src == -1 when no copy is needed."""
    slot, src, dst = ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
    _check(lib.pkv_seq_append_slot_cow(h, seq, ctypes.byref(slot), ctypes.byref(src), ctypes.byref(dst)),
           "pkv_seq_append_slot_cow")
    return slot.value, src.value, dst.value


def pkv_seq_append_slots_cow(h, seqs):
    """(slots int64 [n], copies int32 [k][2]) for one new token of each sequence; all or nothing."""
    import numpy as np

    s = np.ascontiguousarray(seqs, dtype=np.int32)
    slots = np.empty(len(s), dtype=np.int64)
    copies = np.empty((max(1, len(s)), 2), dtype=np.int32)
    nc = ctypes.c_int32()
    _check(lib.pkv_seq_append_slots_cow(h, s.ctypes.data, len(s), slots.ctypes.data, copies.ctypes.data,
                                        ctypes.byref(nc)), "pkv_seq_append_slots_cow")
    return slots, copies[:nc.value].copy()


def pkv_copy_blocks(k_cache, v_cache, pairs, stream=None) -> None:
    """Copy whole blocks src -> dst (pairs: CUDA int32 [n][2]) in both pools."""
    import torch

    _require(pairs, "pairs")
    if pairs.dtype != torch.int32:
        raise TypeError("pairs must be int32")
    n = pairs.numel() // 2
    _check(lib.pkv_copy_blocks(cache_desc(k_cache), cache_desc(v_cache), pairs.data_ptr() if n else None, n,
                               _stream_ptr(stream)), "pkv_copy_blocks")


def pkv_seq_free(h, seq: int) -> None:
    _check(lib.pkv_seq_free(h, seq), "pkv_seq_free")


def pkv_seq_block_table(h, seq: int):
    import numpy as np

    n = ctypes.c_int32()
    _check(lib.pkv_seq_block_table(h, seq, None, 0, ctypes.byref(n)), "pkv_seq_block_table")
    out = np.empty(n.value, dtype=np.int32)
    _check(lib.pkv_seq_block_table(h, seq, out.ctypes.data, n.value, ctypes.byref(n)), "pkv_seq_block_table")
    return out


def pkv_seq_context_len(h, seq: int) -> int:
    return int(lib.pkv_seq_context_len(h, seq))


def pkv_batch_tables(h, seqs, cap: int):
    """(block_tables [n][cap] int32 padded with -1, context_lens [n] int32) for a batch."""
    import numpy as np

    s = np.ascontiguousarray(seqs, dtype=np.int32)
    tables = np.empty((len(s), cap), dtype=np.int32)
    lens = np.empty(len(s), dtype=np.int32)
    _check(lib.pkv_batch_tables(h, s.ctypes.data, len(s), tables.ctypes.data, cap, lens.ctypes.data),
           "pkv_batch_tables")
    return tables, lens


def pkv_batch_prefix_groups(h, seqs):
    """(group_start [G+1] int32, shared_lens [n] int32) of a batch: runs of
    consecutive sequences that start with the same shared block."""
    import numpy as np

    s = np.ascontiguousarray(seqs, dtype=np.int32)
    starts = np.empty(len(s) + 1, dtype=np.int32)
    shared = np.empty(len(s), dtype=np.int32)
    ng = _c_i32(0)
    _check(lib.pkv_batch_prefix_groups(h, s.ctypes.data, len(s), starts.ctypes.data, ctypes.byref(ng),
                                       shared.ctypes.data), "pkv_batch_prefix_groups")
    return starts[:ng.value + 1].copy(), shared


def pkv_shared_prefix_workspace_bytes(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                                      max_context_len: int, num_groups: int) -> int:
    return int(lib.pkv_shared_prefix_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                     max_context_len, num_groups))


def pkv_append_decode_attention_shared_prefix(k_new, v_new, slot_mapping, q, k_cache, v_cache, block_tables,
                                              context_lens, group_start, shared_lens, scale: float, out,
                                              workspace, stream=None) -> None:
    """A decode step (append optional: k_new = v_new = slot_mapping = None)
    whose sharing groups' common prefixes are read once per group."""
    import torch

    _check_decode_args(q, k_cache, block_tables, context_lens, out)
    for t, n in ((group_start, "group_start"), (shared_lens, "shared_lens"), (workspace, "workspace")):
        _require(t, n)
    if group_start.dtype != torch.int32 or shared_lens.dtype != torch.int32:
        raise TypeError("group_start and shared_lens must be int32")
    b = q.shape[0]
    if shared_lens.numel() != b or group_start.numel() < 1:
        raise ValueError("shapes: group_start [G+1], shared_lens [B]")
    ptrs = (None, None, None)
    if k_new is not None or v_new is not None or slot_mapping is not None:
        for t, n in ((k_new, "k_new"), (v_new, "v_new"), (slot_mapping, "slot_mapping")):
            _require(t, n)
        if slot_mapping.dtype != torch.int64 or k_new.dtype != q.dtype or v_new.dtype != q.dtype:
            raise TypeError("slot_mapping int64; k_new / v_new in q's dtype")
        if k_new.shape != (b, k_cache.shape[1], k_cache.shape[3]) or v_new.shape != k_new.shape or \
                slot_mapping.numel() != b:
            raise ValueError("shapes: k_new/v_new [B][Hkv][D], slot_mapping [B]")
        ptrs = (k_new.data_ptr(), v_new.data_ptr(), slot_mapping.data_ptr())
    st = lib.pkv_append_decode_attention_shared_prefix(
        *ptrs, q.data_ptr(), b, q.shape[1], cache_desc(k_cache), cache_desc(v_cache), block_tables.data_ptr(),
        block_tables.shape[1], context_lens.data_ptr(), group_start.data_ptr(), group_start.numel() - 1,
        shared_lens.data_ptr(), float(scale), out.data_ptr(), workspace.data_ptr(),
        workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    _check(st, "pkv_append_decode_attention_shared_prefix")


class BlockAllocator:
    """Owning wrapper of one allocator handle."""

    def __init__(self, num_blocks: int, block_size: int):
        self.handle = pkv_alloc_create(num_blocks, block_size)
        self.num_blocks, self.block_size = num_blocks, block_size

    def close(self):
        if self.handle:
            pkv_alloc_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    alloc = lambda self: pkv_block_alloc(self.handle)
    incref = lambda self, b: pkv_block_incref(self.handle, b)
    decref = lambda self, b: pkv_block_decref(self.handle, b)
    num_free = lambda self: pkv_num_free(self.handle)
    refcount = lambda self, b: pkv_refcount(self.handle, b)
    seq_create = lambda self: pkv_seq_create(self.handle)
    seq_fork = lambda self, p, n: pkv_seq_fork(self.handle, p, n)
    append_slot = lambda self, s: pkv_seq_append_slot(self.handle, s)
    append_slots = lambda self, seqs: pkv_seq_append_slots(self.handle, seqs)
    seq_free = lambda self, s: pkv_seq_free(self.handle, s)
    seq_fork_tokens = lambda self, p, n: pkv_seq_fork_tokens(self.handle, p, n)
    append_slot_cow = lambda self, s: pkv_seq_append_slot_cow(self.handle, s)
    append_slots_cow = lambda self, seqs: pkv_seq_append_slots_cow(self.handle, seqs)
    block_table = lambda self, s: pkv_seq_block_table(self.handle, s)
    context_len = lambda self, s: pkv_seq_context_len(self.handle, s)
    batch_tables = lambda self, seqs, cap: pkv_batch_tables(self.handle, seqs, cap)
    prefix_groups = lambda self, seqs: pkv_batch_prefix_groups(self.handle, seqs)


class Scheduler:
    """Iteration-level scheduler over a BlockAllocator (host only)."""

    def __init__(self, alloc: "BlockAllocator", max_batch_tokens: int, max_seqs: int, chunk_tokens: int = 512):
        import numpy as np

        self.alloc = alloc
        self.cfg = pkv_sched_config(max_batch_tokens, max_seqs, chunk_tokens, alloc.block_size)
        h = ctypes.c_void_p()
        _check(lib.pkv_sched_create(alloc.handle, ctypes.byref(self.cfg), ctypes.byref(h)), "pkv_sched_create")
        self.handle = h
        self._arr = dict(request_ids=np.zeros(max_seqs, np.int64), seq_ids=np.zeros(max_seqs, np.int32),
                         query_lens=np.zeros(max_seqs, np.int32), context_lens=np.zeros(max_seqs, np.int32),
                         slots=np.zeros(max_batch_tokens, np.int64), finished_ids=np.zeros(max_seqs, np.int64),
                         preempted_ids=np.zeros(max_seqs, np.int64))
        self._batch = pkv_sched_batch(0, 0, 0, 0, *(self._arr[k].ctypes.data for k in (
            "request_ids", "seq_ids", "query_lens", "context_lens", "slots", "finished_ids", "preempted_ids")))

    def add(self, request_id: int, prompt_len: int, max_new_tokens: int) -> None:
        _check(lib.pkv_sched_add(self.handle, request_id, prompt_len, max_new_tokens), "pkv_sched_add")

    def step(self) -> dict:
        _check(lib.pkv_sched_step(self.handle, ctypes.byref(self._batch)), "pkv_sched_step")
        b, a = self._batch, self._arr
        return dict(request_ids=a["request_ids"][:b.num_seqs].copy(), seq_ids=a["seq_ids"][:b.num_seqs].copy(),
                    query_lens=a["query_lens"][:b.num_seqs].copy(),
                    context_lens=a["context_lens"][:b.num_seqs].copy(), slots=a["slots"][:b.num_tokens].copy(),
                    finished=a["finished_ids"][:b.num_finished].copy(),
                    preempted=a["preempted_ids"][:b.num_preempted].copy())

    @property
    def num_waiting(self) -> int:
        return int(lib.pkv_sched_num_waiting(self.handle))

    @property
    def num_running(self) -> int:
        return int(lib.pkv_sched_num_running(self.handle))

    def close(self):
        if self.handle:
            lib.pkv_sched_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
