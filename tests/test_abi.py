"""The C-ABI library loads on a CPU-only host and exports every symbol that
include/pkv.h declares; invalid arguments are refused before any launch."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        for m in re.finditer(r"\b(pkv_\w+)\s*\([^;{]*\)\s*;", text):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("pkv_append", "pkv_decode_attention", "pkv_decode_workspace_bytes", "pkv_alloc_create",
                 "pkv_block_alloc", "pkv_block_incref", "pkv_block_decref", "pkv_seq_fork",
                 "pkv_seq_append_slot", "pkv_seq_free", "pkv_get_last_error"):
        assert must in names


def test_library_exports_every_declared_symbol():
    import paged_kv_cache_437_b200 as pkv

    lib = ctypes.CDLL(pkv.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    out = subprocess.run(["nm", "-D", "--defined-only", pkv.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    assert set(declared_functions()) <= exported


def test_status_strings():
    import paged_kv_cache_437_b200 as pkv

    assert pkv.pkv_status_string(pkv.PKV_OK) == "ok"
    assert "out of" in pkv.pkv_status_string(pkv.PKV_ERR_OOM)
    assert pkv.pkv_status_string(123) == "unknown status"


def _cache(pkv, **kw):
    base = dict(data=0x10000, dtype=pkv.PKV_F16, num_blocks=8, block_size=16, num_kv_heads=2, head_dim=128)
    base.update(kw)
    return pkv.pkv_cache(base["data"], base["dtype"], base["num_blocks"], base["block_size"],
                         base["num_kv_heads"], base["head_dim"], None)


@pytest.mark.parametrize("bad", [
    dict(head_dim=96), dict(block_size=8), dict(block_size=24), dict(num_kv_heads=3),
    dict(dtype=7), dict(data=0x10008), dict(data=0), dict(num_blocks=0),
])
def test_decode_rejects_bad_cache(bad):
    import paged_kv_cache_437_b200 as pkv

    kc = _cache(pkv, **bad)
    vc = _cache(pkv, **{k: v for k, v in bad.items() if k != "data"})
    st = pkv.lib.pkv_decode_attention(0x20000, 2, 4, kc, vc, 0x30000, 4, 0x40000, 0.1, 0x50000, None, 0,
                                      pkv.PKV_PARTITION_NONE, None)
    assert st == pkv.PKV_ERR_INVALID


@pytest.mark.parametrize("case", ["ragged_heads", "bad_partition", "misaligned_q", "null_out", "neg_seqs",
                                  "partition_without_ws", "shape_mismatch", "nan_scale"])
def test_decode_rejects_bad_args(case):
    import paged_kv_cache_437_b200 as pkv

    kc, vc = _cache(pkv), _cache(pkv)
    args = dict(q=0x20000, B=2, Hq=4, tables=0x30000, mb=4, lens=0x40000, scale=0.1, out=0x50000,
                ws=None, wsb=0, part=pkv.PKV_PARTITION_NONE)
    if case == "ragged_heads":
        args["Hq"] = 5
    elif case == "bad_partition":
        args.update(part=24, ws=0x60000, wsb=1 << 30)
    elif case == "misaligned_q":
        args["q"] = 0x20002
    elif case == "null_out":
        args["out"] = None
    elif case == "neg_seqs":
        args["B"] = -1
    elif case == "partition_without_ws":
        args["part"] = 512
    elif case == "shape_mismatch":
        vc = _cache(pkv, num_blocks=9)
    elif case == "nan_scale":
        args["scale"] = float("nan")
    st = pkv.lib.pkv_decode_attention(args["q"], args["B"], args["Hq"], kc, vc, args["tables"], args["mb"],
                                      args["lens"], args["scale"], args["out"], args["ws"], args["wsb"],
                                      args["part"], None)
    assert st == pkv.PKV_ERR_INVALID


def test_empty_batch_is_a_noop():
    import paged_kv_cache_437_b200 as pkv

    kc, vc = _cache(pkv), _cache(pkv)
    assert pkv.lib.pkv_decode_attention(None, 0, 4, kc, vc, None, 4, None, 0.1, None, None, 0,
                                        pkv.PKV_PARTITION_AUTO, None) == pkv.PKV_OK
    assert pkv.lib.pkv_append(None, None, None, 0, kc, vc, None) == pkv.PKV_OK


@pytest.mark.parametrize("case", ["neg_tokens", "misaligned_new", "null_slots", "mismatch"])
def test_append_rejects_bad_args(case):
    import paged_kv_cache_437_b200 as pkv

    kc, vc = _cache(pkv), _cache(pkv)
    a = dict(k=0x20000, v=0x30000, s=0x40000, T=3)
    if case == "neg_tokens":
        a["T"] = -1
    elif case == "misaligned_new":
        a["k"] = 0x20004
    elif case == "null_slots":
        a["s"] = None
    elif case == "mismatch":
        vc = _cache(pkv, head_dim=64)
    assert pkv.lib.pkv_append(a["k"], a["v"], a["s"], a["T"], kc, vc, None) == pkv.PKV_ERR_INVALID


def test_workspace_query_without_gpu_is_zero_or_sized():
    import paged_kv_cache_437_b200 as pkv

    assert pkv.pkv_decode_workspace_bytes(4, 8, 2, 128, 4096, pkv.PKV_PARTITION_NONE) == 0
    assert pkv.pkv_decode_workspace_bytes(4, 8, 2, 96, 4096, 512) == 0      # bad head_dim
    assert pkv.pkv_decode_workspace_bytes(4, 8, 3, 128, 4096, 512) == 0     # Hq % Hkv


def test_binding_without_the_library_fails_loudly(tmp_path):
    """No CPU fallback: a copy of the package without libpkv.so refuses to import."""
    import shutil
    import subprocess
    import sys

    src = os.path.join(ROOT, "paged_kv_cache_437_b200")
    dst = tmp_path / "paged_kv_cache_437_b200"
    shutil.copytree(src, dst, ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    r = subprocess.run([sys.executable, "-c", "import paged_kv_cache_437_b200"], cwd=tmp_path,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "not built" in r.stderr
