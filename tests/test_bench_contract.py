"""The GPU-free parts of bench.py: the algorithmic byte count behind every
roofline figure, the lookup of profiled DRAM traffic by kernel-source hash,
and the JSON line of the reference arm (the fp64 oracle on the host)."""
import json
import os
import subprocess
import sys

import pytest

import bench
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# KV bytes of every context position (K and V, every KV head, 2-byte
# elements) + Q + O + 4 bytes per used block-table entry + 4 per length,
# worked out by hand from each workload's shape:
#   tiny:  (17+33+64+100) * 2*4*64*2 + 2*4*4*64*2 + (2+3+4+7)*4 + 4*4
#   13B:   32*2048 * 2*40*128*2 + 2*32*40*128*2 + 32*128*4 + 32*4
#   70B:   30*4096 * 2*8*128*2 + 2*30*64*128*2 + 30*256*4 + 30*4
#   long:  2*65536 * 2*8*128*2 + 2*2*64*128*2 + 2*4096*4 + 2*4
EXPECTED = {
    "tiny": 214 * 1024 + 4096 + 64 + 16,
    "llama13b": 65536 * 20480 + 655360 + 16384 + 128,
    "llama70b_gqa": 122880 * 4096 + 983040 + 30720 + 120,
    "long_split": 131072 * 4096 + 65536 + 32768 + 8,
}


@pytest.mark.parametrize("name", sorted(EXPECTED))
def test_algorithmic_bytes_closed_form(name):
    w = workloads.make(name, fill_pool=False)
    assert bench.algorithmic_bytes(w)["total"] == EXPECTED[name]


def test_tiny_byte_count_matches_the_sizing_table():
    assert EXPECTED["tiny"] == 223_312
    assert EXPECTED["llama70b_gqa"] == 504_330_360


def test_profiled_traffic_is_keyed_to_the_kernel_sources(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "PROFILE_DIR", str(tmp_path))
    p = tmp_path / "paged_decode_tiny.md"
    p.write_text(f"# x\nkernel_sources_sha256_16: {bench.kernel_hash()}\ndram_bytes_per_launch: 12345\n")
    assert bench.profiled_traffic("tiny") == 12345
    p.write_text("# x\nkernel_sources_sha256_16: 0000000000000000\ndram_bytes_per_launch: 12345\n")
    assert bench.profiled_traffic("tiny") is None
    assert bench.profiled_traffic("no_such_workload") is None


def test_reference_arm_json_line():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "3", "--warmup", "3"], capture_output=True, text=True, timeout=300, env=env,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "GB/s" and line["higher_is_better"] is True and line["value"] > 0
    assert line["steps"] == 3 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["config"]["workload"] == "tiny"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"] and line["cpu_baseline"]["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_warmup_below_three_is_rejected():
    with pytest.raises(SystemExit):
        bench.parse_args(["--warmup", "2"])
