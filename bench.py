"""Benchmark one paged decode step (append + attention) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--partition P] [--flush-l2] [--impl reference]
    python bench.py --row cow|prefill|sched|fp8 [--workload NAME]

A step is the whole hot path on one batch: the append of every sequence's new
token and the attention (decode kernel + log-sum-exp merge when the schedule
splits contexts), by default through the fused pkv_append_decode_attention
call (``--unfused``: pkv_append then pkv_decode_attention).  Inputs are
synthetic and seeded (``workloads``), shaped like the pages' examples; the
default workload is the 13B-shaped layer (32 sequences x 2048 context, 40/40
heads, D 128, block 16, fp16).  ``--row`` measures one of the rows next to
the hot path instead (copy-on-write block copies, chunked prefill, the host
scheduler, E4M3 decode) and prints one JSON line tagged "row".

Metric: achieved HBM GB/s of algorithmic bytes (KV read for every sequence's
context + Q + O + used block-table entries + context lengths) per step time,
with decode tokens/s/layer beside it.  Device-timed with CUDA events on the
launching stream; the per-step KV working set is larger than L2, so no flush
is needed (``--flush-l2`` flushes anyway).  ``e2e`` repeats the step through
the same C ABI with the per-step inputs copied from pinned host memory and
the output copied back inside the timed region.

Multi-GPU: one process per GPU (torchrun); every rank runs its own replica of
the workload (the path has no exchange step), value = all ranks' bytes / the
slowest rank's time.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload (the reference arm); only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode attention: achieved HBM GB/s (% of B200 peak); decode tokens/s/layer"
DEFAULT_WORKLOAD = "llama13b"
PROFILE_DIR = os.path.join(ROOT, "profiles")
# the sources the decode kernel's profiled traffic depends on (its code, the
# instruction wrappers and the host plan that sizes its launch)
KERNEL_SOURCES = [os.path.join(ROOT, "paged_kv_cache_437_b200", "csrc", f)
                  for f in ("decode.cuh", "ptx.cuh", "pkv_cuda.cu")]


# ------------------------------------------------------------------ bytes

def algorithmic_bytes(w) -> dict:
    """Bytes the step must move at minimum, per the roofline definition:
    every sequence reads K and V of its whole context for every KV head, plus
    Q, O, the used block-table entries and the context lengths."""
    sp = w.spec
    e = 2  # fp16 / bf16
    ctx = w.context_lens.astype(np.int64)
    kv = int(ctx.sum()) * 2 * sp.num_kv_heads * sp.head_dim * e
    qo = 2 * sp.num_seqs * sp.num_q_heads * sp.head_dim * e
    used_blocks = -(-ctx // sp.block_size)
    tables = int(used_blocks.sum()) * 4
    lens = sp.num_seqs * 4
    total = kv + qo + tables + lens
    # shared prefix blocks counted once (their positions are read by every sharer)
    shared_tokens = 0
    seen = set()
    for s in range(sp.num_seqs):
        for i in range(w.shared_blocks[s]):
            b = int(w.block_tables[s, i])
            if b in seen:
                shared_tokens += sp.block_size
            seen.add(b)
    unique_kv = kv - shared_tokens * 2 * sp.num_kv_heads * sp.head_dim * e
    append = sp.num_seqs * 2 * sp.num_kv_heads * sp.head_dim * e * 2 + sp.num_seqs * 8
    return dict(total=total, kv=kv, qo=qo, tables=tables, lens=lens,
                unique_total=unique_kv + qo + tables + lens, append=append)


# ------------------------------------------------------------------ helpers

def nvtx(name: str):
    """An NVTX range around one phase of the run (visible to a system
    profiler), never inside a per-step loop."""
    import torch

    return torch.cuda.nvtx.range(name)


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        out = dict(hbm_gbs=float(d["hbm_gbs"]), source="measured")
        if "bf16_tflops" in d:
            out["bf16_tflops"] = float(d["bf16_tflops"])
        return out
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, source="fallback")


def kernel_hash() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per decode launch from the committed ncu summary of this
    workload, or None when there is none or the kernel changed since."""
    path = os.path.join(PROFILE_DIR, f"paged_decode_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    mh = re.search(r"kernel_sources_sha256_16:\s*([0-9a-f]+)", text)
    mt = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    if not mh or not mt or mh.group(1) != kernel_hash():
        return None
    return int(mt.group(1))


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.tmp = None

    def __enter__(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.tmp, stderr=subprocess.DEVNULL)
            time.sleep(0.25)
        except (OSError, ValueError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.tmp is None:
            return None
        rows = []
        with open(self.tmp.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(parts)
                except ValueError:
                    continue
        os.unlink(self.tmp.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ distributed plumbing

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def reduce_max(value: float, group=None) -> float:
    """Max over ranks of a per-rank number (timing only; no data-path exchange)."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized():
        return value
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def barrier():
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def weak_scaling_value(bytes_per_rank_step: int, world: int, steps: int, max_ms: float) -> float:
    """Whole-job GB/s: every rank's bytes over the slowest rank's time."""
    return bytes_per_rank_step * world * steps / (max_ms * 1e-3) / 1e9


# ------------------------------------------------------------------ GPU arm

def run_gpu(args, rank, world, local):
    import torch

    import paged_kv_cache_437_b200 as pkv
    import workloads

    torch.cuda.set_device(local)
    w = make_workload(args)
    sp = w.spec
    dt = torch.float16 if sp.dtype == workloads.F16 else torch.bfloat16
    nb_bytes = algorithmic_bytes(w)

    def dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dt).cuda()

    # slots of the new tokens from the library's own host allocator: the pool's
    # blocks are handed out in the workload's (seeded, shuffled) order by
    # returning them to the LIFO free list in reverse, then every sequence is
    # built up to ctx - 1 tokens (prefix blocks shared through fork).
    alloc = pkv.BlockAllocator(w.num_blocks, sp.block_size)
    slots_np, alloc_us, groups = allocator_slots(pkv, alloc, w)
    # --cascade: a workload whose sequences share prefix blocks runs its step
    # through the shared-prefix call (each group's prefix read once) instead of
    # the plain decode step
    cascade = groups is not None and args.cascade and not args.unfused

    q = dev(w.q)
    kc, vc = dev(w.k_cache), dev(w.v_cache)
    kn, vn = dev(w.k_new), dev(w.v_new)
    slots = torch.from_numpy(slots_np).cuda()
    tables = torch.from_numpy(np.ascontiguousarray(w.block_tables)).cuda()
    lens = torch.from_numpy(np.ascontiguousarray(w.context_lens)).cuda()
    out = torch.empty_like(q)
    part = args.partition
    ws = None
    if part != pkv.PKV_PARTITION_NONE:
        n = pkv.pkv_decode_workspace_bytes(sp.num_seqs, sp.num_q_heads, sp.num_kv_heads, sp.head_dim,
                                           w.max_blocks_per_seq * sp.block_size, part)
        ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    merge_launched = part != pkv.PKV_PARTITION_NONE and not (
        part > 0 and -(-w.max_blocks_per_seq * sp.block_size // part) <= 1)
    launches_per_step = (1 if not args.unfused else 2) + (1 if merge_launched else 0)
    if cascade:
        starts_np, claims_np = groups
        gstart = torch.from_numpy(starts_np).cuda()
        claims = torch.from_numpy(claims_np).cuda()
        ngroups = len(starts_np) - 1
        n = pkv.pkv_shared_prefix_workspace_bytes(sp.num_seqs, sp.num_q_heads, sp.num_kv_heads, sp.head_dim,
                                                  w.max_blocks_per_seq * sp.block_size, ngroups)
        ws = torch.empty(n, dtype=torch.uint8, device="cuda")
        launches_per_step = 4  # preparation, shared-prefix kernel, decode kernel, merge
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda") if args.flush_l2 else None

    # the C ABI calls with their arguments marshalled once (the Python
    # binding's checks ran above; the timed loops make the raw calls)
    import ctypes

    sptr = ctypes.c_void_p(stream.cuda_stream)
    kdesc, vdesc = pkv.cache_desc(kc), pkv.cache_desc(vc)
    append_args = (kn.data_ptr(), vn.data_ptr(), slots.data_ptr(), slots.numel(), kdesc, vdesc, sptr)
    ws_ptr = ws.data_ptr() if ws is not None else None
    ws_bytes = ws.numel() if ws is not None else 0
    decode_args = (q.data_ptr(), q.shape[0], q.shape[1], kdesc, vdesc, tables.data_ptr(), tables.shape[1],
                   lens.data_ptr(), ctypes.c_float(w.scale), out.data_ptr(), ws_ptr, ws_bytes, part, sptr)
    c_append, c_decode = pkv.lib.pkv_append, pkv.lib.pkv_decode_attention
    c_fused = pkv.lib.pkv_append_decode_attention
    fused_args = (kn.data_ptr(), vn.data_ptr(), slots.data_ptr()) + decode_args
    if cascade:
        # the step's one call: append + shared-prefix decode
        c_fused = pkv.lib.pkv_append_decode_attention_shared_prefix
        fused_args = (kn.data_ptr(), vn.data_ptr(), slots.data_ptr(), q.data_ptr(), q.shape[0], q.shape[1], kdesc,
                      vdesc, tables.data_ptr(), tables.shape[1], lens.data_ptr(), gstart.data_ptr(), ngroups,
                      claims.data_ptr(), ctypes.c_float(w.scale), out.data_ptr(), ws_ptr, ws_bytes, sptr)

    def make_step(q, kn, vn, slots, tables, lens, gstart=None, claims=None, out=out):
        """The step's raw C ABI calls on these device inputs (and output)."""
        a_args = (kn.data_ptr(), vn.data_ptr(), slots.data_ptr(), slots.numel(), kdesc, vdesc, sptr)
        d_args = (q.data_ptr(), q.shape[0], q.shape[1], kdesc, vdesc, tables.data_ptr(), tables.shape[1],
                  lens.data_ptr(), ctypes.c_float(w.scale), out.data_ptr(), ws_ptr, ws_bytes, part, sptr)
        f_args = (kn.data_ptr(), vn.data_ptr(), slots.data_ptr()) + d_args
        if cascade:
            f_args = (kn.data_ptr(), vn.data_ptr(), slots.data_ptr(), q.data_ptr(), q.shape[0], q.shape[1], kdesc,
                      vdesc, tables.data_ptr(), tables.shape[1], lens.data_ptr(), gstart.data_ptr(), ngroups,
                      claims.data_ptr(), ctypes.c_float(w.scale), out.data_ptr(), ws_ptr, ws_bytes, sptr)
        if args.unfused:
            def step():
                c_append(*a_args)
                c_decode(*d_args)
        else:
            def step():
                c_fused(*f_args)
        return step

    step_inputs = (q, kn, vn, slots, tables, lens) + ((gstart, claims) if cascade else ())
    step = make_step(*step_inputs)

    # the binding path once, with its argument checks
    pkv.pkv_append(kn, vn, slots, kc, vc, stream)
    pkv.pkv_decode_attention(q, kc, vc, tables, lens, w.scale, out, ws, part, stream)
    if cascade:
        pkv.pkv_append_decode_attention_shared_prefix(kn, vn, slots, q, kc, vc, tables, lens, gstart, claims,
                                                      w.scale, out, ws, stream)
    else:
        pkv.pkv_append_decode_attention(kn, vn, slots, q, kc, vc, tables, lens, w.scale, out, ws, part, stream)
    with nvtx("pkv warm-up"):
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
    if pkv.pkv_get_last_error() != pkv.PKV_OK:
        raise RuntimeError("device check failed during warm-up")

    ev = lambda: torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        # K whole steps, events only around the region (no events between the
        # kernels, so each launch can overlap the previous kernel's tail)
        t0, t1 = ev(), ev()
        with nvtx("pkv timed steps"):
            t0.record(stream)
            for i in range(args.steps):
                if flush is not None:
                    flush.zero_()
                step()
            t1.record(stream)
            torch.cuda.synchronize()
        barrier()
        step_ms = t0.elapsed_time(t1)
        # the dominant kernel: K launches of the decode kernel (the fused
        # append + decode call of the step, or the decode call alone) back to
        # back, plus its merge when contexts are split
        d0, d1 = ev(), ev()
        with nvtx("pkv dominant kernel"):
            d0.record(stream)
            for i in range(args.steps):
                if args.unfused:
                    c_decode(*decode_args)
                else:
                    c_fused(*fused_args)
            d1.record(stream)
            torch.cuda.synchronize()
    barrier()
    dec_ms = d0.elapsed_time(d1) / args.steps
    if flush is not None:
        # the flush runs inside the step region: subtract its own time
        f0, f1 = ev(), ev()
        f0.record(stream)
        for _ in range(args.steps):
            flush.zero_()
        f1.record(stream)
        torch.cuda.synchronize()
        step_ms -= f0.elapsed_time(f1)
    max_ms = reduce_max(step_ms)
    if pkv.pkv_get_last_error() != pkv.PKV_OK:
        raise RuntimeError("device check failed in the timed region")

    # ---- end to end through the C ABI with host buffers
    with nvtx("pkv end-to-end"):
        e2e = None if args.no_e2e else measure_e2e(args, make_step, stream, step_inputs, out)
    peaks = load_peaks()
    ms_per_step = max_ms / args.steps
    value = weak_scaling_value(nb_bytes["total"], world, args.steps, max_ms)
    achieved = nb_bytes["total"] / (dec_ms * 1e-3) / 1e9
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": workloads.DTYPE_NAMES[sp.dtype],
        "data": "synthetic (seeded N(0,1), shapes of the pages' examples)",
        "config": {
            "workload": sp.name,
            "description": sp.description,
            "num_seqs": sp.num_seqs,
            "context_tokens_total": int(w.context_lens.sum()),
            "max_context": int(w.context_lens.max()),
            "num_q_heads": sp.num_q_heads,
            "num_kv_heads": sp.num_kv_heads,
            "head_dim": sp.head_dim,
            "block_size": sp.block_size,
            "pool_blocks": w.num_blocks,
            "partition": {0: "auto (work-balanced)", -1: "none"}.get(part, f"{part} tokens"),
            "products": "ffma (CUDA-core variant)" if os.environ.get("PKV_FMA") == "1" else "mma m16n8k16",
            "l2": "flushed between steps" if args.flush_l2 else "per-step KV working set > L2 (no flush)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "step_call": ("pkv_append + pkv_decode_attention" if args.unfused else
                          "pkv_append_decode_attention_shared_prefix" if cascade else "pkv_append_decode_attention"),
        },
        "tokens_per_s_per_layer": round(sp.num_seqs * world / (ms_per_step * 1e-3), 1),
        "algorithmic_bytes_per_step": nb_bytes["total"],
        "unique_bytes_per_step": nb_bytes["unique_total"],
        "frac_of_8TBs": round(value / world / 8000.0, 4),
        "frac_of_measured_hbm": round(value / world / peaks["hbm_gbs"], 4),
        "roofline": {
            "bound": "hbm",
            # the split rows are merged by lse_merge_kernel or, where rows
            # split into few pieces, inside the decode kernel (fold_zero_kernel
            # then zeroes its counters): the library decides per shape
            "kernel": ("cascade_prep_kernel+mq_attention_kernel+" if cascade else "") + "paged_decode_kernel" +
                      ("+merge of split rows" if merge_launched else ""),
            "achieved": round(achieved, 2),
            "peak": peaks["hbm_gbs"],
            "peak_source": peaks["source"],
            "unit": "GB/s",
            "frac": round(achieved / peaks["hbm_gbs"], 4),
            # shared-prefix blocks counted once: the bandwidth really needed
            "frac_unique": round(nb_bytes["unique_total"] / (dec_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            # the committed profile covers the plain decode step only
            "traffic": None if cascade else profiled_traffic(sp.name),
            "algorithmic_bytes_per_launch": nb_bytes["total"],
            "us_per_launch": round(dec_ms * 1e3, 3),
        },
        "e2e": None if e2e is None else {
            "value": round(weak_scaling_value(nb_bytes["total"], world, args.steps, e2e["ms"]), 2),
            "unit": "GB/s",
            "h2d_bytes_per_step": e2e["h2d"],
            "d2h_bytes_per_step": e2e["d2h"],
            "ms_per_step": round(e2e["ms"] / args.steps, 5),
            "copies_per_step": e2e["copies_per_step"],
        },
        # the host allocator's per-step work (append slots + batch tables) is
        # not on the device timeline; this adds its measured time to e2e's
        "e2e_with_alloc": None if e2e is None else {
            "value": round(nb_bytes["total"] * world / ((e2e["ms"] / args.steps + alloc_us * 1e-3) * 1e-3) / 1e9, 2),
            "unit": "GB/s",
            "ms_per_step": round(e2e["ms"] / args.steps + alloc_us * 1e-3, 5),
        },
        "allocator_us_per_step": round(alloc_us, 2),
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        result["cpu_baseline"] = cpu_baseline(w, nb_bytes, args.cpu_seconds)
    alloc.close()
    return result


def _build_sequences(alloc, w):
    """Create the workload's sequences through the allocator: one holder
    sequence per sharing group owns the group's prefix blocks, members fork
    it (refcounted sharing of whole blocks) and grow to ctx - 1 tokens."""
    sp = w.spec
    holders = {}
    if sp.share_group:
        for s in range(sp.num_seqs):
            g = s // sp.share_group
            holders[g] = max(holders.get(g, 0), w.shared_blocks[s])
        for g in sorted(holders):
            h = alloc.seq_create()
            for _ in range(holders[g] * sp.block_size):
                alloc.append_slot(h)
            holders[g] = h
    seqs = []
    for s in range(sp.num_seqs):
        if sp.share_group:
            seq = alloc.seq_fork(holders[s // sp.share_group], w.shared_blocks[s])
        else:
            seq = alloc.seq_create()
        while alloc.context_len(seq) < int(w.context_lens[s]) - 1:
            alloc.append_slot(seq)
        seqs.append(seq)
    return seqs, holders


def measure_e2e(args, make_step, stream, inputs, out):
    """The same step through the C ABI with the per-step inputs in pinned host
    memory: q, the new K/V, slots, tables and lengths (and the sharing groups,
    when the step uses them) packed into one pinned staging buffer and sent
    with one host-to-device copy, the kernels, and one device-to-host copy of
    the output, all inside the timed region.  As a serving loop would, the
    copies run on their own stream, double-buffered: step k+1's inputs go up
    and step k-1's output comes down while step k computes."""
    import torch

    offs, off = [], 0
    for t in inputs:
        off = (off + 255) // 256 * 256           # every input 256-byte aligned in the buffer
        offs.append(off)
        off += t.numel() * t.element_size()
    h_buf = torch.empty(off, dtype=torch.uint8).pin_memory()
    for t, o in zip(inputs, offs):
        n = t.numel() * t.element_size()
        h_buf[o:o + n].copy_(t.reshape(-1).view(torch.uint8).cpu())
    d_buf = [torch.empty(off, dtype=torch.uint8, device="cuda") for _ in range(2)]
    d_out = [torch.empty_like(out) for _ in range(2)]
    h_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    steps = []
    for b in range(2):
        views = [d_buf[b][o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
                 for t, o in zip(inputs, offs)]
        steps.append(make_step(*views, out=d_out[b]))
    h2d = sum(t.numel() * t.element_size() for t in inputs)
    d2h = h_out[0].numel() * h_out[0].element_size()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()  # uploads never queue behind downloads
    ev = lambda: torch.cuda.Event()
    in_ready = [ev(), ev()]
    computed = [ev(), ev()]
    out_done = [ev(), ev()]
    started = [False, False]

    def run(n):
        for k in range(n):
            b = k & 1
            with torch.cuda.stream(up):
                if started[b]:
                    up.wait_event(computed[b])                # step k-2 has read d_buf[b]
                d_buf[b].copy_(h_buf, non_blocking=True)
                in_ready[b].record(up)
            stream.wait_event(in_ready[b])
            if started[b]:
                stream.wait_event(out_done[b])                # step k-2's output is down
            steps[b]()
            computed[b].record(stream)
            started[b] = True
            with torch.cuda.stream(down):
                down.wait_event(computed[b])
                h_out[b].copy_(d_out[b], non_blocking=True)
                out_done[b].record(down)

    run(max(2, args.warmup))
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(up)
    stream.wait_event(e0)
    down.wait_event(e0)
    run(args.steps)
    # the region ends when the last output is on the host
    down.wait_stream(stream)
    down.wait_stream(up)
    e1.record(down)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1))
    barrier()
    return dict(ms=e2e_ms, h2d=h2d, d2h=d2h, copies_per_step=2)


def allocator_slots(pkv, alloc, w):
    """Build the workload's tables through the library's host allocator and
    return the slots of this step's new tokens and the allocator's host time
    per step (us).  A dry run on a scratch allocator (whose pops come out
    0, 1, 2, ...) shows which table entry each pop serves; returning the pool
    to the real allocator's LIFO free list in the reverse of the wanted order
    then makes its pops reproduce the workload's seeded block assignment."""
    sp = w.spec
    scratch = pkv.BlockAllocator(w.num_blocks, sp.block_size)
    seqs, holders = _build_sequences(scratch, w)
    scratch.append_slots(seqs)
    want = {}
    for s, seq in enumerate(seqs):
        for i, k in enumerate(scratch.block_table(seq)):
            want[int(k)] = int(w.block_tables[s, i])
    scratch.close()
    order = [want[k] for k in range(len(want))]
    rest = sorted(set(range(w.num_blocks)) - set(order))
    got = [alloc.alloc() for _ in range(w.num_blocks)]
    assert got == list(range(w.num_blocks))
    for b in reversed(order + rest):
        alloc.decref(b)
    seqs, holders = _build_sequences(alloc, w)
    for h in holders.values():
        alloc.seq_free(h)
    t0 = time.perf_counter()
    slots = alloc.append_slots(seqs)
    tables, lens = alloc.batch_tables(seqs, w.max_blocks_per_seq)
    groups = alloc.prefix_groups(seqs) if w.spec.share_group else None
    alloc_us = (time.perf_counter() - t0) * 1e6
    if not (np.array_equal(tables, w.block_tables) and np.array_equal(lens, w.context_lens)):
        raise RuntimeError("allocator tables differ from the workload's")
    return slots, alloc_us, groups


# ------------------------------------------------------------------ CPU oracle (baseline / reference arm)

def pair_share_bytes(w, s: int) -> float:
    """Algorithmic bytes attributable to one (sequence, query head) pair."""
    sp = w.spec
    g = sp.num_q_heads // sp.num_kv_heads
    ctx = int(w.context_lens[s])
    kv = ctx * 2 * sp.head_dim * 2 / g
    return kv + 2 * sp.head_dim * 2 + (-(-ctx // sp.block_size) * 4 + 4) / sp.num_q_heads


def cpu_baseline(w, nb_bytes, seconds: float) -> dict:
    import oracle

    sp = w.spec
    rng = np.random.default_rng(123)
    pairs_all = np.array([(s, h) for s in range(sp.num_seqs) for h in range(sp.num_q_heads)], dtype=np.int64)
    rng.shuffle(pairs_all)
    oracle.load()
    cores = oracle.num_threads()
    # pilot to size the sample: about `seconds` of oracle work, the whole
    # workload repeated if it is shorter than that
    pilot = pairs_all[:max(1, cores)]
    t0 = time.perf_counter()
    oracle.attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, sp.dtype, pairs=pilot)
    t_pilot = max(time.perf_counter() - t0, 1e-4)
    n = int(min(len(pairs_all), max(len(pilot), len(pilot) * seconds / t_pilot)))
    sample = pairs_all[:n]
    done = 0.0
    reps = 0
    t0 = time.perf_counter()
    while True:
        oracle.attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, sp.dtype,
                         pairs=sample)
        reps += 1
        done += sum(pair_share_bytes(w, int(s)) for s, _ in sample)
        dt = time.perf_counter() - t0
        if dt >= seconds or reps >= 1000:
            break
    value = done / dt / 1e9
    # the same oracle on one host core, on a smaller sample (about a fifth of
    # the time budget)
    one = None
    if cores > 1:
        oracle.set_num_threads(1)
        try:
            n1 = max(1, int(n * (seconds / 5) / (dt / reps) / cores))
            s1 = sample[:min(n1, len(sample))]
            t1 = time.perf_counter()
            oracle.attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, sp.dtype,
                             pairs=s1)
            d1 = time.perf_counter() - t1
            one = {"value": round(sum(pair_share_bytes(w, int(s)) for s, _ in s1) / d1 / 1e9, 4), "unit": "GB/s",
                   "cores": 1, "sample": f"{len(s1)} pairs, {d1:.1f} s"}
        finally:
            oracle.set_num_threads(cores)
    return {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"{n} of {len(pairs_all)} (sequence, query head) pairs of {sp.name} x {reps}, fp64 C "
                      f"oracle (gather through block tables + two-pass softmax), {dt:.1f} s",
            "seconds": round(dt, 2), "one_core": one if one is not None else {"value": round(value, 4), "cores": 1}}


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or the platform's."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform

    return platform.processor() or platform.machine()


def make_workload(args):
    import dataclasses

    import workloads

    spec = workloads.CONFIGS[args.workload]
    if args.seqs:
        n = min(args.seqs, spec.num_seqs)
        kw = dict(num_seqs=n, name=f"{spec.name}_first{n}")
        if spec.context_lens is not None:
            kw["context_lens"] = spec.context_lens[:n]
        if spec.num_blocks is not None:
            kw["num_blocks"] = None
        spec = dataclasses.replace(spec, **kw)
    return workloads.make(spec)


def run_reference(args, rank, world):
    import oracle

    w = make_workload(args)
    sp = w.spec
    nb_bytes = algorithmic_bytes(w)
    oracle.load()
    cores = oracle.num_threads()
    rng = np.random.default_rng(7)
    pairs_all = np.array([(s, h) for s in range(sp.num_seqs) for h in range(sp.num_q_heads)], dtype=np.int64)
    rng.shuffle(pairs_all)
    # each step: a bounded sample, sized so the whole run stays within minutes
    budget = max(2.0, args.cpu_seconds) / max(1, args.steps + args.warmup)
    pilot = pairs_all[:max(1, cores)]
    t0 = time.perf_counter()
    oracle.attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, sp.dtype, pairs=pilot)
    t_pilot = max(time.perf_counter() - t0, 1e-4)
    n = int(min(len(pairs_all), max(len(pilot), len(pilot) * budget / t_pilot)))
    sample = pairs_all[:n]
    share = sum(pair_share_bytes(w, int(s)) for s, _ in sample)
    for _ in range(args.warmup):
        oracle.attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, sp.dtype,
                         pairs=sample)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, sp.dtype,
                         pairs=sample)
    dt = time.perf_counter() - t0
    value = share * args.steps / dt / 1e9
    # time per full step, extrapolated from the sample's share of the bytes
    ms_full = dt / args.steps * (nb_bytes["total"] / share) * 1e3
    sample_desc = (f"{n} of {len(pairs_all)} (sequence, query head) pairs of {sp.name} per step, fp64 C oracle "
                   f"on {cores} host threads")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_full, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded N(0,1), shapes of the pages' examples)",
        "config": {"workload": sp.name, "description": sp.description, "parallelism": "host CPU"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "cpu_model": cpu_model(), "sample": sample_desc},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


# ------------------------------------------------------------------ main

# ------------------------------------------------------------------ NEXT rows

def run_row(args) -> dict:
    """Measurements of the rows next to the hot path (one JSON line each)."""
    import torch

    import paged_kv_cache_437_b200 as pkv
    import workloads

    rng = np.random.default_rng(5)
    if args.row == "sched":
        alloc = pkv.BlockAllocator(65536, 16)
        sched = pkv.Scheduler(alloc, max_batch_tokens=8192, max_seqs=256, chunk_tokens=512)
        lens = np.clip(np.exp(rng.uniform(np.log(16), np.log(4096), 1024)), 16, 4096).astype(int)
        for i, p in enumerate(lens):
            sched.add(i, int(p), int(rng.integers(16, 256)))
        t0 = time.perf_counter()
        steps = tokens = 0
        while (sched.num_waiting or sched.num_running) and steps < 2000:
            b = sched.step()
            steps += 1
            tokens += len(b["slots"])
        dt = time.perf_counter() - t0
        return {"row": "scheduler", "metric": "host scheduler step time", "value": round(dt / steps * 1e6, 2),
                "unit": "us/step", "higher_is_better": False, "steps": steps, "tokens": tokens,
                "config": {"requests": 1024, "prompt": "log-uniform [16, 4096]", "max_new": "uniform [16, 256)",
                           "max_batch_tokens": 8192, "max_seqs": 256, "chunk_tokens": 512, "pool_blocks": 65536}}

    torch.cuda.set_device(0)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    if args.row == "cow":
        nb, hkv, bs, d = 8192, 40, 16, 128          # 13B-shaped blocks: 160 KB of K + 160 KB of V
        kc = torch.randn((nb, hkv, bs, d), dtype=torch.float16, device="cuda")
        vc = torch.randn_like(kc)
        n = 2048
        perm = rng.permutation(nb)
        pairs = torch.from_numpy(np.stack([perm[:n], perm[n:2 * n]], 1).astype(np.int32)).cuda()
        for _ in range(args.warmup):
            pkv.pkv_copy_blocks(kc, vc, pairs)
        t0, t1 = ev(), ev()
        t0.record()
        for _ in range(args.steps):
            pkv.pkv_copy_blocks(kc, vc, pairs)
        t1.record()
        torch.cuda.synchronize()
        ms = t0.elapsed_time(t1) / args.steps
        moved = n * 2 * (hkv * bs * d * 2) * 2     # read + write of K and V blocks
        return {"row": "copy_on_write", "metric": "block copy HBM GB/s (read + write)",
                "value": round(moved / (ms * 1e-3) / 1e9, 1), "unit": "GB/s", "ms_per_call": round(ms, 4),
                "peak": load_peaks()["hbm_gbs"], "config": {"pairs": n, "block": [hkv, bs, d], "dtype": "f16"}}

    if args.row == "prefill":
        # 70B-shaped layer: 2 prompts of a 2048-token prefix + one 512-token
        # chunk each, interleaved with 30 decode sequences of 4096 context
        hq, hkv, d, bs = 64, 8, 128, 16
        chunks = [(2048 + 512, 512)] * 2 + [(4096, 1)] * 30
        ctx = np.array([c for c, _ in chunks], np.int32)
        nq = np.array([n for _, n in chunks], np.int32)
        qs = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
        t = int(qs[-1])
        nblk = -(-ctx // bs)
        mb = int(nblk.max())
        nb = int(nblk.sum()) + 8
        perm = rng.permutation(nb).astype(np.int32)
        tables = np.full((len(chunks), mb), -1, np.int32)
        cur = 0
        for i, k in enumerate(nblk):
            tables[i, :k] = perm[cur:cur + k]
            cur += k
        kc = torch.randn((nb, hkv, bs, d), dtype=torch.bfloat16, device="cuda")
        vc = torch.randn_like(kc)
        q = torch.randn((t, hq, d), dtype=torch.bfloat16, device="cuda")
        out = torch.empty_like(q)
        ws = torch.empty(pkv.pkv_prefill_workspace_bytes(t, hq, hkv, d, mb * bs), dtype=torch.uint8, device="cuda")
        td, qsd, cd = (torch.from_numpy(x).cuda() for x in (tables, qs, ctx))

        def timed(mq: bool, nseq: int = len(chunks)) -> float:
            # nseq < len(chunks): the first nseq sequences only (the chunks)
            os.environ["PKV_PREFILL_MQ"] = "1" if mq else "0"
            tt = int(qs[nseq])
            qq, oo = q[:tt], out[:tt]
            tq, qq_s, cc = td[:nseq], qsd[:nseq + 1], cd[:nseq]
            try:
                for _ in range(args.warmup):
                    pkv.pkv_prefill_attention(qq, kc, vc, tq, qq_s, cc, 0.088, oo, ws)
                t0, t1 = ev(), ev()
                t0.record()
                for _ in range(args.steps):
                    pkv.pkv_prefill_attention(qq, kc, vc, tq, qq_s, cc, 0.088, oo, ws)
                t1.record()
                torch.cuda.synchronize()
            finally:
                os.environ.pop("PKV_PREFILL_MQ", None)
            if pkv.pkv_get_last_error() != pkv.PKV_OK:
                raise RuntimeError("device check failed in the prefill row")
            return t0.elapsed_time(t1) / args.steps

        if args.chunks_only:
            # profiling case: the two prefill chunks alone, multi-query kernel only
            ms_chunks = timed(True, 2)
            return {"row": "chunked_prefill_chunks_only", "ms_per_step": round(ms_chunks, 4),
                    "steps": args.steps, "warmup": args.warmup}
        ms = timed(True)
        ms_tok = timed(False)
        ms_chunks = timed(True, 2)     # the two prefill chunks alone (multi-query kernel)
        # work: each query token attends to its causal window
        windows = np.concatenate([np.arange(c - n + 1, c + 1) for c, n in chunks]).astype(np.int64)
        flops = int(windows.sum()) * hq * d * 2 * 2
        flops_chunks = int(windows[:int(qs[2])].sum()) * hq * d * 2 * 2
        unique = int((ctx.astype(np.int64)).sum()) * hkv * d * 2 * 2
        peaks = load_peaks()
        bf16_peak = peaks.get("bf16_tflops", 1590.0)
        t_hbm = unique / (peaks["hbm_gbs"] * 1e9)
        t_tc = flops / (bf16_peak * 1e12)
        bound_s = max(t_hbm, t_tc)
        return {"row": "chunked_prefill", "metric": "chunked prefill + decode step: query tokens/s",
                "value": round(t / (ms * 1e-3), 1), "unit": "tokens/s", "ms_per_step": round(ms, 4),
                "ms_per_step_per_token_path": round(ms_tok, 4),
                "ms_chunks_only": round(ms_chunks, 4),
                "chunks_only_tflops": round(flops_chunks / (ms_chunks * 1e-3) / 1e12, 2),
                "speedup_vs_per_token_path": round(ms_tok / ms, 3),
                "tflops": round(flops / (ms * 1e-3) / 1e12, 2), "unique_kv_gbs": round(unique / (ms * 1e-3) / 1e9, 1),
                "roofline": {"bound": "hbm" if t_hbm >= t_tc else "tensor", "bound_us": round(bound_s * 1e6, 2),
                             "hbm_us": round(t_hbm * 1e6, 2), "tensor_us": round(t_tc * 1e6, 2),
                             "frac": round(bound_s / (ms * 1e-3), 4), "hbm_peak_gbs": peaks["hbm_gbs"],
                             "bf16_peak_tflops": bf16_peak, "peak_source": peaks["source"]},
                "flops": flops, "unique_kv_bytes": unique,
                "config": {"shape": "70B GQA 64/8, D128, bs16, bf16", "prefill": "2 x (2048 prefix + 512 chunk)",
                           "decode": "30 x 4096", "query_tokens": t,
                           "kernels": "multi-query tcgen05 kernel for the chunks, decode kernel for the decode tokens"}}

    if args.row == "fp8":
        # the workload's decode over E4M3 pools (1 byte per element + one fp32
        # scale per row) beside the same decode over its 16-bit pools; K
        # launches back to back between two events, like the dominant-kernel
        # loop of the main step (both working sets are larger than L2)
        w = make_workload(args)
        sp = w.spec
        dt = torch.float16 if sp.dtype == workloads.F16 else torch.bfloat16
        dev16 = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dt).cuda()
        shape = w.k_cache.shape
        gen = torch.Generator(device="cuda").manual_seed(11)

        def codes():  # any finite E4M3 code: magnitude bits 0x00..0x7e, random sign
            mag = torch.randint(0, 0x7f, shape, generator=gen, device="cuda", dtype=torch.int16)
            sign = torch.randint(0, 2, shape, generator=gen, device="cuda", dtype=torch.int16) << 7
            return (mag | sign).to(torch.uint8)

        k8, v8 = codes(), codes()
        ks = torch.rand(shape[:3], generator=gen, device="cuda") * 0.01 + 0.001
        vs = torch.rand(shape[:3], generator=gen, device="cuda") * 0.01 + 0.001
        kc, vc, q = dev16(w.k_cache), dev16(w.v_cache), dev16(w.q)
        out = torch.empty_like(q)
        tables, lens = torch.from_numpy(w.block_tables).cuda(), torch.from_numpy(w.context_lens).cuda()
        part = args.partition
        mctx = w.max_blocks_per_seq * sp.block_size
        ws = torch.empty(max(1, pkv.pkv_decode_workspace_bytes(sp.num_seqs, sp.num_q_heads, sp.num_kv_heads,
                                                                sp.head_dim, mctx, part)),
                         dtype=torch.uint8, device="cuda")
        calls = {
            "e4m3": lambda: pkv.pkv_decode_attention_e4m3(q, k8, ks, v8, vs, tables, lens, w.scale, out, ws, part),
            "16bit": lambda: pkv.pkv_decode_attention(q, kc, vc, tables, lens, w.scale, out, ws, part),
        }
        ms = {}
        for name, call in calls.items():
            for _ in range(args.warmup):
                call()
            t0, t1 = ev(), ev()
            t0.record()
            for _ in range(args.steps):
                call()
            t1.record()
            torch.cuda.synchronize()
            assert pkv.pkv_get_last_error() == pkv.PKV_OK
            ms[name] = t0.elapsed_time(t1) / args.steps
        nb = algorithmic_bytes(w)
        ctx = int(w.context_lens.astype(np.int64).sum())
        kv8 = ctx * 2 * sp.num_kv_heads * (sp.head_dim + 4)
        bytes8 = kv8 + nb["qo"] + nb["tables"] + nb["lens"]
        peak = load_peaks()
        gbs8 = bytes8 / (ms["e4m3"] * 1e-3) / 1e9
        return {"row": "fp8_kv", "metric": "E4M3 paged decode HBM GB/s (algorithmic bytes / kernel time)",
                "value": round(gbs8, 1), "unit": "GB/s", "us_per_launch": round(ms["e4m3"] * 1e3, 2),
                "us_per_launch_16bit": round(ms["16bit"] * 1e3, 2),
                "speedup_vs_16bit": round(ms["16bit"] / ms["e4m3"], 3),
                "gbs_16bit": round(nb["total"] / (ms["16bit"] * 1e-3) / 1e9, 1),
                "peak": peak["hbm_gbs"], "frac": round(gbs8 / peak["hbm_gbs"], 4),
                "algorithmic_bytes": bytes8, "steps": args.steps, "warmup": args.warmup,
                "config": {"workload": sp.name, "partition": part, "l2": "working sets > L2 (no flush)",
                           "kv": "E4M3 codes + fp32 scale per (slot, head) row",
                           "q_out": workloads.DTYPE_NAMES[sp.dtype]}}
    raise SystemExit(f"unknown row {args.row}")


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--partition", type=int, default=None,
                    help="partition tokens: 0 auto (default), -1 none, P > 0 fixed P-token partitions")
    ap.add_argument("--flush-l2", action="store_true")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--row", default=None, choices=["cow", "prefill", "sched", "fp8"],
                    help="measure a row next to the hot path instead (one JSON line tagged 'row')")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end pass (profiling runs)")
    ap.add_argument("--no-extra-workloads", action="store_true",
                    help="default workload only (else the 70B, continuous-batching and long-context "
                         "workloads are measured after it and reported under 'workloads')")
    ap.add_argument("--unfused", action="store_true",
                    help="step = pkv_append + pkv_decode_attention (default: pkv_append_decode_attention)")
    ap.add_argument("--chunks-only", action="store_true",
                    help="--row prefill: time only the two prefill chunks (a small case for profiling)")
    ap.add_argument("--cascade", action="store_true",
                    help="workloads with shared prefixes: the shared-prefix call instead of the plain decode step")
    ap.add_argument("--seqs", type=int, default=None,
                    help="run the workload with its first N sequences only (small profiling cases)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.partition is None:
        import workloads

        args.partition = workloads.CONFIGS[args.workload].partition_tokens or 0
    return args


# measured after the headline in the default run (same process, same ranks):
# the two configurations the bandwidth target names and the long-context split
EXTRA_WORKLOADS = ("llama70b_gqa", "cb_mixed", "long_split")


def workload_summary(r: dict) -> dict:
    """The figures of one extra workload's run kept in the headline line."""
    keep = {k: r[k] for k in ("value", "unit", "ms_per_step", "tokens_per_s_per_layer",
                              "algorithmic_bytes_per_step", "unique_bytes_per_step", "dtype", "clocks")}
    keep["config"] = {k: r["config"][k] for k in ("workload", "description", "partition", "step_call")}
    keep["roofline"] = {k: r["roofline"][k] for k in ("kernel", "achieved", "peak", "unit", "frac", "frac_unique",
                                                      "traffic", "us_per_launch")}
    if r.get("e2e"):
        keep["e2e"] = {k: r["e2e"][k] for k in ("value", "unit", "ms_per_step")}
    return keep


def relaunch_per_gpu(argv, n: int) -> int:
    """Run this script once per GPU (torch.distributed.run, one node,
    rendezvous on 127.0.0.1) and return the launcher's exit status."""
    import socket

    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]
    proc = subprocess.Popen(cmd, start_new_session=True)
    try:
        return proc.wait(timeout=3600)
    except subprocess.TimeoutExpired:
        os.killpg(proc.pid, 9)
        proc.wait()
        return 124


def main(argv=None):
    argv = list(sys.argv[1:] if argv is None else argv)
    args = parse_args(argv)
    rank, world, local = dist_env()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ and not args.row:
        # `bench.py --gpus N` outside a launcher: one process per GPU
        return relaunch_per_gpu(argv, args.gpus)
    if args.row:
        if rank == 0:
            print(json.dumps(run_row(args)), flush=True)
        return 0
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, rank, world)), flush=True)
        return 0
    if world > 1:
        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        result = run_gpu(args, rank, world, local)
        if not args.no_extra_workloads and args.workload == DEFAULT_WORKLOAD and args.seqs is None:
            import copy

            import torch
            import workloads

            subs = {}
            for name in EXTRA_WORKLOADS + ("cb_mixed_shared_prefix",):
                a2 = copy.copy(args)
                a2.workload = "cb_mixed" if name == "cb_mixed_shared_prefix" else name
                a2.cascade = name == "cb_mixed_shared_prefix"
                a2.partition = workloads.CONFIGS[a2.workload].partition_tokens or 0
                a2.no_cpu_baseline = True
                subs[name] = workload_summary(run_gpu(a2, rank, world, local))
                torch.cuda.empty_cache()
            result["workloads"] = subs
        if rank == 0:
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
