"""Benchmark of the paged decode step on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl reference] [--no-extras]

Step = one pass of the whole hot path over one batch: copy-on-write block
copies (when the batch has shared partial blocks), the cache write of each
sequence's new token through its slot, and the decode (plus the partition
reduce) over every token.  ``value`` times that step on the device with every
input already in HBM; ``e2e`` times the same step through the public Python
API including, every step, the host block-manager append (one token per
sequence), the table build, the host->device copies of q / new K,V / slots /
tables / lengths from pinned memory and the device->host copy of the output.

Metric: algorithmic KV bytes the decode reads (sum over sequences of
context_len * num_kv_heads * head_dim * 2 bytes * 2 for K and V) per second;
seq*layers/s is reported beside it.  Multi-GPU: one process per GPU, each an
independent replica of the batch (the path has no exchange step), timed
between barriers, max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("paged decode KV GB/s and % of B200 HBM peak; "
          "seq·layers/s at 1 GPU")
SPEC_HBM_GBS = 8000.0          # the spec figure the target is quoted against
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--workload", default="llama3_70b_gqa8")
    p.add_argument("--impl", default="native", choices=["native", "reference"])
    p.add_argument("--kernel", default="auto")
    p.add_argument("--partition-size", type=int, default=-1)
    p.add_argument("--no-extras", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-spinup", action="store_true",
                   help="skip the 1 s untimed clock spin-up (profiling)")
    p.add_argument("--extras-only", action="store_true",
                   help="time only the side measurements (prefill, prefix "
                        "cache, swap) and print them (tuning and profiling)")
    p.add_argument("--extra", default="all",
                   choices=["all", "prefill", "prefix_cache", "swap",
                            "spec_verify"],
                   help="with --extras-only: run just this side measurement "
                        "(small profiling captures)")
    return p.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing (timing only; the data path has no collective)

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "native" else "gloo"
        if backend == "nccl":
            import torch
            torch.cuda.set_device(local)
        dist.init_process_group(backend,
                                timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64,
                     device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index),
                 f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), f[5], f[6], f[7], f[8]))
            except ValueError:
                continue
        if not rows:
            return None
        sm = [r[0] for r in rows]
        load = [r[0] for r in rows if r[0] > 0.5 * r[1]] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if r[2 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(load)), "sm_max_mhz": rows[0][1],
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# native arm

def measured_hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def decode_source_hash() -> str:
    """Hash of the decode kernel's code (decode.cu, device_utils.cuh and
    order.cuh with comments and blank space removed, so a comment edit
    keeps a capture current and any code change makes it stale)."""
    h = hashlib.sha256()
    for name in ("decode.cu", "device_utils.cuh", "order.cuh"):
        with open(os.path.join(ROOT, "paged_kv_cache_383_b200", "csrc",
                               name)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per decode launch from the committed ncu summary, if it was
    taken on the current decode source (else None)."""
    path = os.path.join(ROOT, "profiles", f"decode_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_hash = re.search(r"source_hash:\s*([0-9a-f]+)", text)
    m_tr = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not (m_hash and m_tr) or m_hash.group(1) != decode_source_hash():
        return None
    return float(m_tr.group(1))


def kv_bytes(lengths, w) -> int:
    return int(np.sum(lengths)) * w.num_kv_heads * w.head_dim * 2 * 2


def make_timer(stream, steps, flush_buf):
    """timed(fn) -> total ms of ``steps`` calls of fn on ``stream``, CUDA
    events on that stream.  With ``flush_buf`` (data below twice the L2
    size) a write of that buffer flushes L2 before each call, outside the
    per-call events; otherwise the calls run back to back between two
    events (an event between the kernels would break their
    programmatic-launch overlap)."""
    import torch

    def timed(fn):
        if flush_buf is None:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(steps):
                fn()
            e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1)
        evs = [(torch.cuda.Event(enable_timing=True),
                torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        for e0, e1 in evs:
            flush_buf.fill_(1)
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize()
        return sum(e0.elapsed_time(e1) for e0, e1 in evs)
    return timed


def run_native(args, rank, world, local):
    import torch
    import paged_kv_cache_383_b200 as pkv
    from paged_kv_cache_383_b200 import flow
    from paged_kv_cache_383_b200 import workloads as wl

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = wl.WORKLOADS[args.workload]
    ps = w.partition_size if args.partition_size < 0 else args.partition_size

    # CPU baseline inputs are gathered later from the same device tensors;
    # start the oracle pool before any GPU work (spawn context).
    pool = None
    want_cpu = (rank == 0 and world == 1 and not args.no_cpu_baseline)
    if want_cpu:
        pool = start_oracle_pool()

    spec = setup_prefix(w, dev, pkv, flow, wl) if w.lengths == "prefix" \
        else setup_paged(w, dev, wl)
    inp = spec.inp
    bt, cl, slots, pairs = spec.bt, spec.cl, spec.slots, spec.pairs
    out = torch.empty_like(inp.q)
    max_ctx = int(inp.lengths.max())
    desc = pkv.make_desc(inp.q, inp.k_cache, bt, partition_size=ps,
                         max_context_len=max_ctx, kernel=args.kernel)
    ws_bytes = pkv.pa_decode_workspace_bytes(desc)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    step_bytes = kv_bytes(inp.lengths, w)

    def writes():
        # on the current stream (the timing stream, or a graph's capture
        # stream)
        if pairs is not None:
            pkv.pa_copy_blocks(inp.k_cache, inp.v_cache, pairs, dev_err=err)
        pkv.pa_cache_write(inp.k_cache, inp.v_cache, spec.write_k,
                           spec.write_v, slots, dev_err=err)

    def step():
        writes()
        pkv.pa_decode(out, inp.q, inp.k_cache, inp.v_cache, bt, cl,
                      w.softmax_scale, desc=desc, workspace=ws, dev_err=err)

    clocks = ClockSampler(local)
    t_spin = time.time()
    while not args.no_spinup and time.time() - t_spin < 1.0:
        # bring clocks up (untimed)
        step()
        torch.cuda.synchronize()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # K/V a step reads at least once; below twice the L2 size the data would
    # stay cached between steps, so L2 is flushed (a 256 MB write) between
    # timed steps and each step is timed on its own.
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    unique_bytes = spec.info.get("unique_kv_bytes_per_step", step_bytes)
    flush = unique_bytes < 2 * l2_bytes
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev) \
        if flush else None

    timed = make_timer(stream, args.steps, flush_buf)

    # Timed region: exactly K steps.
    launches0 = pkv.pa_launch_count()
    barrier(world)
    torch.cuda.synchronize()
    ms_local = timed(step)
    barrier(world)
    launches = pkv.pa_launch_count() - launches0
    ms_total = max_over_ranks(ms_local, world)
    # The dominant kernel's launch duration: K pa_decode calls on the same
    # inputs, timed the same way on the same stream.
    dec_ms = max_over_ranks(timed(lambda: pkv.pa_decode(
        out, inp.q, inp.k_cache, inp.v_cache, bt, cl, w.softmax_scale,
        desc=desc, workspace=ws, dev_err=err, stream=stream)), world) \
        / args.steps
    clk = clocks.stop()
    if err.item() != 0:
        raise RuntimeError(f"device error flag {err.item()} during bench")

    ms_step = ms_total / args.steps
    value = world * step_bytes / (ms_step * 1e-3) / 1e9
    peak, peak_kind = measured_hbm_peak()
    achieved = step_bytes / (dec_ms * 1e-3) / 1e9
    res = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bfloat16" else "fp16",
        "data": "synthetic (seeded N(0,1) q/K/V, shuffled physical blocks)",
        "seq_layers_per_s": round(world * w.num_seqs / (ms_step * 1e-3), 1),
        "pct_of_spec_8000": round(100 * value / world / SPEC_HBM_GBS, 2),
        "pct_of_measured_copy": round(100 * value / world / peak, 2),
        "config": {
            "workload": w.name,
            "num_seqs": w.num_seqs, "num_q_heads": w.num_q_heads,
            "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim,
            "block_size": w.block_size, "total_tokens": int(inp.lengths.sum()),
            "max_context_len": max_ctx,
            "partition_size": pkv.pa_decode_partition_size(desc),
            "kernel": args.kernel,
            "kv_bytes_per_step": step_bytes,
            **spec.info,
            "l2": (f"L2 flushed between timed steps (256 MB write outside "
                   f"the per-step events): {unique_bytes / 1e6:.1f} MB of "
                   f"K/V per step" if flush else
                   f"inputs larger than L2 (no flush): {unique_bytes / 1e9:.2f}"
                   f" GB of distinct K/V per step"),
            "parallelism": f"{world} independent replicas" if world > 1
                           else "1 GPU",
        },
        "roofline": {
            "bound": "hbm",
            "kernel": "pa_decode (decode + partition reduce)",
            "achieved": round(achieved, 2),
            "peak": peak,
            "peak_kind": f"{peak_kind} HBM copy bandwidth",
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "frac_of_spec_8000": round(achieved / SPEC_HBM_GBS, 4),
            "traffic": profiled_traffic(w.name),
            "decode_ms": round(dec_ms, 5),
            "decode_ms_how": ("K pa_decode calls on the step's inputs, CUDA "
                              "events on the launch stream" +
                              (", L2 flushed before each" if flush else
                               ", back to back")),
        },
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_extras:
        res["extras"] = extras(args, w, inp, dev, pkv, bt, cl)
        # The same step captured once in a CUDA graph and replayed: what
        # the host's launch calls cost per step.
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        g_ms = timed(graph.replay) / args.steps
        res["extras"]["cuda_graph"] = {
            "step_ms_eager": round(ms_step, 5),
            "step_ms_graph": round(g_ms, 5),
            "note": "one captured step (cache write, prep, decode) replayed "
                    "K times, timed as the main step"}
        del graph
        probe = res["extras"].get("read_probe_gbs")
        if probe:
            res["roofline"]["read_probe_gbs"] = probe
            res["roofline"]["frac_of_read_probe"] = round(achieved / probe, 4)
        res["extras"]["configs"] = config_block(args, pkv, flow, wl, dev,
                                                probe)
    if not args.no_e2e:
        if w.lengths == "prefix":
            res["e2e"] = run_e2e_fixed(args, w, spec, dev, pkv, world, ps)
        else:
            res["e2e"] = run_e2e(args, w, inp, dev, pkv, flow, world, rank,
                                 ps)
    if flush and "e2e" in res:
        res["e2e"]["l2"] = (f"the {unique_bytes / 1e6:.1f} MB of K/V stay in "
                            f"L2 between end-to-end steps (not flushed there)")
    if want_cpu and w.lengths != "prefix":
        res["cpu_baseline"] = cpu_baseline(pool, inp, w, dev)
    if pool is not None:
        pool.close()
    return res


# The serving mixes besides the headline one (batch 256, block 16): each is
# timed like the headline line, into extras["configs"].
CONFIG_WORKLOADS = ("tiny_mha_d64", "llama3_8b_gqa4", "llama3_70b_gqa8_bs32",
                    "shared_prefix_cow", "long_context_split")


def config_block(args, pkv, flow, wl, dev, probe_gbs):
    """Per configuration: the step (copy-on-write copies and cache write
    where the mix has them, then the decode) and the decode alone, each over
    K calls timed with CUDA events on the launch stream exactly like the
    headline line (L2 flushed between calls when the distinct K/V is below
    twice the L2 size), with the clocks sampled during the timed calls.
    GB/s are algorithmic K/V bytes (logical bytes for the shared-prefix mix:
    its prefix is read once per sequence and stays in L2)."""
    import torch
    peak, peak_kind = measured_hbm_peak()
    stream = torch.cuda.current_stream(dev)
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    steps = max(args.steps, 10)
    res = {}
    for name in CONFIG_WORKLOADS:
        w = wl.WORKLOADS[name]
        spec = setup_prefix(w, dev, pkv, flow, wl) if w.lengths == "prefix" \
            else setup_paged(w, dev, wl)
        inp = spec.inp
        out = torch.empty_like(inp.q)
        desc = pkv.make_desc(inp.q, inp.k_cache, spec.bt,
                             partition_size=w.partition_size,
                             max_context_len=int(inp.lengths.max()))
        ws = torch.empty(max(pkv.pa_decode_workspace_bytes(desc), 16),
                         dtype=torch.uint8, device=dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)

        def decode():
            pkv.pa_decode(out, inp.q, inp.k_cache, inp.v_cache, spec.bt,
                          spec.cl, w.softmax_scale, desc=desc, workspace=ws,
                          dev_err=err)

        def step():
            if spec.pairs is not None:
                pkv.pa_copy_blocks(inp.k_cache, inp.v_cache, spec.pairs,
                                   dev_err=err)
            pkv.pa_cache_write(inp.k_cache, inp.v_cache, spec.write_k,
                               spec.write_v, spec.slots, dev_err=err)
            decode()

        for _ in range(5):
            step()
        torch.cuda.synchronize()
        step_bytes = kv_bytes(inp.lengths, w)
        unique = spec.info.get("unique_kv_bytes_per_step", step_bytes)
        flush = unique < 2 * l2_bytes
        flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev) \
            if flush else None
        timed = make_timer(stream, steps, flush_buf)
        # the timed calls last milliseconds: the clocks are sampled over an
        # untimed 0.5 s run of the same step just before them, and the
        # timed calls themselves
        clocks = ClockSampler(dev.index or 0)
        t0 = time.time()
        while time.time() - t0 < 0.5:
            step()
            torch.cuda.synchronize()
        ms_step = timed(step) / steps
        ms_dec = timed(decode) / steps
        clk = clocks.stop()
        if err.item() != 0:
            raise RuntimeError(f"{name}: device error flag {err.item()}")
        dec_gbs = step_bytes / (ms_dec * 1e-3) / 1e9
        entry = {
            "step": spec.info["step"],
            "seqs": w.num_seqs, "heads_q_kv": [w.num_q_heads,
                                               w.num_kv_heads],
            "head_dim": w.head_dim, "block_size": w.block_size,
            "dtype": w.dtype, "tokens": int(inp.lengths.sum()),
            "kv_bytes": step_bytes,
            "partition_size": pkv.pa_decode_partition_size(desc),
            "partition_spec": w.partition_size or "auto",
            "ms_step": round(ms_step, 5), "ms_decode": round(ms_dec, 5),
            "step_gbs": round(step_bytes / (ms_step * 1e-3) / 1e9, 1),
            "decode_gbs": round(dec_gbs, 1),
            "seq_layers_per_s": round(w.num_seqs / (ms_dec * 1e-3), 1),
            "frac_of_copy_peak": round(dec_gbs / peak, 4),
            "copy_peak": f"{peak} GB/s ({peak_kind})",
            "frac_of_read_probe": round(dec_gbs / probe_gbs, 4)
            if probe_gbs else None,
            "frac_of_spec_8000": round(dec_gbs / SPEC_HBM_GBS, 4),
            "l2": "flushed between calls" if flush else "inputs larger than "
                                                        "L2, back to back",
            "calls": steps, "clocks": clk,
            "clocks_how": "nvidia-smi every 100 ms over a 0.5 s untimed run "
                          "of the step and the timed calls"}
        if w.lengths == "prefix":
            entry["note"] = spec.info["note"]
        res[name] = entry
        del spec, inp, out, ws, flush_buf
        torch.cuda.empty_cache()
    return res


class StepSpec:
    """Device inputs of one step: the decode batch plus the writes that
    precede it (new tokens' K/V and their slots, copy-on-write pairs)."""

    def __init__(self, inp, bt, cl, write_k, write_v, slots, pairs, info):
        self.inp, self.bt, self.cl = inp, bt, cl
        self.write_k, self.write_v, self.slots = write_k, write_v, slots
        self.pairs, self.info = pairs, info


def setup_paged(w, dev, wl):
    """Shuffled-pool batch; each step rewrites every sequence's newest token
    (position L-1) through its slot, then decodes over all L tokens."""
    import torch
    inp = wl.make_paged(w, device=dev)
    if inp.k_new is None:
        g = torch.Generator(device=dev)
        g.manual_seed(w.seed + 7)
        shp = (w.num_seqs, w.num_kv_heads, w.head_dim)
        inp.k_new = torch.randn(shp, generator=g, device=dev).to(inp.q.dtype)
        inp.v_new = torch.randn(shp, generator=g, device=dev).to(inp.q.dtype)
        pos = inp.lengths - 1
        inp.new_slots = (inp.block_tables[np.arange(w.num_seqs),
                                          pos // w.block_size]
                         .astype(np.int64) * w.block_size
                         + pos % w.block_size)
    bt = torch.from_numpy(inp.block_tables).to(dev)
    cl = torch.from_numpy(inp.lengths.astype(np.int32)).to(dev)
    slots = torch.from_numpy(inp.new_slots).to(dev)
    return StepSpec(inp, bt, cl, inp.k_new, inp.v_new, slots, None,
                    {"step": "cache write of 1 token/seq + decode"})


def setup_prefix(w, dev, pkv, flow, wl):
    """Shared-prefix mix built through the block manager: sequence 0 takes
    the prefix, the others fork from it (reference count = batch), then one
    append per sequence gives the suffix slots and the copy-on-write pairs.
    Each step copies the shared partial block for every writer but the last,
    writes all suffix tokens, and decodes (idempotent: the same copies and
    writes every step)."""
    import torch
    pin = wl.make_prefix(w, device=dev)
    shape = (pin.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed + 1)
    dt = wl.torch_dtype(w.dtype)
    kc = torch.randn(shape, generator=g, device=dev).to(dt)
    vc = torch.randn(shape, generator=g, device=dev).to(dt)
    bm = pkv.BlockManager(pin.num_blocks, w.block_size,
                          free_order=pin.free_order)
    flow.shared_prefix_batch(bm, kc, vc, pin.prefix_k, pin.prefix_v,
                             w.num_seqs)
    ids = list(range(w.num_seqs))
    slots, pairs = bm.append_batch(ids, pin.suffix_lens)
    max_blocks = int(wl.blocks_needed(pin.lengths, w.block_size).max())
    table, lens = bm.block_table(ids, max_blocks)
    bm.close()
    inp = wl.PagedInputs(w, pin.lengths, table, pin.num_blocks, pin.q, kc, vc)
    unique = (w.prefix_len + int(pin.suffix_lens.sum())) * \
        w.num_kv_heads * w.head_dim * 4
    info = {"step": f"{len(pairs)} copy-on-write block copies + cache write "
                    f"of {int(pin.suffix_lens.sum())} suffix tokens + decode",
            "cow_pairs": int(len(pairs)),
            "unique_kv_bytes_per_step": int(unique),
            "note": "KV bytes are logical: the shared prefix is read once per "
                    "sequence and stays L2-resident"}
    return StepSpec(inp, torch.from_numpy(table).to(dev),
                    torch.from_numpy(lens).to(dev), pin.suffix_k, pin.suffix_v,
                    torch.from_numpy(slots).to(dev),
                    torch.from_numpy(pairs).to(dev) if len(pairs) else None,
                    info)


def run_e2e_fixed(args, w, spec, dev, pkv, world, ps):
    """End-to-end step of the shared-prefix mix through the public API: the
    step's inputs (q, suffix K/V, slots, copy pairs, tables, lengths) go
    host->device from pinned memory, then copies, writes and decode, then
    the output comes back device->host; one sync per step."""
    import torch
    inp = spec.inp
    host = {k: t.cpu().pin_memory() for k, t in (
        ("q", inp.q), ("k", spec.write_k), ("v", spec.write_v),
        ("slots", spec.slots), ("bt", spec.bt), ("cl", spec.cl))}
    if spec.pairs is not None:
        host["pairs"] = spec.pairs.cpu().pin_memory()
    devt = {k: torch.empty_like(t, device=dev) for k, t in host.items()}
    hout = torch.empty(inp.q.shape, dtype=inp.q.dtype).pin_memory()
    dout = torch.empty_like(inp.q)
    stream = torch.cuda.current_stream(dev)
    max_ctx = int(inp.lengths.max())

    def one():
        for k in host:
            devt[k].copy_(host[k], non_blocking=True)
        if "pairs" in devt:
            pkv.pa_copy_blocks(inp.k_cache, inp.v_cache, devt["pairs"])
        pkv.pa_cache_write(inp.k_cache, inp.v_cache, devt["k"], devt["v"],
                           devt["slots"])
        pkv.pa_decode(dout, devt["q"], inp.k_cache, inp.v_cache, devt["bt"],
                      devt["cl"], w.softmax_scale, partition_size=ps,
                      max_context_len=max_ctx)
        hout.copy_(dout, non_blocking=True)
        stream.synchronize()

    for _ in range(args.warmup):
        one()
    barrier(world)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        one()
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(a.elapsed_time(b), world)
    return {"value": round(world * args.steps * kv_bytes(inp.lengths, w) /
                           (ms * 1e-3) / 1e9, 2),
            "unit": "GB/s",
            "h2d_bytes_per_step": int(sum(t.nbytes for t in host.values())),
            "d2h_bytes_per_step": int(hout.nbytes),
            "ms_per_step": round(ms / args.steps, 4),
            "includes": "pinned H2D of the step's inputs, copy-on-write "
                        "copies, cache write, decode, D2H of the output, one "
                        "sync per step"}


def extras(args, w, inp, dev, pkv, bt, cl):
    """Side measurements on the same inputs: the SIMT kernel, a partition
    size sweep, the separate reduce kernel, and the read bandwidth of the
    library's streaming read probe over a 4 GiB buffer (the achievable read
    roofline) beside a torch reduction."""
    import torch
    out = {}
    o = torch.empty_like(inp.q)
    max_ctx = int(inp.lengths.max())

    def time_decode(kernel, ps, reduce="auto"):
        desc = pkv.make_desc(inp.q, inp.k_cache, bt, partition_size=ps,
                             max_context_len=max_ctx, kernel=kernel,
                             reduce=reduce)
        ws = torch.empty(max(pkv.pa_decode_workspace_bytes(desc), 16),
                         dtype=torch.uint8, device=dev)
        for _ in range(3):
            pkv.pa_decode(o, inp.q, inp.k_cache, inp.v_cache, bt, cl,
                          w.softmax_scale, desc=desc, workspace=ws)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(20):
            pkv.pa_decode(o, inp.q, inp.k_cache, inp.v_cache, bt, cl,
                          w.softmax_scale, desc=desc, workspace=ws)
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / 20
        return round(kv_bytes(inp.lengths, w) / (ms * 1e-3) / 1e9, 1)

    out["decode_gbs_simt"] = time_decode("simt", w.partition_size)
    out["decode_gbs_mma"] = time_decode("mma", w.partition_size)
    out["decode_gbs_mma_reduce_kernel"] = time_decode("mma", w.partition_size,
                                                      "kernel")
    for ps in (0, 256, 512, 1024, 2048):
        out[f"decode_gbs_mma_ps{ps}"] = time_decode("mma", ps)
    x = torch.empty(1 << 30, dtype=torch.float32, device=dev).fill_(1.0)
    sink = torch.zeros(4, dtype=torch.int32, device=dev)
    for _ in range(3):
        pkv.pa_read_probe(x, sink)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(10):
        pkv.pa_read_probe(x, sink)
    b.record()
    torch.cuda.synchronize()
    out["read_probe_gbs"] = round(4 * (1 << 30) / (a.elapsed_time(b) / 10 *
                                                    1e-3) / 1e9, 1)
    for _ in range(3):
        x.sum()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(10):
        x.sum()
    b.record()
    torch.cuda.synchronize()
    out["torch_sum_read_gbs"] = round(4 * (1 << 30) / (a.elapsed_time(b) /
                                                        10 * 1e-3) / 1e9, 1)
    del x
    out["identity_vs_shuffled"] = identity_vs_shuffled(pkv, w, inp, dev)
    from paged_kv_cache_383_b200 import workloads as wl
    out["prefill"] = [time_prefill(pkv, wl, n, c, dev, sustain_s=2.0)
                      for n, c in PREFILL_CASES]
    out["prefix_cache"] = prefix_cache_measure(pkv, dev)
    out["swap"] = swap_measure(pkv, dev)
    out["spec_verify"] = spec_verify_measure(pkv, dev)
    out["spec_verify_8"] = spec_verify_measure(pkv, dev, drafts=8)
    return out


def identity_vs_shuffled(pkv, w, inp, dev, repeats=12, calls=10):
    """The same decode over the shuffled pool and over a copy laid out so
    every sequence's blocks are consecutive (identity tables): the whole
    batch, and batch 1 (its longest sequence; L2 flushed before each call,
    the data being smaller than L2).  The two arms alternate, ``repeats``
    times, each time ``calls`` calls; each arm reports the median and the
    min..max of its repeats (GB/s of K/V read), so a difference of about a
    percent can be told from run-to-run noise."""
    import torch
    B = inp.block_tables.shape[0]
    rows = [inp.block_tables[b][inp.block_tables[b] >= 0] for b in range(B)]
    order = torch.from_numpy(np.concatenate(rows).astype(np.int64)).to(dev)
    kc = inp.k_cache[order].contiguous()
    vc = inp.v_cache[order].contiguous()
    ident = np.full_like(inp.block_tables, -1)
    base = 0
    for b, r in enumerate(rows):
        ident[b, :len(r)] = np.arange(base, base + len(r))
        base += len(r)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def prepare(seqs, tables, k, v):
        q = inp.q[seqs].contiguous()
        bt = torch.from_numpy(tables[seqs]).to(dev)
        lens = inp.lengths[seqs]
        cl = torch.from_numpy(lens.astype(np.int32)).to(dev)
        o = torch.empty_like(q)
        desc = pkv.make_desc(q, k, bt, max_context_len=int(lens.max()))
        ws = torch.empty(pkv.pa_decode_workspace_bytes(desc),
                         dtype=torch.uint8, device=dev)
        f = lambda: pkv.pa_decode(o, q, k, v, bt, cl, w.softmax_scale,
                                  desc=desc, workspace=ws)
        for _ in range(3):
            f()
        return f, kv_bytes(lens, w)

    def once(f, nbytes, flush):
        total = 0.0
        for _ in range(calls):
            if flush:
                flush_buf.fill_(1)
            a = torch.cuda.Event(enable_timing=True)
            b_ = torch.cuda.Event(enable_timing=True)
            a.record()
            f()
            b_.record()
            torch.cuda.synchronize()
            total += a.elapsed_time(b_)
        return nbytes / (total / calls * 1e-3) / 1e9

    def compare(seqs, flush):
        arms = {"shuffled": prepare(seqs, inp.block_tables, inp.k_cache,
                                    inp.v_cache),
                "identity": prepare(seqs, ident, kc, vc)}
        got = {k: [] for k in arms}
        for r in range(repeats):
            for k in (("shuffled", "identity") if r % 2 == 0
                      else ("identity", "shuffled")):
                got[k].append(once(*arms[k], flush))
        out = {}
        for k, v in got.items():
            out[f"{k}_gbs_median"] = round(float(np.median(v)), 1)
            out[f"{k}_gbs_range"] = [round(min(v), 1), round(max(v), 1)]
        lo_i, hi_i = out["identity_gbs_range"]
        lo_s, hi_s = out["shuffled_gbs_range"]
        out["ranges_overlap"] = bool(lo_i <= hi_s and lo_s <= hi_i)
        return out

    allb = np.arange(B)
    one = np.array([int(np.argmax(inp.lengths))])
    res = {"repeats": repeats, "calls_per_repeat": calls,
           "batch": compare(allb, False),
           "batch1_tokens": int(inp.lengths[one[0]]),
           "batch1": compare(one, True)}
    del kc, vc
    return res


def measured_bf16_peak(sustained: bool = False):
    """The measured bf16 GEMM peak: the burst figure (a kernel timed alone),
    or the sustained one (seconds of back-to-back work under the power cap).
    """
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)[key]), "measured"
    except (OSError, KeyError, ValueError):
        return (FALLBACK_BF16_TFLOPS_SUSTAINED if sustained
                else FALLBACK_BF16_TFLOPS), "fallback"


def prefill_flops(lengths, q_lens, num_q_heads, head_dim) -> int:
    """Algorithmic FLOPs of causal attention of the new tokens: per query
    head, new token and key it attends to, 2*D for q.k and 2*D for p*v."""
    keys = 0
    for L, n in zip(lengths, q_lens):
        L, n = int(L), int(n)
        keys += n * (L - n) + n * (n + 1) // 2
    return 4 * head_dim * num_q_heads * keys


PREFILL_CASES = (
    # (workload, new tokens per sequence or None for the whole prompt)
    ("chunked_prefill_gqa8", 512),
    ("prompt_prefill_gqa8", None),
)


def time_prefill(pkv, wl, name, chunk, dev, iters=10, sustain_s=0.0):
    """pa_prefill on a prefill workload: CUDA events around ``iters``
    back-to-back launches on the launch stream (inputs > L2), for each
    precision of P in P . V (the default "auto" adds P's residual only in
    the tiles that need it; "split" in every tile; "single" never).  With
    ``sustain_s`` > 0 the default precision then runs back to back for that
    long, rounds of ``iters`` calls timed by CUDA events, with the clocks
    sampled: the median of the second half of the rounds is the sustained
    rate, against the sustained GEMM peak."""
    import torch
    w = wl.WORKLOADS[name]
    rng_lens = wl.make_paged(w, values=False).lengths
    q_lens = rng_lens if chunk is None else np.minimum(rng_lens, chunk)
    pin = wl.make_prefill(w, q_lens, device=dev)
    inp = pin.paged
    out = torch.empty_like(pin.q)
    bt = torch.from_numpy(inp.block_tables).to(dev)
    cl = torch.from_numpy(inp.lengths.astype(np.int32)).to(dev)
    qs = torch.from_numpy(pin.query_start).to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    kw = dict(max_q_len=int(pin.q_lens.max()),
              max_context_len=int(inp.lengths.max()), dev_err=err,
              workspace=torch.empty(
                  pkv.pa_prefill_workspace_bytes(pin.q, inp.k_cache, bt),
                  dtype=torch.uint8, device=dev))
    def run(pv):
        for _ in range(3):
            pkv.pa_prefill(out, pin.q, inp.k_cache, inp.v_cache, bt, cl, qs,
                           w.softmax_scale, pv=pv, **kw)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(iters):
            pkv.pa_prefill(out, pin.q, inp.k_cache, inp.v_cache, bt, cl, qs,
                           w.softmax_scale, pv=pv, **kw)
        b.record()
        torch.cuda.synchronize()
        if err.item():
            raise RuntimeError(f"pa_prefill device error {err.item()}")
        return a.elapsed_time(b) / iters

    flops = prefill_flops(inp.lengths, pin.q_lens, w.num_q_heads, w.head_dim)
    peak, kind = measured_bf16_peak()
    ms = {pv: run(pv) for pv in ("auto", "split", "single")}
    tf = {pv: flops / (t * 1e-3) / 1e12 for pv, t in ms.items()}
    sustained = None
    if sustain_s > 0:
        clocks = ClockSampler(dev.index or 0)
        rounds = []
        t_end = time.time() + sustain_s
        while time.time() < t_end:
            rounds.append(flops / (run("auto") * 1e-3) / 1e12)
        clk = clocks.stop()
        speak, skind = measured_bf16_peak(sustained=True)
        tail = float(np.median(rounds[len(rounds) // 2:]))
        sustained = {"seconds": sustain_s, "rounds": len(rounds),
                     "tflops": round(tail, 1),
                     "tflops_first_round": round(rounds[0], 1),
                     "peak_tflops": speak,
                     "peak_kind": f"{skind} bf16 dense, sustained (cuBLAS "
                                  f"GEMM back to back under the power cap)",
                     "frac": round(tail / speak, 4), "clocks": clk}
    return {"workload": name, "seqs": w.num_seqs,
            "new_tokens": int(pin.q_lens.sum()),
            "context_tokens": int(inp.lengths.sum()),
            "ms": round(ms["auto"], 4), "tflops": round(tf["auto"], 1),
            "peak_tflops": peak,
            "peak_kind": f"{kind} bf16 dense (cuBLAS GEMM)",
            "frac": round(tf["auto"] / peak, 4),
            "pv": "auto (P's residual . V only in tiles where a key may end "
                  "with weight > 1/16)",
            "tflops_pv_split": round(tf["split"], 1),
            "frac_pv_split": round(tf["split"] / peak, 4),
            "tflops_pv_single": round(tf["single"], 1),
            "frac_pv_single": round(tf["single"] / peak, 4),
            "sustained": sustained,
            "note": "algorithmic FLOPs (4 D per query head, new token and "
                    "key attended); with pv=split the tensor cores do 1.5x "
                    "that (P.V twice)"}


def prefix_cache_measure(pkv, dev, requests=128, prompt_len=2048,
                         q_low=64, q_high=512, seed=383009):
    """A shared system prompt: ``requests`` requests of one 2048-token prompt
    plus a question of U[64, 512] tokens (Llama-3-70B heads, block 16,
    bf16).  Host: microseconds per request of match + append + cache insert
    through the C ABI.  GPU: one pa_prefill over the whole batch when every
    request prefills its full prompt, against the suffix-only prefill the
    cache leaves (the tokens of the first request's prompt are computed
    once, in an earlier pass that is not timed).  Also the blocks held."""
    import time
    import torch
    bs, hq, hkv, d = 16, 64, 8, 128
    rng = np.random.default_rng(seed)
    qlens = rng.integers(q_low, q_high + 1, size=requests)
    prompt = np.arange(prompt_len, dtype=np.int32) + 1_000_000
    toks = [np.concatenate([prompt, rng.integers(0, 100_000, size=n)
                            .astype(np.int32)]) for n in qlens]
    need = int(sum(-(-len(t) // bs) for t in toks))
    bm = pkv.BlockManager(need + 64, bs)
    hits = np.zeros(requests, dtype=np.int64)
    t0 = time.perf_counter()
    for r in range(requests):
        bm.add_seq(r)
        hits[r] = bm.match_prefix(r, toks[r])
        bm.append(r, len(toks[r]) - int(hits[r]))
        bm.cache_insert(r, toks[r])
    host_us = (time.perf_counter() - t0) / requests * 1e6
    blocks_cached = need + 64 - bm.num_free()
    max_blocks = max(-(-len(t) // bs) for t in toks)
    table, lens = bm.block_table(list(range(requests)), max_blocks)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    shape = (need + 64, hkv, bs, d)
    kc = torch.randn(shape, generator=g, device=dev).to(torch.bfloat16)
    vc = torch.randn(shape, generator=g, device=dev).to(torch.bfloat16)
    bt = torch.from_numpy(table).to(dev)
    cl = torch.from_numpy(lens).to(dev)
    res = {"requests": requests, "prompt_tokens": prompt_len,
           "question_tokens_mean": float(qlens.mean()),
           "host_us_per_request": round(host_us, 2),
           "blocks_with_cache": int(blocks_cached), "blocks_without": need,
           "matched_tokens_mean": float(hits[1:].mean())}
    for mode, q_lens in (("full", lens.astype(np.int64)),
                         ("cached", lens.astype(np.int64) - hits)):
        qs = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
        q = torch.randn(int(qs[-1]), hq, d, generator=g,
                        device=dev).to(torch.bfloat16)
        out = torch.empty_like(q)
        qsd = torch.from_numpy(qs).to(dev)
        kw = dict(max_q_len=int(q_lens.max()),
                  max_context_len=int(lens.max()),
                  workspace=torch.empty(
                      pkv.pa_prefill_workspace_bytes(q, kc, bt),
                      dtype=torch.uint8, device=dev))
        for _ in range(2):
            pkv.pa_prefill(out, q, kc, vc, bt, cl, qsd, d ** -0.5, **kw)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(5):
            pkv.pa_prefill(out, q, kc, vc, bt, cl, qsd, d ** -0.5, **kw)
        b.record()
        torch.cuda.synchronize()
        res[f"prefill_ms_{mode}"] = round(a.elapsed_time(b) / 5, 3)
        res[f"prefill_tokens_{mode}"] = int(qs[-1])
    res["prefill_speedup"] = round(res["prefill_ms_full"] /
                                   res["prefill_ms_cached"], 2)
    bm.close()
    return res


def swap_measure(pkv, dev, group_size=64, seed=383010):
    """Preempting ``group_size`` of the 256 Llama-3-70B-shaped sequences
    (log-normal lengths, block 16, bf16): block-manager swap-out / swap-in
    (host microseconds) and pa_swap_blocks moving their K/V to a pinned host
    pool and back (GB/s), beside torch's own pinned copy of the same bytes
    in one piece (the host link's copy bandwidth)."""
    import time
    import torch
    from paged_kv_cache_383_b200 import workloads as wl
    w = wl.WORKLOADS["llama3_70b_gqa8"]
    lengths = wl.make_paged(w, values=False).lengths
    bs, hkv, d = w.block_size, w.num_kv_heads, w.head_dim
    need = int(sum(-(-int(L) // bs) for L in lengths))
    nb = need + 64
    bm = pkv.BlockManager(nb, bs)
    for b, L in enumerate(lengths):
        bm.add_seq(b)
        bm.append(b, int(L))
    rng = np.random.default_rng(seed)
    group = sorted(rng.choice(len(lengths), group_size, replace=False)
                   .tolist())
    host_blocks = int(sum(-(-int(lengths[b]) // bs) for b in group))
    bm.set_host_blocks(host_blocks)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    shape = (nb, hkv, bs, d)
    kc = torch.randn(shape, generator=g, device=dev).to(torch.bfloat16)
    vc = torch.randn(shape, generator=g, device=dev).to(torch.bfloat16)
    hk = torch.empty((host_blocks, hkv, bs, d), dtype=torch.bfloat16,
                     pin_memory=True)
    hv = torch.empty_like(hk, pin_memory=True)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    block_bytes = hkv * bs * d * 2 * 2          # K and V
    res = {"group": group_size, "blocks": host_blocks,
           "bytes": host_blocks * block_bytes}
    ev = lambda: torch.cuda.Event(enable_timing=True)
    t_out = t_in = 0.0
    ms_out, ms_in, reps = [], [], 3
    for _ in range(reps):
        t0 = time.perf_counter()
        pairs = bm.swap_out(group)
        t_out += time.perf_counter() - t0
        pd = torch.from_numpy(pairs).to(dev)
        a, b = ev(), ev()
        a.record()
        pkv.pa_swap_blocks(hk, hv, kc, vc, pd, dev_err=err)
        b.record()
        torch.cuda.synchronize()
        ms_out.append(a.elapsed_time(b))
        t0 = time.perf_counter()
        pairs = bm.swap_in(group)
        t_in += time.perf_counter() - t0
        pd = torch.from_numpy(pairs).to(dev)
        a, b = ev(), ev()
        a.record()
        pkv.pa_swap_blocks(kc, vc, hk, hv, pd, dev_err=err)
        b.record()
        torch.cuda.synchronize()
        ms_in.append(a.elapsed_time(b))
    if err.item():
        raise RuntimeError(f"pa_swap_blocks device error {err.item()}")
    gbs = lambda ms: round(res["bytes"] / (ms * 1e-3) / 1e9, 2)
    res["host_us_swap_out"] = round(t_out / reps * 1e6, 1)
    res["host_us_swap_in"] = round(t_in / reps * 1e6, 1)
    res["d2h_ms"] = round(min(ms_out[1:]), 3)
    res["h2d_ms"] = round(min(ms_in[1:]), 3)
    res["d2h_gbs"] = gbs(res["d2h_ms"])
    res["h2d_gbs"] = gbs(res["h2d_ms"])
    # torch's pinned copy of the same number of bytes, one contiguous piece
    n = host_blocks * hkv * bs * d
    dflat = kc.view(-1)[:n]
    hflat = hk.view(-1)
    for direction in ("d2h", "h2d"):
        best = None
        for _ in range(3):
            a, b = ev(), ev()
            a.record()
            for _ in range(2):  # K and V
                if direction == "d2h":
                    hflat.copy_(dflat, non_blocking=True)
                else:
                    dflat.copy_(hflat, non_blocking=True)
            b.record()
            torch.cuda.synchronize()
            ms = a.elapsed_time(b)
            best = ms if best is None else min(best, ms)
        res[f"torch_copy_{direction}_gbs"] = gbs(best)
        res[f"frac_{direction}"] = round(res[f"{direction}_gbs"] /
                                         res[f"torch_copy_{direction}_gbs"], 3)
    bm.close()
    return res


def spec_verify_measure(pkv, dev, drafts=4):
    """Speculative verification on the batch-256 mix (Llama-3-70B heads,
    log-normal lengths, block 16, bf16): every sequence checks ``drafts``
    new tokens in one pa_prefill call.  Reported as GB/s of K/V read (it
    reads every cached token once, like a decode) beside the decode of the
    same batch."""
    import torch
    from paged_kv_cache_383_b200 import workloads as wl
    w = wl.WORKLOADS["llama3_70b_gqa8"]
    lens = wl.make_paged(w, values=False).lengths
    pin = wl.make_prefill(w, np.full(w.num_seqs, drafts), device=dev)
    inp = pin.paged
    bt = torch.from_numpy(inp.block_tables).to(dev)
    cl = torch.from_numpy(inp.lengths.astype(np.int32)).to(dev)
    qs = torch.from_numpy(pin.query_start).to(dev)
    out = torch.empty_like(pin.q)
    kw = dict(max_q_len=drafts, max_context_len=int(lens.max()),
              workspace=torch.empty(
                  pkv.pa_prefill_workspace_bytes(pin.q, inp.k_cache, bt),
                  dtype=torch.uint8, device=dev))

    def time_kernel(kernel, pv="auto"):
        f = lambda: pkv.pa_prefill(out, pin.q, inp.k_cache, inp.v_cache, bt,
                                   cl, qs, w.softmax_scale, kernel=kernel,
                                   pv=pv, **kw)
        for _ in range(3):
            f()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(20):
            f()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / 20

    ms = time_kernel("auto")
    ms_split = time_kernel("auto", "split")
    ms_single = time_kernel("auto", "single")
    gbs = lambda t: round(kv_bytes(inp.lengths, w) / (t * 1e-3) / 1e9, 1) \
        if t else None
    return {"seqs": w.num_seqs, "drafts": drafts,
            "kv_bytes": kv_bytes(inp.lengths, w), "ms": round(ms, 4),
            "kv_gbs": gbs(ms),
            "tflops": round(prefill_flops(inp.lengths, pin.q_lens,
                                          w.num_q_heads, w.head_dim)
                            / (ms * 1e-3) / 1e12, 1),
            "kernel": "the tile kernel",
            "pv": "auto",
            "kv_gbs_pv_split": gbs(ms_split),
            "kv_gbs_pv_single": gbs(ms_single)}


def run_extras_only(args):
    import torch
    import paged_kv_cache_383_b200 as pkv
    from paged_kv_cache_383_b200 import workloads as wl
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    want = lambda name: args.extra in ("all", name)
    res = {"metric": "side measurements: prefill attention TFLOP/s "
                     "(algorithmic), prefix cache, swap, speculative "
                     "verification"}
    if want("prefill"):
        res["prefill"] = [time_prefill(pkv, wl, n, c, dev,
                                       iters=max(args.steps, 1))
                          for n, c in PREFILL_CASES]
    if want("prefix_cache"):
        res["prefix_cache"] = prefix_cache_measure(pkv, dev)
    if want("swap"):
        res["swap"] = swap_measure(pkv, dev)
    if want("spec_verify"):
        res["spec_verify"] = spec_verify_measure(pkv, dev)
        res["spec_verify_8"] = spec_verify_measure(pkv, dev, drafts=8)
    res["gpu_launches"] = pkv.pa_launch_count()
    return res


def run_e2e(args, w, inp, dev, pkv, flow, world, rank, ps):
    """Same step through the public API with host buffers.  Every step:
    the block manager appends one token to every sequence and rebuilds the
    tables (on the host), the step's inputs (q, the new tokens' K/V, slots,
    tables, lengths) go host->device from pinned memory in one packed copy,
    then cache write and decode, and the output comes back device->host;
    the host waits for each step's output.  Steps are pipelined the way a
    serving loop overlaps them: while the GPU decodes step n, the host
    builds step n+1's inputs and copies them up on a copy stream, and
    earlier steps' outputs come down on another; the host reads step n's
    output while step n+2 is issued (three staging buffers on each side).
    Every step's copies and kernels lie inside the timed region."""
    import torch
    bm = pkv.BlockManager(inp.num_blocks, w.block_size,
                          free_order=_free_order(inp))
    ids = np.arange(w.num_seqs, dtype=np.int64)
    for b in ids:
        bm.add_seq(int(b))
    bm.append_batch(ids, inp.lengths.astype(np.int32) - 1)
    steps = args.steps
    final_lens = inp.lengths + steps + args.warmup + 1
    max_blocks = int(wl_blocks(final_lens, w.block_size).max())
    B = w.num_seqs
    # packed staging layout: (name, bytes, dtype, shape), 256-byte aligned
    parts = [("q", inp.q), ("k", inp.k_new), ("v", inp.v_new)]
    fields, off = {}, 0
    for name, t in parts:
        fields[name] = (off, t.nbytes, t.dtype, tuple(t.shape))
        off = (off + t.nbytes + 255) & ~255
    for name, nbytes, dt, shape in (
            ("slots", B * 8, torch.int64, (B,)),
            ("table", B * max_blocks * 4, torch.int32, (B, max_blocks)),
            ("lens", B * 4, torch.int32, (B,))):
        fields[name] = (off, nbytes, dt, shape)
        off = (off + nbytes + 255) & ~255
    total = off

    def views(buf):
        return {k: buf[o:o + n].view(dt).view(shape)
                for k, (o, n, dt, shape) in fields.items()}

    depth = 3
    stage = [torch.empty(total, dtype=torch.uint8).pin_memory()
             for _ in range(depth)]
    hv = [views(x) for x in stage]
    for v in hv:
        for name, t in parts:
            v[name].copy_(t.cpu())
    dstage = [torch.empty(total, dtype=torch.uint8, device=dev)
              for _ in range(depth)]
    dv = [views(x) for x in dstage]
    dout = [torch.empty_like(inp.q) for _ in range(depth)]
    hout = [torch.empty(inp.q.shape, dtype=inp.q.dtype).pin_memory()
            for _ in range(depth)]
    desc = pkv.make_desc(inp.q, inp.k_cache, dv[0]["table"],
                         partition_size=ps,
                         max_context_len=int(final_lens.max()))
    ws = torch.empty(max(pkv.pa_decode_workspace_bytes(desc), 16),
                     dtype=torch.uint8, device=dev)
    ones = np.ones(B, dtype=np.int32)
    stream = torch.cuda.current_stream(dev)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_up = [torch.cuda.Event() for _ in range(depth)]
    ev_run = [torch.cuda.Event() for _ in range(depth)]
    ev_down = [torch.cuda.Event() for _ in range(depth)]

    def prepare(i):
        """Host work of one step into staging buffer i."""
        ev_up[i].synchronize()          # its previous upload has left
        _, pairs = bm.append_batch(ids, ones, slots_out=hv[i]["slots"].numpy())
        _, lens = bm.block_table(ids, max_blocks,
                                 table_out=hv[i]["table"].numpy(),
                                 lens_out=hv[i]["lens"].numpy())
        return pairs, int(lens.sum())

    def upload(i):
        up.wait_event(ev_run[i])        # kernels of `depth` steps ago
        with torch.cuda.stream(up):
            dstage[i].copy_(stage[i], non_blocking=True)
        ev_up[i].record(up)

    def launch(i, pairs):
        stream.wait_event(ev_up[i])
        stream.wait_event(ev_down[i])   # dout[i] of `depth` steps ago
        nb = 0
        if len(pairs):
            d_pairs = torch.from_numpy(pairs).pin_memory().to(
                dev, non_blocking=True)
            pkv.pa_copy_blocks(inp.k_cache, inp.v_cache, d_pairs)
            nb = pairs.nbytes
        pkv.pa_cache_write(inp.k_cache, inp.v_cache, dv[i]["k"], dv[i]["v"],
                           dv[i]["slots"])
        pkv.pa_decode(dout[i], dv[i]["q"], inp.k_cache, inp.v_cache,
                      dv[i]["table"], dv[i]["lens"], w.softmax_scale,
                      desc=desc, workspace=ws)
        ev_run[i].record(stream)
        down.wait_event(ev_run[i])
        with torch.cuda.stream(down):
            hout[i].copy_(dout[i], non_blocking=True)
        ev_down[i].record(down)
        return nb

    def run(n0, count, start=None):
        """Steps n0 .. n0+count-1; returns (tokens attended, pair bytes)."""
        if count == 0:
            return 0, 0
        if start is not None:
            up.wait_event(start)
        tokens, nb = 0, 0
        nxt = prepare(n0 % depth)
        upload(n0 % depth)
        for n in range(n0, n0 + count):
            pairs, tok = nxt
            nb = max(nb, launch(n % depth, pairs))
            tokens += tok
            if n + 1 < n0 + count:
                nxt = prepare((n + 1) % depth)
                upload((n + 1) % depth)
            if n >= n0 + depth - 1:
                ev_down[(n - depth + 1) % depth].synchronize()  # its output
        stream.wait_event(ev_down[(n0 + count - 1) % depth])
        return tokens, nb

    run(0, args.warmup)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    tot_tokens, nb = run(args.warmup, steps, start=a)
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(a.elapsed_time(b), world)
    # The last step's output, as it reached the host, must equal a decode of
    # the same inputs run on its own now (the kernel is deterministic).
    last = (args.warmup + steps - 1) % depth
    again = torch.empty_like(dout[last])
    pkv.pa_decode(again, dv[last]["q"], inp.k_cache, inp.v_cache,
                  dv[last]["table"], dv[last]["lens"], w.softmax_scale,
                  desc=desc, workspace=ws)
    if steps and not torch.equal(again.cpu(), hout[last]):
        raise RuntimeError("end-to-end output differs from a plain decode "
                           "of the same step")
    bm.close()
    tot_bytes = tot_tokens * w.num_kv_heads * w.head_dim * 2 * 2
    return {"value": round(world * tot_bytes / (ms * 1e-3) / 1e9, 2),
            "unit": "GB/s", "h2d_bytes_per_step": int(total + nb),
            "d2h_bytes_per_step": int(hout[0].nbytes),
            "ms_per_step": round(ms / steps, 4),
            "includes": "host block-manager append + table build, one packed "
                        "pinned H2D of q/new K,V/slots/tables/lengths, cache "
                        "write, decode, D2H of the output, host wait for each "
                        "output; step n+1's host work and H2D and earlier "
                        "steps' D2H overlap step n's kernels (3 buffers)"}


def wl_blocks(lengths, bs):
    from paged_kv_cache_383_b200 import workloads as wl
    return wl.blocks_needed(lengths, bs)


def _free_order(inp):
    """The pool order under which a fresh block manager hands out exactly
    the workload's tables: their blocks in sequence order, then the rest."""
    used = [inp.block_tables[b, : int(wl_blocks([L], inp.workload.block_size)
                                      [0])]
            for b, L in enumerate(inp.lengths)]
    used = np.concatenate(used) if used else np.zeros(0, np.int32)
    rest = np.setdiff1d(np.arange(inp.num_blocks), used, assume_unique=False)
    return np.concatenate([used, rest]).astype(np.int32)


# ---------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)

def _oracle_task(task):
    import numpy as _np
    from oracle import attention as oa
    q, kc, vc, L, scale = task
    sub = _np.arange(kc.shape[0])[None, :]
    return oa.paged_decode(q, kc, vc, sub, _np.array([L]), scale)


POOL_SIZE = os.cpu_count() or 1


def start_oracle_pool():
    import multiprocessing as mp
    os.environ.setdefault("OMP_NUM_THREADS", "1")
    os.environ.setdefault("OPENBLAS_NUM_THREADS", "1")
    os.environ.setdefault("MKL_NUM_THREADS", "1")
    ctx = mp.get_context("spawn")
    return ctx.Pool(POOL_SIZE)


def _tasks_from_device(inp, w, seqs):
    import torch
    tasks = []
    for b in seqs:
        L = int(inp.lengths[b])
        n = int(wl_blocks([L], w.block_size)[0])
        idx = torch.from_numpy(inp.block_tables[b, :n].astype(np.int64)).to(
            inp.k_cache.device)
        tasks.append((inp.q[b:b + 1].float().cpu().numpy(),
                      inp.k_cache.index_select(0, idx).float().cpu().numpy(),
                      inp.v_cache.index_select(0, idx).float().cpu().numpy(),
                      L, w.softmax_scale))
    return tasks


def time_oracle(pool, tasks, min_seconds):
    t0 = time.time()
    reps = 0
    while True:
        pool.map(_oracle_task, tasks, chunksize=1)
        reps += 1
        if time.time() - t0 >= min_seconds:
            break
    return time.time() - t0, reps


def cpu_baseline(pool, inp, w, dev):
    seqs = list(range(min(64, w.num_seqs)))
    tasks = _tasks_from_device(inp, w, seqs)
    secs, reps = time_oracle(pool, tasks, 10.0)
    toks = int(inp.lengths[seqs].sum())
    gbs = reps * kv_bytes(inp.lengths[seqs], w) / secs / 1e9
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": POOL_SIZE,
            "kind": "oracle",
            "seq_layers_per_s": round(reps * len(seqs) / secs, 2),
            "sample": f"first {len(seqs)} of {w.num_seqs} sequences of "
                      f"{w.name} ({toks} tokens), fp64 oracle repeated "
                      f"{reps}x over {secs:.1f} s, process pool of "
                      f"{POOL_SIZE} (1 BLAS thread each)"}


def run_reference(args, rank, world):
    """The reference arm: the fp64 CPU oracle on this workload's shape, each
    step a bounded sample of the batch (inputs drawn on the host)."""
    from paged_kv_cache_383_b200 import workloads as wl
    pool = start_oracle_pool()
    w = wl.WORKLOADS[args.workload]
    n = min(16, w.num_seqs)
    ws = w.scaled(num_seqs=n) if w.lengths != "fixed" else w
    inp = wl.make_paged(ws, device="cpu")
    tasks = _tasks_from_device(inp, ws, range(ws.num_seqs))
    for _ in range(args.warmup):
        pool.map(_oracle_task, tasks, chunksize=1)
    t0 = time.time()
    for _ in range(args.steps):
        pool.map(_oracle_task, tasks, chunksize=1)
    secs = time.time() - t0
    pool.close()
    step_bytes = kv_bytes(inp.lengths, ws)
    value = args.steps * step_bytes / secs / 1e9
    cores = POOL_SIZE
    sample = (f"{ws.num_seqs} sequences drawn with {w.name}'s length "
              f"distribution ({int(inp.lengths.sum())} tokens) per step")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4),
            "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(1e3 * secs / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "sample": sample},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s",
                             "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s",
                    "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse_args()
    rank, world, local = dist_setup(args)
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    if args.extras_only:
        print(json.dumps(run_extras_only(args)), flush=True)
        return
    res = run_native(args, rank, world, local)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
