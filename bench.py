#!/usr/bin/env python
"""Benchmark of the Sketch&Walk hot path on B200 (one process per GPU).

Default run (N=1): the long-context prefill workload of 4 layers, 32 query /
8 KV heads, d=128, n=131072, B=128, k=32, s=8, 20% density (bf16); one step =
one pass of sws_sketch -> sws_walk_select -> sws_sparse_attn_prefill over all
4 layers. The same workload at 10% density, the 8-layer 65536-token workload
and the 4-layer 16384-token workload are timed in the same run and reported
under "prefill_workloads"; the decode workload (16 sequences x 131072 cached
tokens, 8 layers, 64 steps) under "decode". Every input is seeded synthetic
data resident in HBM before the timed region; "e2e" repeats the headline step
with the inputs copied from pinned host memory and the outputs copied back
inside the timed region.

With --gpus N under torchrun each rank runs an independent replica (the path
has no data exchange); times are the max over ranks.
--impl reference times the oracle (fp64, host cores) on a bounded sample.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill tokens/s + % tensor peak at 20% density; decode step µs + HBM GB/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-steps", type=int, default=None, help="decode steps to run (default: the workload's 64)")
    ap.add_argument("--decode-batch", type=int, default=None, help="smaller decode batch (profiling only)")
    ap.add_argument("--decode-n0", type=int, default=None, help="shorter cached prompt (profiling only)")
    ap.add_argument("--decode-layers", type=int, default=None, help="fewer decode layers (profiling only)")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill measurement (profiling only)")
    ap.add_argument("--no-variants", action="store_true", help="skip the elementwise-walk and dense-first variants")
    ap.add_argument("--profile-prefill", action="store_true",
                    help="profiling run: the headline prefill workload alone (scaled by --prefill-n), no bench line")
    ap.add_argument("--prefill-n", type=int, default=None, help="tokens of the profiled prefill workload")
    ap.add_argument("--profile-workload", default="headline", choices=sorted(PROFILE_WORKLOADS),
                    help="the prefill workload --profile-prefill runs")
    ap.add_argument("--json-out", default=None)
    return ap.parse_args()


def profiled_traffic(name: str, source: str):
    """DRAM bytes per launch (read + write) recorded in profiles/<name>.md by an
    ncu capture, if that capture was taken of the current kernel source."""
    import hashlib
    path = os.path.join(ROOT, "profiles", name + ".md")
    src = os.path.join(ROOT, "block_sparse_attention_sws_b200", "csrc", source)
    if not (os.path.exists(path) and os.path.exists(src)):
        return None
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
    fields = {}
    for line in open(path):
        if line.startswith("- ") and ": " in line:
            k, v = line[2:].split(": ", 1)
            fields[k.strip()] = v.strip().strip("`")
    if fields.get("kernel source sha256") != digest:
        return None
    try:
        return float(fields["dram bytes per launch (read + write)"])
    except (KeyError, ValueError):
        return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    """nvidia-smi sampling of the SM clock and throttle reasons during the timed region."""

    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str):
        self.bus_id = bus_id.lower()
        self.lines = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.th = threading.Thread(target=self._read, daemon=True)
        self.th.start()
        # nvidia-smi takes a moment to start: wait for its first sample so that
        # the samples cover the timed region that follows
        t0 = time.time()
        while not self.lines and time.time() - t0 < 5.0 and self.proc.poll() is None:
            time.sleep(0.01)
        self.skip = len(self.lines)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.th.join(timeout=2)
        mhz, mx, reasons, watts = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines[max(0, getattr(self, "skip", 0) - 1):]:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            bus = parts[0].lower()
            if self.bus_id and not (bus.endswith(self.bus_id) or self.bus_id.endswith(bus)):
                continue
            try:
                mhz.append(float(parts[1]))
                mx.append(float(parts[2]))
                watts.append(float(parts[3]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(watts) if watts else None, "samples": len(mhz), "reasons": sorted(reasons)}


def gpu_bus_id(torch) -> str:
    p = torch.cuda.get_device_properties(torch.cuda.current_device())
    return f"{getattr(p, 'pci_domain_id', 0):08x}:{getattr(p, 'pci_bus_id', 0):02x}:{getattr(p, 'pci_device_id', 0):02x}.0"


# ------------------------------------------------------------- distributed --

def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() and dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------ cpu baseline --

ORACLE_SAMPLE_BLOCKS = 64  # query blocks per head-layer whose attention the oracle computes


def oracle_head_layers(w, sample_blocks=ORACLE_SAMPLE_BLOCKS):
    """The oracle over the workload one (head, layer) at a time, head by head,
    each head's walk state carried through its layers. Per head-layer it runs
    the sketch, walk and selection in full and the attention of a seeded
    sample of query blocks (every block when the workload has no more than
    sample_blocks), and yields (seconds of the sketch-walk-select part, seconds
    of the sampled attention, key-block pairs of all query blocks / pairs of
    the sampled ones). Input generation is not timed."""
    import numpy as np
    import oracle
    import sws_inputs as W
    from oracle import sws_oracle as so
    Hd = oracle.srht_matrix(w.d, w.k, w.seed)
    rng = np.random.default_rng(w.seed)
    h = 0
    while True:
        st = so.PrefillState()
        for layer in range(w.layers):
            q, k, v = W.prefill_head_inputs(w, layer, h % w.hq)
            q64, k64, v64 = (x.double().numpy() for x in (q, k, v))
            t0 = time.perf_counter()
            out = so.prefill_layer(q64[None], k64[None], v64[None], Hd, w.B, w.s, w.density, st, heads=[0],
                                   attention_blocks=None)[0]
            t1 = time.perf_counter()
            rp, ci = out["row_ptr"], out["col_idx"]
            blocks = (list(range(w.b)) if w.b <= sample_blocks
                      else sorted(int(x) for x in rng.choice(w.b, sample_blocks, replace=False)))
            so.sparse_attention(q64, k64, v64, rp, ci, w.B, blocks)
            t2 = time.perf_counter()
            sampled = sum(int(rp[i + 1] - rp[i]) for i in blocks)
            yield t1 - t0, t2 - t1, int(rp[-1]) / sampled
        h += 1


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def head_layer_estimate(t_sws, t_attn, scale) -> float:
    """Oracle seconds of one whole head-layer: the sketch, walk and selection as
    run, plus the sampled attention scaled linearly by key-block pairs."""
    return t_sws + t_attn * scale


def cpu_baseline(w, budget_s=15.0):
    """The oracle on whole heads (every layer of a head, its walk carried) until
    the budget is spent; one pass = hq x layers head-layers."""
    measured, est, done = 0.0, 0.0, 0
    for t_sws, t_attn, scale in oracle_head_layers(w):
        measured += t_sws + t_attn
        est += head_layer_estimate(t_sws, t_attn, scale)
        done += 1
        if done % w.layers == 0 and (measured >= budget_s or done >= w.hq * w.layers):
            break
    full = est / done * w.hq * w.layers
    sampled = "every query block" if w.b <= ORACLE_SAMPLE_BLOCKS else \
        f"attention of {ORACLE_SAMPLE_BLOCKS} seeded query blocks of {w.b} per head-layer"
    return {"value": w.n / full, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"oracle (fp64 numpy) on {done // w.layers} of {w.hq} query heads x {w.layers} layers: "
                      f"sketch, walk and selection in full, {sampled}; {measured:.1f} s measured, extrapolated "
                      f"linearly (attention by key-block pairs, then by heads) to the whole pass",
            "extrapolated": w.b > ORACLE_SAMPLE_BLOCKS or done < w.hq * w.layers,
            "host_cpus": os.cpu_count()}


# --------------------------------------------------------------- reference --

def workload_config(w, world) -> dict:
    """The config dict of a prefill workload, the same in both arms."""
    return {"workload": w.name, "layers": w.layers, "hq": w.hq, "hkv": w.hkv, "d": w.d, "n": w.n, "B": w.B,
            "k": w.k, "s": w.s, "density": f"{w.density[0]}/{w.density[1]}", "parallelism": f"replicas x{world}",
            "l2": f"inputs larger than L2 ({prefill_input_bytes(w) / 1e6:.0f} MB per step)"}


def prefill_input_bytes(w) -> int:
    elem = 4 if w.dtype == "fp32" else 2
    return w.layers * (w.hq + 2 * w.hkv) * w.n * w.d * elem


def run_reference(args, world, rank):
    import sws_inputs as W
    if rank != 0:
        return 0
    w = headline_workload(W)
    # one step = one (head, layer) of the pass, heads in turn with their walk
    # state carried across steps: sketch, walk and selection in full, attention
    # on a seeded sample of query blocks
    it = oracle_head_layers(w)
    for _ in range(args.warmup):
        next(it)
    runs = [next(it) for _ in range(args.steps)]
    measured = statistics.mean(a + b for a, b, _ in runs)
    full = statistics.mean(head_layer_estimate(*r) for r in runs) * w.hq * w.layers
    value = w.n / full
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": measured * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, world),
        "extrapolated_ms_per_full_pass": full * 1e3,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "kind": "oracle", "cores": blas_threads(),
                         "sample": f"each step: the oracle (fp64 numpy) on one head-layer ({w.hq} query heads x "
                                   f"{w.layers} layers make a pass): sketch, walk and selection in full, attention "
                                   f"of {min(w.b, ORACLE_SAMPLE_BLOCKS)} seeded query blocks of {w.b}; ms_per_step is "
                                   f"that measured step; value extrapolates it linearly (attention by key-block "
                                   f"pairs, then by the {w.hq * w.layers} head-layers) to the whole pass"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------- ours ---

# --profile-prefill's choice of workload (attribute names in sws_inputs)
PROFILE_WORKLOADS = {"headline": "PREFILL_128K", "prefill_128k_d10": "PREFILL_128K_D10", "prefill_64k": "PREFILL_64K",
                     "prefill_16k": "PREFILL_16K"}


def headline_workload(W):
    """The N=1 workload: the longest prefill (131072 tokens, 4 layers) at 20% density."""
    return W.PREFILL_128K


def extra_workloads(W):
    """The other prefill workloads, timed after the headline: the same long
    context at 10% density, 65536 tokens over 8 layers, 16384 tokens over 4."""
    return [W.PREFILL_128K_D10, W.PREFILL_64K, W.PREFILL_16K]


def bench_prefill(args, world, S, W, torch, w, steps):
    cfg = S.make_config(w.d, w.B, w.k, w.s, 0, w.density, w.seed)
    h = S.Handle(cfg)
    path = S.PrefillPath(h, w.n, w.hq, w.hkv, torch.bfloat16)
    inputs = [W.prefill_layer_inputs(w, layer, "cuda") for layer in range(w.layers)]
    stream = torch.cuda.current_stream()
    in_bytes = sum(x.numel() * x.element_size() for t in inputs for x in t)

    def step(ev=None):
        for layer, (Q, K, V) in enumerate(inputs):
            if ev is not None:
                ev[layer][0].record(stream)
            path.sketch(Q, K)
            if ev is not None:
                ev[layer][1].record(stream)
            path.walk_select(layer == 0)
            if ev is not None:
                ev[layer][2].record(stream)
            path.attention(Q, K, V)
            if ev is not None:
                ev[layer][3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert S.sws_sync_check(h) == 0
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(w.layers)]
           for _ in range(steps)]
    clocks = ClockSampler(gpu_bus_id(torch))
    clocks.start()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    launches0 = S.sws_launch_count()
    t_start.record(stream)
    for i in range(steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    launches = S.sws_launch_count() - launches0
    barrier(world)
    clk = clocks.stop()
    assert S.sws_sync_check(h) == 0
    ms = t_start.elapsed_time(t_end)
    ms_max = max_over_ranks(ms, world)
    stage = {"sketch": 0.0, "walk_select": 0.0, "attention": 0.0}
    attn_ms = []
    for i in range(steps):
        for layer in range(w.layers):
            e = evs[i][layer]
            stage["sketch"] += e[0].elapsed_time(e[1])
            stage["walk_select"] += e[1].elapsed_time(e[2])
            a = e[2].elapsed_time(e[3])
            stage["attention"] += a
            attn_ms.append(a)
    stage = {k: v / steps for k, v in stage.items()}
    flops = w.hq * path.nnz * 4 * w.B * w.B * w.d  # executed block pairs x 4 B^2 d
    # Q and K read once, the sketches written; the score matrix only when it is formed in memory
    sketch_bytes = (w.hq + w.hkv) * w.n * w.d * 2 + 8 * (w.hq + w.hkv) * path.b * w.k
    if path.scores_in_memory:
        sketch_bytes += 8 * w.hq * path.b * (path.b + 1) // 2
    res = dict(w=w, h=h, path=path, inputs=inputs, ms=ms_max, steps=steps, launches=launches, clocks=clk,
               stage=stage, attn_ms=statistics.mean(attn_ms), flops=flops, sketch_bytes=sketch_bytes,
               in_bytes=in_bytes, mma_work=mma_work(path, w, torch))
    return res


# Whether attn_tc_kernel skips the products of a (query tile, key tile) pair in
# which no query block of the tile selected a key block of the tile.
ATTN_SKIPS_UNSELECTED_TILES = False


def mma_work(path, w, torch) -> dict:
    """Tensor-core work that attn_tc_kernel executes for the last layer's CSR
    against the algorithmic work (4 B^2 d flops per selected block pair). The
    kernel takes 256 query rows at a time (two 128-row tiles) over the union of
    their query blocks' key blocks, 128 keys per tile, and runs both tiles' score
    and PV products on every key tile of the union unless a tile has no selected
    pair, which it skips."""
    b, B, QB = path.b, w.B, 256 // w.B
    rp = path.row_ptr.long()
    ci = path.col_idx.long()
    sel = torch.zeros(w.hq, b, b, dtype=torch.bool, device=rp.device)
    rows = torch.repeat_interleave(torch.arange(b, device=rp.device), rp[0, 1:] - rp[0, :-1])
    for h in range(w.hq):
        sel[h, rows, ci[h, :rows.numel()]] = True
    nslab = -(-b // QB)
    pad = torch.zeros(w.hq, nslab * QB, b, dtype=torch.bool, device=rp.device)
    pad[:, :b] = sel
    slab = pad.reshape(w.hq, nslab, QB, b)
    union = slab.any(dim=2)                                    # [hq, slab, key block]
    kb_per_tile = 128 // B
    # key tiles of the merged stream: union blocks taken kb_per_tile at a time
    tiles = (union.sum(dim=2) + kb_per_tile - 1) // kb_per_tile  # [hq, slab]
    qpt = 128 // B  # query blocks per 128-row tile
    tile_sel = slab.reshape(w.hq, nslab, 2, qpt, b).any(dim=3)  # [hq, slab, query tile, key block]
    if ATTN_SKIPS_UNSELECTED_TILES:
        # a query tile runs a key tile only if one of its query blocks selected one of the tile's key blocks
        ts = tile_sel[..., :b]
        if kb_per_tile > 1:  # key tiles are consecutive union blocks: count per merged tile
            executed = 0
            for h in range(w.hq):
                for p in range(nslab):
                    blocks = union[h, p].nonzero().flatten()
                    for t in range(0, blocks.numel(), kb_per_tile):
                        blk = blocks[t:t + kb_per_tile]
                        executed += int(ts[h, p][:, blk].any(dim=1).sum().item())
        else:
            executed = int(ts.sum().item())
    else:
        executed = 2 * int(tiles.sum().item())  # both query tiles on every key tile of the union
    algorithmic = int(sel.sum().item())
    flops_tile = 4 * 128 * 128 * w.d
    return {"executed_tile_products": executed, "selected_block_pairs": algorithmic,
            "executed_flops": executed * flops_tile, "algorithmic_flops": algorithmic * 4 * B * B * w.d,
            "executed_over_algorithmic": executed * flops_tile / (algorithmic * 4 * B * B * w.d)}


def prefill_summary(pf, world, peaks, peak_kind) -> dict:
    """tokens/s, the attention kernel's roofline (its peak chosen by the clocks the
    timed region saw), the sketch stage's HBM roofline and the stage split."""
    w = pf["w"]
    ms_step = pf["ms"] / pf["steps"]
    attn_tflops = pf["flops"] / (pf["attn_ms"] * 1e-3) / 1e12
    # The burst GEMM peak was measured at full SM clocks, the sustained one under
    # the power cap at lower clocks: take the one whose clocks the timed region saw.
    sm, smx = pf["clocks"].get("sm_mhz"), pf["clocks"].get("sm_max_mhz")
    burst = peaks.get("bf16_tflops", peaks.get("bf16_tflops_sustained"))
    sustained = peaks.get("bf16_tflops_sustained", burst)
    at_full_clock = sm is None or smx is None or sm >= 0.9 * smx
    peak_t = burst if at_full_clock else sustained
    peak_name = "bf16 burst" if at_full_clock else "bf16 sustained"
    sk = pf["sketch_bytes"] / (pf["stage"]["sketch"] / w.layers * 1e-3) / 1e9
    return {
        "tokens_per_s": world * w.n / (ms_step * 1e-3), "ms_per_step": ms_step, "steps": pf["steps"],
        "config": workload_config(w, world),
        "stages_ms_per_step": pf["stage"],
        "roofline": {"kernel": f"attn_tc_kernel<{w.d},{w.B}> (sws_sparse_attn_prefill)", "bound": "tensor",
                     "achieved": attn_tflops, "peak": peak_t, "unit": "TFLOP/s", "frac": attn_tflops / peak_t,
                     "traffic": profiled_traffic(f"attn_tc_prefill_n{w.n}_B{w.B}", "k_attn_tc.cu"),
                     "peak_source": f"{peak_kind} {peak_name}",
                     "frac_of_burst": attn_tflops / burst, "frac_of_sustained": attn_tflops / sustained,
                     "flops_per_launch": pf["flops"], "ms_per_launch": pf["attn_ms"]},
        "sketch_roofline": {"bound": "hbm", "achieved": sk, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": sk / peaks["hbm_gbs"], "bytes_per_layer": pf["sketch_bytes"]},
        "clocks": pf["clocks"], "gpu_launches": pf["launches"],
        "attention_mma_work": pf["mma_work"],
    }


def bench_scores_on_chip(args, world, S, torch, pf):
    """The headline step with the sketched scores formed on chip inside the walk
    (sws_sketch without the score matrix, then sws_walk_select_sketch), on the
    same inputs: the route that keeps the b x b matrix out of device memory."""
    w, inputs = pf["w"], pf["inputs"]
    path = S.PrefillPath(pf["h"], w.n, w.hq, w.hkv, torch.bfloat16, scores_in_memory=False)
    stream = torch.cuda.current_stream()
    steps = max(3, min(args.steps, 20))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(w.layers * steps)]

    def step(rec):
        for layer, (Q, K, V) in enumerate(inputs):
            e = ev[rec * w.layers + layer] if rec is not None else None
            if e:
                e[0].record(stream)
            path.sketch(Q, K)
            path.walk_select(layer == 0)
            if e:
                e[1].record(stream)
            path.attention(Q, K, V)
            if e:
                e[2].record(stream)

    for _ in range(args.warmup):
        step(None)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    a.record(stream)
    for i in range(steps):
        step(i)
    b.record(stream)
    torch.cuda.synchronize()
    assert S.sws_sync_check(pf["h"]) == 0
    ms = max_over_ranks(a.elapsed_time(b), world) / steps
    sw = sum(e[0].elapsed_time(e[1]) for e in ev) / steps
    del path
    return {"tokens_per_s": world * w.n / (ms * 1e-3), "ms_per_step": ms, "steps": steps,
            "sketch_walk_select_ms_per_step": sw}


def bench_prefill_variants(args, world, S, W, torch, pf):
    """The pages' own alternatives on the inputs of a prefill measurement (the
    16384-token workload), timed like its step: the entrywise walk power (the
    other reading of (.)^s) and the dense-first-two-layers policy of §7."""
    w, inputs = pf["w"], pf["inputs"]
    stream = torch.cuda.current_stream()
    steps = max(3, min(args.steps, 20))
    out = {}
    for name, mode, dense in (("elementwise_walk", S.SWS_WALK_ELEMENTWISE, 0),
                              ("dense_first_2_layers", S.SWS_WALK_MATRIX_POWER, 2)):
        cfg = S.make_config(w.d, w.B, w.k, w.s, mode, w.density, w.seed)
        h = S.Handle(cfg)
        path = S.PrefillPath(h, w.n, w.hq, w.hkv, torch.bfloat16, dense_layers=dense)

        def step():
            for layer, (Q, K, V) in enumerate(inputs):
                path.layer(Q, K, V, layer == 0, layer=layer)

        for _ in range(args.warmup):
            step()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(steps):
            step()
        b.record(stream)
        torch.cuda.synchronize()
        assert S.sws_sync_check(h) == 0
        ms = max_over_ranks(a.elapsed_time(b), world) / steps
        out[name] = {"tokens_per_s": world * w.n / (ms * 1e-3), "ms_per_step": ms, "steps": steps}
        h.close()
        if path.h_dense is not None:
            path.h_dense.close()
        del path
    out["batch_8x2048"] = bench_prefill_batch(args, world, S, W, torch)
    out["batch_mixed_lengths"] = bench_prefill_batch(args, world, S, W, torch, MIXED_LENGTHS)
    return out


# sequence lengths of the mixed prefill batch (tokens; 33,276 in all)
MIXED_LENGTHS = (8192, 6144, 4096, 3000, 2048, 2048, 1536, 1024, 1024, 2900, 700, 564)


def bench_prefill_batch(args, world, S, W, torch, lengths=None):
    """Prefill batching: eight 2048-token sequences (or the given lengths) of the
    headline workload's shape (4 layers, 32/8 heads), through PrefillBatch:
    each sequence's layer on its own stream; the sequences packed end to end
    with one attention launch for all (the sketches and walks on their
    streams); and, for comparison, the same paths one after another on one
    stream."""
    base = W.PREFILL_16K
    lengths = (2048,) * 8 if lengths is None else tuple(lengths)
    ws = [base.scaled(name=f"seq{i}", n=n, seed=base.seed + 100 + i) for i, n in enumerate(lengths)]
    inputs = [[W.prefill_layer_inputs(w, layer, "cuda") for w in ws] for layer in range(base.layers)]
    h = S.Handle(S.make_config(base.d, base.B, base.k, base.s, 0, base.density, base.seed))
    batch = S.PrefillBatch(h, [w.n for w in ws], base.hq, base.hkv, torch.bfloat16)
    stream = torch.cuda.current_stream()
    steps = max(3, min(args.steps, 20))
    out = {"sequences": len(ws), "tokens_per_sequence": list(lengths) if len(set(lengths)) > 1 else lengths[0],
           "steps": steps}
    packed = [[torch.cat([x[j] for x in ins], dim=1) for j in range(3)] for ins in inputs]
    for mode in ("concurrent_streams", "packed_launch", "one_stream"):
        def step():
            for layer, ins in enumerate(inputs):
                if mode == "concurrent_streams":
                    batch.layer([x[0] for x in ins], [x[1] for x in ins], [x[2] for x in ins], layer == 0)
                elif mode == "packed_launch":
                    batch.layer_packed(*packed[layer], layer == 0)
                else:
                    for p, (Q, K, V) in zip(batch.paths, ins):
                        p.layer(Q, K, V, layer == 0)

        for _ in range(args.warmup):
            step()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(steps):
            step()
        b.record(stream)
        torch.cuda.synchronize()
        assert S.sws_sync_check(h) == 0
        ms = max_over_ranks(a.elapsed_time(b), world) / steps
        out[mode] = {"tokens_per_s": world * sum(w.n for w in ws) / (ms * 1e-3), "ms_per_step": ms}
    h.close()
    return out


def bench_prefill_e2e(args, world, S, torch, pf):
    """The same path through the C ABI with every layer's Q, K, V copied in
    from pinned host memory and O copied back, all inside the timed region.
    Copies in, compute and copies out run on three streams, so a layer's
    transfers overlap the neighbouring layers' work and the two directions of
    the host link overlap each other; per-layer events keep every buffer's
    reuse ordered."""
    w, path, inputs = pf["w"], pf["path"], pf["inputs"]
    host_in = [tuple(x.cpu().pin_memory() for x in t) for t in inputs]
    host_out = [torch.empty_like(path.o, device="cpu").pin_memory() for _ in range(w.layers)]
    outs = [torch.empty_like(path.o) for _ in range(w.layers)]
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(w.layers)]
    ev_comp = [torch.cuda.Event() for _ in range(w.layers)]
    ev_out = [torch.cuda.Event() for _ in range(w.layers)]
    for e in ev_comp + ev_out:
        e.record(torch.cuda.current_stream())
    torch.cuda.synchronize()

    def step():
        for layer in range(w.layers):
            dq, dk, dv = inputs[layer]
            hq_, hk_, hv_ = host_in[layer]
            s_in.wait_event(ev_comp[layer])  # the previous step's layer is done reading its inputs
            with torch.cuda.stream(s_in):
                dq.copy_(hq_, non_blocking=True)
                dk.copy_(hk_, non_blocking=True)
                dv.copy_(hv_, non_blocking=True)
            ev_in[layer].record(s_in)
            s_comp.wait_event(ev_in[layer])
            s_comp.wait_event(ev_out[layer])  # the previous step's output has left the device
            path.layer(dq, dk, dv, layer == 0, out=outs[layer], stream=s_comp)
            ev_comp[layer].record(s_comp)
            s_out.wait_event(ev_comp[layer])
            with torch.cuda.stream(s_out):
                host_out[layer].copy_(outs[layer], non_blocking=True)
            ev_out[layer].record(s_out)

    for _ in range(args.warmup):
        step()
    steps = max(3, args.steps // 2)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    a.record(s_comp)
    s_in.wait_event(a)
    s_out.wait_event(a)
    for _ in range(steps):
        step()
    s_comp.wait_stream(s_in)
    s_comp.wait_stream(s_out)
    b.record(s_comp)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), world) / steps
    h2d = sum(x.numel() * x.element_size() for t in host_in for x in t)
    d2h = sum(x.numel() * x.element_size() for x in host_out)
    return {"value": world * w.n / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "overlap": "copies in, compute, copies out "
            "on three streams"}


def bench_decode(args, world, S, W, torch, peaks):
    wd = W.DECODE_128K
    if args.decode_steps is not None:
        wd = wd.scaled(steps=max(2, min(wd.steps, args.decode_steps)))
    if args.decode_batch is not None:
        wd = wd.scaled(batch=args.decode_batch)
    if args.decode_n0 is not None:
        wd = wd.scaled(n0=args.decode_n0)
    if args.decode_layers is not None:
        wd = wd.scaled(layers=args.decode_layers)
    cfg = S.make_config(wd.d, wd.B, wd.k, wd.s, 0, wd.density, wd.seed)
    h = S.Handle(cfg)
    path = S.DecodePath(h, wd.batch, wd.hq, wd.hkv, wd.max_len, wd.layers)
    toks_k = torch.empty(wd.steps, wd.layers, wd.batch, wd.hkv, wd.d, dtype=torch.bfloat16, device="cuda")
    toks_v = torch.empty_like(toks_k)
    toks_q = torch.empty(wd.steps, wd.layers, wd.batch, wd.hq, wd.d, dtype=torch.bfloat16, device="cuda")
    for layer in range(wd.layers):
        for s_ in range(wd.batch):
            K, V = W.decode_cache_inputs(wd, s_, layer, "cuda")
            path.k_cache[layer][s_].copy_(K)
            path.v_cache[layer][s_].copy_(V)
            toks_k[:, layer, s_] = K[:, wd.n0:].transpose(0, 1)
            toks_v[:, layer, s_] = V[:, wd.n0:].transpose(0, 1)
            del K, V
            toks_q[:, layer, s_] = W.decode_queries(wd, s_, layer, "cuda").transpose(0, 1)
    path.init_cache(torch.full((wd.batch,), wd.n0, dtype=torch.int32, device="cuda"))
    union_log = torch.zeros(wd.steps, wd.layers, wd.batch, wd.hkv, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    warm = min(args.warmup, wd.steps - 1)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * wd.layers + 1)] for _ in range(wd.steps)]

    def step(t, rec, h=h):
        path.begin_step()
        if rec:
            ev[t][0].record(stream)
        for layer in range(wd.layers):
            L = S
            if path.paged:
                L.sws_decode_step_paged(h, toks_q[t, layer], toks_k[t, layer], toks_v[t, layer], path.k_cache[layer],
                                        path.v_cache[layer], path.block_table, path.seq_lens, path.k_psum[layer],
                                        path.k_sketch[layer], layer == 0, path.walk_state, path.head_sel,
                                        path.head_cnt, path.sel, path.sel_mask, path.sel_cnt)
            else:
                L.sws_decode_step(h, toks_q[t, layer], toks_k[t, layer], toks_v[t, layer], path.seq_lens,
                                  path.k_cache[layer], path.v_cache[layer], path.k_psum[layer], path.k_sketch[layer],
                                  layer == 0, path.walk_state, path.head_sel, path.head_cnt, path.sel, path.sel_mask,
                                  path.sel_cnt)
            if rec:
                ev[t][1 + 2 * layer].record(stream)
            if path.paged:
                L.sws_sparse_attn_decode_paged(h, toks_q[t, layer], path.k_cache[layer], path.v_cache[layer],
                                               path.block_table, path.seq_lens, path.sel, path.sel_mask, path.sel_cnt,
                                               path.o, path.ws)
            else:
                L.sws_sparse_attn_decode(h, toks_q[t, layer], path.k_cache[layer], path.v_cache[layer],
                                         path.seq_lens, path.sel, path.sel_mask, path.sel_cnt, path.o, path.ws)
            if rec:
                ev[t][2 + 2 * layer].record(stream)
            union_log[t, layer].copy_(path.sel_cnt, non_blocking=True)

    for t in range(warm):
        step(t, False)
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_bus_id(torch))
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for t in range(warm, wd.steps):
        step(t, True)
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    assert S.sws_sync_check(h) == 0
    timed = wd.steps - warm
    step_ms = max_over_ranks(a.elapsed_time(b), world) / timed
    attn_ms, sel_ms = [], []
    for t in range(warm, wd.steps):
        for layer in range(wd.layers):
            sel_ms.append(ev[t][2 * layer].elapsed_time(ev[t][1 + 2 * layer]))
            attn_ms.append(ev[t][1 + 2 * layer].elapsed_time(ev[t][2 + 2 * layer]))
    u = union_log[warm:].double()
    kv_bytes = float(u.sum().item()) * wd.B * wd.d * 2 * 2 / timed  # union blocks x (K + V) per step
    nb = -(-(wd.n0 + wd.steps) // wd.B)
    units = wd.batch * wd.hkv * wd.layers
    sk_bytes = units * nb * wd.k * 8 + wd.batch * wd.hq * wd.layers * nb * 8 * 2  # k~ reads, rho read+write
    tok_bytes = wd.layers * wd.batch * (2 * wd.hq + 2 * wd.hkv) * wd.d * 2
    step_bytes = kv_bytes + sk_bytes + tok_bytes
    attn_launch_ms = statistics.mean(attn_ms)
    attn_bytes = kv_bytes / wd.layers
    hbm = peaks["hbm_gbs"]
    dense_bytes = units * (wd.n0 + wd.steps) * wd.d * 4
    out = {
        "workload": wd.name, "step_us": step_ms * 1e3, "steps_timed": timed, "clocks": clk,
        "hbm_gbs": step_bytes / (step_ms * 1e-3) / 1e9,
        "bytes_per_step": step_bytes, "kv_bytes_per_step": kv_bytes, "dense_kv_bytes_per_step": dense_bytes,
        "union_blocks_per_unit": float(u.mean().item()),
        "stages_us_per_layer": {"decode_step": statistics.mean(sel_ms) * 1e3, "attention": attn_launch_ms * 1e3},
        "roofline": {"kernel": "sws_sparse_attn_decode (split + combine)", "bound": "hbm",
                     "achieved": attn_bytes / (attn_launch_ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                     "frac": attn_bytes / (attn_launch_ms * 1e-3) / 1e9 / hbm,
                     "traffic": profiled_traffic("decode_attn_b16_n131072", "k_decode.cu")},
    }
    if not args.no_variants:
        # the group-shared selection variant on the same caches and tokens: the
        # caches are rebuilt to the prompt and the same steps replayed
        hs = S.Handle(S.make_config(wd.d, wd.B, wd.k, wd.s, 0, wd.density, wd.seed, select_group=wd.hq // wd.hkv))
        path.init_cache(torch.full((wd.batch,), wd.n0, dtype=torch.int32, device="cuda"))
        for t in range(warm):
            step(t, False, hs)
        barrier(world)
        torch.cuda.synchronize()
        a.record(stream)
        for t in range(warm, wd.steps):
            step(t, False, hs)
        b.record(stream)
        torch.cuda.synchronize()
        assert S.sws_sync_check(hs) == 0
        sh_ms = max_over_ranks(a.elapsed_time(b), world) / timed
        us = union_log[warm:].double()
        sh_kv = float(us.sum().item()) * wd.B * wd.d * 2 * 2 / timed
        out["variants"] = {"group_shared_selection": {
            "step_us": sh_ms * 1e3, "kv_bytes_per_step": sh_kv, "union_blocks_per_unit": float(us.mean().item()),
            "hbm_gbs": (sh_kv + sk_bytes + tok_bytes) / (sh_ms * 1e-3) / 1e9}}
        hs.close()
        out["variants"]["exact_walk_rows"] = bench_decode_exact_rows(args, world, S, W, torch, wd, path, toks_q,
                                                                     toks_k, toks_v, warm, union_log)
        # the paged cache: the same caches moved to a pool whose pages hold the
        # blocks in a seeded random order, the same steps replayed
        perm = torch.randperm(wd.batch * path.mb, generator=torch.Generator().manual_seed(wd.seed))
        path.to_paged(perm.to(torch.int32).reshape(wd.batch, path.mb).cuda(), wd.batch * path.mb)
        path.init_cache(torch.full((wd.batch,), wd.n0, dtype=torch.int32, device="cuda"))
        for t in range(warm):
            step(t, False)
        barrier(world)
        torch.cuda.synchronize()
        a.record(stream)
        for t in range(warm, wd.steps):
            step(t, False)
        b.record(stream)
        torch.cuda.synchronize()
        assert S.sws_sync_check(h) == 0
        pg_ms = max_over_ranks(a.elapsed_time(b), world) / timed
        up = union_log[warm:].double()
        pg_kv = float(up.sum().item()) * wd.B * wd.d * 2 * 2 / timed
        out["variants"]["paged_kv"] = {
            "step_us": pg_ms * 1e3, "kv_bytes_per_step": pg_kv, "union_blocks_per_unit": float(up.mean().item()),
            "hbm_gbs": (pg_kv + sk_bytes + tok_bytes) / (pg_ms * 1e-3) / 1e9,
            "same_selection_as_contiguous": bool(torch.equal(up, u))}
    h.close()
    return out


def bench_decode_exact_rows(args, world, S, W, torch, wd, path, toks_q, toks_k, toks_v, warm, union_log):
    """The exact decode walk with stored rows (sws_decode_step_exact_rows) on the
    decode workload's own caches and tokens: the prompt's queries give every
    block's q~ (one sequence at a time), the rows of every layer are built, and
    the same steps are replayed with the exact walk selecting."""
    cfg = path.h.cfg
    h = S.Handle(S.make_config(wd.d, wd.B, wd.k, wd.s, 0, wd.density, wd.seed))
    lens = torch.full((wd.batch,), wd.n0, dtype=torch.int32, device="cuda")
    path.init_cache(lens)
    f64 = dict(dtype=torch.float64, device="cuda")
    q_psum = [torch.zeros(wd.batch, wd.hq, wd.d, **f64) for _ in range(wd.layers)]
    q_sketch = [torch.zeros(wd.batch, wd.hq, path.mb, wd.k, **f64) for _ in range(wd.layers)]
    e = S.sws_decode_exact_rows_entries(cfg, wd.max_len)
    rows = [torch.empty(wd.batch, wd.hq, e, dtype=torch.int32, device="cuda") for _ in range(wd.layers)]
    len1 = torch.full((1,), wd.n0, dtype=torch.int32, device="cuda")  # one sequence's length, 16-byte aligned
    for layer in range(wd.layers):
        for s_ in range(wd.batch):
            Q = W.decode_sequence_queries(wd, s_, layer, "cuda")[None]  # [1, hq, max_len, d]
            S.sws_decode_init_cache(h, Q, len1, q_psum[layer][s_:s_ + 1], q_sketch[layer][s_:s_ + 1])
            del Q
        S.sws_decode_exact_rows_init(h, q_sketch[layer], path.k_sketch[layer], path.seq_lens, rows[layer])
    torch.cuda.synchronize()
    assert S.sws_sync_check(h) == 0
    stream = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * wd.layers + 1)] for _ in range(wd.steps)]

    def step(t, rec):
        path.begin_step()
        if rec:
            ev[t][0].record(stream)
        for layer in range(wd.layers):
            S.sws_decode_step_exact_rows(h, toks_q[t, layer], toks_k[t, layer], toks_v[t, layer], path.seq_lens,
                                         path.k_cache[layer], path.v_cache[layer], path.k_psum[layer],
                                         path.k_sketch[layer], q_psum[layer], q_sketch[layer], rows[layer],
                                         layer == 0, path.walk_state, path.head_sel, path.head_cnt, path.sel,
                                         path.sel_mask, path.sel_cnt)
            if rec:
                ev[t][1 + 2 * layer].record(stream)
            S.sws_sparse_attn_decode(h, toks_q[t, layer], path.k_cache[layer], path.v_cache[layer], path.seq_lens,
                                     path.sel, path.sel_mask, path.sel_cnt, path.o, path.ws)
            if rec:
                ev[t][2 + 2 * layer].record(stream)
            union_log[t, layer].copy_(path.sel_cnt, non_blocking=True)

    for t in range(warm):
        step(t, False)
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for t in range(warm, wd.steps):
        step(t, True)
    b.record(stream)
    torch.cuda.synchronize()
    assert S.sws_sync_check(h) == 0
    timed = wd.steps - warm
    ms = max_over_ranks(a.elapsed_time(b), world) / timed
    sel_ms = statistics.mean(ev[t][2 * l].elapsed_time(ev[t][1 + 2 * l]) for t in range(warm, wd.steps)
                             for l in range(wd.layers))
    attn_ms = statistics.mean(ev[t][1 + 2 * l].elapsed_time(ev[t][2 + 2 * l]) for t in range(warm, wd.steps)
                              for l in range(wd.layers))
    u = union_log[warm:].double()
    rows_bytes = wd.batch * wd.hq * e * 4  # one layer's stored rows, read once by the products (s <= 8)
    h.close()
    del rows, q_psum, q_sketch
    return {"workload": wd.name, "step_us": ms * 1e3, "steps_timed": timed,
            "union_blocks_per_unit": float(u.mean().item()),
            "kv_bytes_per_step": float(u.sum().item()) * wd.B * wd.d * 2 * 2 / timed,
            "stages_us_per_layer": {"exact_select": sel_ms * 1e3, "attention": attn_ms * 1e3},
            "rows_bytes_per_layer": rows_bytes,
            "select_stage_gbs_on_rows": rows_bytes / (sel_ms * 1e-3) / 1e9}


def bench_decode_exact(args, world, S, W, torch):
    """The exact decode walk (sws_decode_step_exact) against the log-domain walk
    (sws_decode_step) on one workload its shared-memory triangle holds: the
    decode workload's shape at a 16K-token prompt. Same caches, tokens and
    step count for both; each step is all layers' selection and attention."""
    wd = W.DECODE_128K.scaled(n0=16384, steps=max(4, min(16, args.decode_steps or 16)))
    cfg = S.make_config(wd.d, wd.B, wd.k, wd.s, 0, wd.density, wd.seed)
    h = S.Handle(cfg)
    path = S.DecodePath(h, wd.batch, wd.hq, wd.hkv, wd.max_len, wd.layers, exact=True)
    toks_k = torch.empty(wd.steps, wd.layers, wd.batch, wd.hkv, wd.d, dtype=torch.bfloat16, device="cuda")
    toks_v = torch.empty_like(toks_k)
    toks_q = torch.empty(wd.steps, wd.layers, wd.batch, wd.hq, wd.d, dtype=torch.bfloat16, device="cuda")
    lens = torch.full((wd.batch,), wd.n0, dtype=torch.int32, device="cuda")
    path.seq_lens.copy_(lens)
    for layer in range(wd.layers):
        qp = torch.empty(wd.batch, wd.hq, wd.max_len, wd.d, dtype=torch.bfloat16, device="cuda")
        for s_ in range(wd.batch):
            K, V = W.decode_cache_inputs(wd, s_, layer, "cuda")
            Q = W.decode_sequence_queries(wd, s_, layer, "cuda")
            path.write_cache(layer, s_, K, V, wd.n0)
            qp[s_] = Q
            toks_k[:, layer, s_] = K[:, wd.n0:].transpose(0, 1)
            toks_v[:, layer, s_] = V[:, wd.n0:].transpose(0, 1)
            toks_q[:, layer, s_] = Q[:, wd.n0:].transpose(0, 1)
            del K, V, Q
        path.init_queries(layer, qp)
        del qp
    stream = torch.cuda.current_stream()
    warm = min(3, wd.steps - 1)
    timed = wd.steps - warm
    out = {"workload": wd.name.replace("n131072", "n16384"), "steps_timed": timed}
    for mode in ("exact_walk", "log_walk"):
        path.exact = mode == "exact_walk"
        path.init_cache(lens)  # back to the prompt: the same steps replayed
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        unions = torch.zeros(wd.steps, wd.layers, wd.batch, wd.hkv, dtype=torch.int32, device="cuda")
        for t in range(wd.steps):
            if t == warm:
                barrier(world)
                torch.cuda.synchronize()
                a.record(stream)
            path.begin_step()
            for layer in range(wd.layers):
                path.layer(layer, toks_q[t, layer], toks_k[t, layer], toks_v[t, layer])
                unions[t, layer].copy_(path.sel_cnt, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize()
        assert S.sws_sync_check(h) == 0
        ms = max_over_ranks(a.elapsed_time(b), world) / timed
        out[mode] = {"step_us": ms * 1e3, "union_blocks_per_unit": float(unions[warm:].double().mean().item())}
    h.close()
    return out


def main():
    args = parse()
    world, rank, local = dist_setup()
    if args.impl == "reference":
        rc = run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return rc
    import torch
    import block_sparse_attention_sws_b200 as S
    import sws_inputs as W
    S.load()
    peaks, peak_kind = load_peaks()
    if args.no_prefill:
        # profiling run of the decode path alone: not a benchmark line
        out = {"profiling_only": True, "decode": bench_decode(args, world, S, W, torch, peaks)}
        if rank == 0:
            print(json.dumps(out), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
        return 0
    if args.profile_prefill:
        # profiling run of one prefill workload (for ncu captures): not a benchmark line
        wp = getattr(W, PROFILE_WORKLOADS[args.profile_workload])
        if args.prefill_n:
            wp = wp.scaled(name=f"prefill_n{args.prefill_n}_B{wp.B}_k{wp.k}_L{wp.layers}", n=args.prefill_n)
        px = bench_prefill(args, world, S, W, torch, wp, args.steps)
        if rank == 0:
            print(json.dumps({"profiling_only": True, "prefill": prefill_summary(px, world, peaks, peak_kind)}),
                  flush=True)
        return 0
    w = headline_workload(W)
    pf = bench_prefill(args, world, S, W, torch, w, args.steps)
    head = prefill_summary(pf, world, peaks, peak_kind)
    line = {
        "metric": METRIC, "value": head["tokens_per_s"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded AR(1) + sink + hub generator (sws_inputs); no datasets or weights",
        "config": head["config"], "stages_ms_per_step": head["stages_ms_per_step"], "roofline": head["roofline"],
        "sketch_roofline": head["sketch_roofline"], "attention_mma_work": head["attention_mma_work"],
        "clocks": head["clocks"], "gpu_launches": head["gpu_launches"],
    }
    if not args.no_e2e:
        line["e2e"] = bench_prefill_e2e(args, world, S, torch, pf)
    if not args.no_variants:
        line["headline_variants"] = {"scores_on_chip": bench_scores_on_chip(args, world, S, torch, pf)}
    pf["h"].close()
    del pf
    torch.cuda.empty_cache()
    line["prefill_workloads"] = {}
    for wx in extra_workloads(W):
        px = bench_prefill(args, world, S, W, torch, wx, max(3, min(args.steps, 20)))
        line["prefill_workloads"][wx.name] = prefill_summary(px, world, peaks, peak_kind)
        if wx is W.PREFILL_16K and not args.no_variants:
            line["variants"] = bench_prefill_variants(args, world, S, W, torch, px)
        px["h"].close()
        del px
        torch.cuda.empty_cache()
    if not args.no_decode:
        line["decode"] = bench_decode(args, world, S, W, torch, peaks)
        if not args.no_variants:
            torch.cuda.empty_cache()
            line["decode"].setdefault("variants", {})["exact_walk_n16384"] = bench_decode_exact(args, world, S, W,
                                                                                                 torch)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        s = json.dumps(line)
        print(s, flush=True)
        if args.json_out:
            with open(args.json_out, "w") as f:
                f.write(s + "\n")
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
