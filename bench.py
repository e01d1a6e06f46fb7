#!/usr/bin/env python3
"""Decode-step benchmark of the B200 persistent megakernel.

Workload: the dense 27B-shaped decoder (64 layers, hidden 5120, 40/8 heads x
128, SwiGLU 17408, vocab 151936, bf16 random-init weights) with a 2048-token
synthetic KV context, greedy decode, batch B (default 1).  A step is one
launch of the megakernel: every layer's attention and FFN, the LM head and
argmax for B sequences.  value = decode tokens/s over the whole job (all
ranks); one process per GPU runs an independent replica (the path does not
shard).  Weights (44 GB) and caches are far larger than L2, so no flush is
needed between steps.

  python bench.py [--gpus N --steps K --warmup W --batch B --config NAME]
  python bench.py --impl reference ...   # the fp64 CPU oracle on host cores
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tokens/s at B=1/8 on 1 B200; achieved HBM GB/s as % of 8 TB/s roofline"
UNIT = "tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--config", default="dense27b")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--sweep", default="1,8", help="extra batch sizes timed for the by_batch table ('' = none)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=16)
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# algorithmic bytes of one decode step (what the method must move)
# ---------------------------------------------------------------------------
def step_bytes(mc, B, positions, weight_bytes, write_logits=True):
    """All streamed weights (the embedding table only for the B rows used),
    the KV rows attended (positions 0..p per sequence, every layer), the KV
    rows written and the logits written."""
    embed_table = mc.vocab * mc.hidden * 2
    w = weight_bytes - embed_table + B * mc.hidden * 2
    kv_tok_layer = 2 * mc.n_kv_heads * mc.head_dim * 2
    kv_read = sum(int(p) for p in positions) * kv_tok_layer * mc.layers   # prefix 0..p-1 read from HBM
    kv_write = B * kv_tok_layer * mc.layers
    logits = B * mc.vocab * 4 if write_logits else 0
    return w + kv_read + kv_write + logits


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class Clocks:
    def __init__(self, index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={index}", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                       "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        self.p.wait()
        self.f.seek(0)
        sm, mx, reasons = [], None, set()
        for line in self.f:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, v in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"), parts[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args, rank, world, local_rank):
    import torch
    import synth
    from persistent_decode_megakernel_sm_b200 import Megakernel

    torch.cuda.set_device(local_rank)
    dev = f"cuda:{local_rank}"
    mc = synth.preset(args.config)
    Bmax = max([args.batch] + [int(b) for b in args.sweep.split(",") if b])
    model = Megakernel(mc, device=local_rank, max_batch=8)
    model.init_random(mc.seed, mc.w_sigma, mc.router_sigma, mc.gain_sigma, mc.fp8_block_base)
    kv = model.kv_cache(8, mc.max_ctx)
    kv.fill_random(synth.SEED_KV, mc.kv_sigma, mc.context)
    ctas, smem, threads = model.launch_info()
    stream = torch.cuda.current_stream()

    def time_batch(B, steps, warmup, clocks=False):
        total = warmup + steps
        assert mc.context + total <= mc.max_ctx
        pos = torch.tensor([[mc.context + i] * B for i in range(total)], dtype=torch.int32, device=dev)
        toks = torch.tensor(synth.tokens(synth.SEED_TOKENS, B, mc.vocab), dtype=torch.int32, device=dev)
        am = [torch.zeros(B, dtype=torch.int32, device=dev) for _ in range(2)]
        logits = torch.empty((B, mc.vocab), dtype=torch.float32, device=dev)
        cur = toks
        for i in range(warmup):
            model.decode_step(cur, pos[i], kv, logits, am[i & 1], stream)
            cur = am[i & 1]
        torch.cuda.synchronize()
        assert model.sync_status() == 0, "device error during warm-up"
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        ck = Clocks(local_rank) if clocks else None
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        ev[0].record(stream)
        for i in range(steps):
            model.decode_step(cur, pos[warmup + i], kv, logits, am[i & 1], stream)
            cur = am[i & 1]
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        clk = ck.stop() if ck else None
        assert model.sync_status() == 0, "device error in the timed region"
        per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
        ms = ev[0].elapsed_time(ev[steps])
        if world > 1:
            t = torch.tensor([ms], device=dev)
            torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
            ms = float(t.item())
        positions = [mc.context + warmup] * B
        return ms, per, clk, positions

    ms, per, clk, positions = time_batch(args.batch, args.steps, args.warmup, clocks=True)
    B = args.batch
    ms_step = ms / args.steps
    value = world * B * args.steps / (ms / 1e3)
    # roofline of the (only) kernel: algorithmic bytes / average launch time
    mid_pos = [p + args.steps // 2 for p in positions]
    abytes = step_bytes(mc, B, mid_pos, model.weight_bytes())
    peak, peak_kind = measured_peaks()
    launch_ms = statistics.mean(per)
    achieved = abytes / (launch_ms / 1e3) / 1e9

    by_batch = {}
    for b in [int(x) for x in args.sweep.split(",") if x]:
        if b == B:
            by_batch[str(b)] = {"tokens_per_s": world * b / (ms_step / 1e3), "ms_per_step": ms_step,
                                "hbm_gbs": achieved}
            continue
        kv.fill_random(synth.SEED_KV, mc.kv_sigma, mc.context)
        msb, perb, _, posb = time_batch(b, max(8, args.steps // 4), 3)
        stepb = msb / max(8, args.steps // 4)
        bb = step_bytes(mc, b, [p + 4 for p in posb], model.weight_bytes())
        by_batch[str(b)] = {"tokens_per_s": world * b / (stepb / 1e3), "ms_per_step": stepb,
                            "hbm_gbs": bb / (statistics.mean(perb) / 1e3) / 1e9}

    # ---- end to end through the public API with host buffers ----
    kv.fill_random(synth.SEED_KV, mc.kv_sigma, mc.context)
    E = args.e2e_steps
    h_tok = torch.tensor(synth.tokens(synth.SEED_TOKENS, B, mc.vocab), dtype=torch.int32).pin_memory()
    h_pos = torch.tensor([mc.context] * B, dtype=torch.int32).pin_memory()
    h_out = torch.empty(B, dtype=torch.int32).pin_memory()
    d_tok = torch.empty(B, dtype=torch.int32, device=dev)
    d_pos = torch.empty(B, dtype=torch.int32, device=dev)
    d_am = torch.empty(B, dtype=torch.int32, device=dev)
    for i in range(3):
        d_tok.copy_(h_tok, non_blocking=True)
        d_pos.copy_(h_pos + i, non_blocking=True)
        model.decode_step(d_tok, d_pos, kv, None, d_am, stream)
        h_out.copy_(d_am, non_blocking=True)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(E):
        h_pos.fill_(mc.context + 3 + i)
        d_tok.copy_(h_tok, non_blocking=True)
        d_pos.copy_(h_pos, non_blocking=True)
        model.decode_step(d_tok, d_pos, kv, None, d_am, stream)
        h_out.copy_(d_am, non_blocking=True)
        stream.synchronize()          # the host needs the token before the next step
        h_tok.copy_(h_out)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([e2e_ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        e2e_ms = float(t.item())
    assert model.sync_status() == 0
    e2e = {"value": world * B * E / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": 2 * B * 4,
           "d2h_bytes_per_step": B * 4}
    kv.close()
    model.close()
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded random-init weights, seeded synthetic KV context)",
        "config": {"workload": f"{args.config} decode, B={B}, context {mc.context} (+ positions advancing)",
                   "model": args.config, "global_batch": B * world, "seq_len": mc.context, "parallelism": f"dp{world}",
                   "l2": "inputs larger than L2 (44 GB weights), no flush"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": peak_kind, "traffic": None,
                     "frac_of_8tbs": achieved / 8000.0, "algorithmic_bytes_per_launch": abytes},
        "by_batch": by_batch,
        "e2e": e2e,
        "gpu_launches": args.steps,
        "launch": {"ctas": ctas, "threads": threads, "smem_bytes": smem},
        "clocks": clk,
    }
    return res


def cpu_baseline(config: str, sample_layers=(1, 4)):
    """Time the fp64 oracle (as it stands) on the host cores for one B=1
    decode step of the workload truncated to 1 and 4 layers (each the better
    of two runs, so thread start-up is not counted), and extrapolate the
    full-depth step linearly: head + L x layer."""
    import oracle
    import synth
    mc = synth.preset(config)
    times = {}
    for nl in sample_layers:
        m = mc.replace(layers=nl, max_seqs=1)
        om = oracle.OracleModel(m)
        om.kv_fill_synthetic(synth.SEED_KV, mc.context)
        tok = synth.tokens(synth.SEED_TOKENS, 1, mc.vocab)
        best = float("inf")
        for rep in range(2):
            t0 = time.perf_counter()
            om.step(tok, [mc.context + rep], want_logits=False)
            best = min(best, time.perf_counter() - t0)
        times[nl] = best
        om.close()
    lo, hi = sample_layers
    t_layer = max((times[hi] - times[lo]) / (hi - lo), 1e-6)
    t_head = max(times[lo] - lo * t_layer, 0.0)
    full = t_head + mc.layers * t_layer
    return {"value": 1.0 / full, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"one B=1 decode step of {config} truncated to {lo} and {hi} layers "
                      f"({times[lo]:.2f} s, {times[hi]:.2f} s, best of 2); full {mc.layers}-layer step "
                      f"extrapolated as head + {mc.layers} x layer = {full:.1f} s",
            "t_layer_s": t_layer, "t_head_s": t_head}


def run_reference(args):
    """The reference arm: the fp64 CPU oracle on the host cores.  Each step
    is a bounded sample - one B=1 decode step of the workload truncated to
    one layer - scaled to the full depth with the head/layer split measured
    by cpu_baseline (1- and 4-layer truncations)."""
    import oracle
    import synth
    mc = synth.preset(args.config)
    fit = cpu_baseline(args.config)
    t_layer, t_head = fit["t_layer_s"], fit["t_head_s"]
    m1 = mc.replace(layers=1, max_seqs=1)
    om = oracle.OracleModel(m1)
    om.kv_fill_synthetic(synth.SEED_KV, mc.context)
    tok = synth.tokens(synth.SEED_TOKENS, 1, mc.vocab)
    for i in range(min(args.warmup, 2)):
        om.step(tok, [mc.context + i], want_logits=False)
    full = []
    for i in range(args.steps):
        t0 = time.perf_counter()
        om.step(tok, [mc.context + (i % 8)], want_logits=False)
        t1 = time.perf_counter() - t0
        # this 1-layer step stands for head + L layers at the fitted ratio
        full.append(t1 * (t_head + mc.layers * t_layer) / (t_head + t_layer))
    om.close()
    ms = 1e3 * sum(full) / len(full)
    value = 1e3 / ms
    cpu = dict(fit)
    cpu["value"] = value
    cpu["sample"] = (f"{args.steps} decode steps of {args.config} truncated to 1 layer, each scaled to the full "
                     f"{mc.layers}-layer step by the measured head/layer split; " + fit["sample"])
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.config} decode, B=1, context {mc.context}", "model": args.config,
                   "global_batch": 1, "seq_len": mc.context, "parallelism": "none (host cores)"},
        "cpu_baseline": cpu,
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    res = run_ours(args, rank, world, local_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(args.config)
    if world > 1:
        import torch
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
