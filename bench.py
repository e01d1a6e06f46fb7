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
    ap.add_argument("--sweep", default="1,2,4,8", help="batch sizes timed for the by_batch table ('' = none)")
    ap.add_argument("--workloads", default="tiny,moe,verify,mla_fp8",
                    help="other workloads of the study timed after the headline ('' = none)")
    ap.add_argument("--verify-steps", type=int, default=256)
    ap.add_argument("--sweep-steps", type=int, default=64,
                    help="timed steps of each other batch size and workload (the study's configs use 64)")
    ap.add_argument("--oracle-steps", type=int, default=3,
                    help="full-depth oracle steps timed for cpu_baseline")
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per launch of the kernel from an ncu capture of the current kernel sources (null if none)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=16)
    return ap.parse_args()


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of the ranks' values, on every rank (the job's time is its
    slowest rank's); x itself when there is one rank."""
    if world <= 1:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Whole-job throughput: the units all ranks processed (each rank the same
    number, weak scaling) per second of the slowest rank's time."""
    return world * units_per_rank / (ms / 1e3)


def recorded_traffic(config: str, B: int):
    """DRAM bytes per launch recorded from an ncu capture under profiles/,
    valid only while the kernel sources are the ones it was taken on (the
    summary carries their hash); None otherwise."""
    import glob
    import hashlib
    import re
    h = hashlib.sha256()
    for f in ("mk_kernel.cu", "mk_host.cu", "mk_internal.h"):
        with open(os.path.join(ROOT, "persistent_decode_megakernel_sm_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    sha = h.hexdigest()[:16]
    pat = re.compile(r"traffic_bytes_per_launch: ([0-9.eE+]+); case: (\S+) B=(\d+) .*sources_sha256_16: (\w+)")
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        with open(path) as fh:
            for line in fh:
                m = pat.search(line)
                if m and m.group(2) == config and int(m.group(3)) == B and m.group(4) == sha:
                    return float(m.group(1))
    return None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class Clocks:
    def __init__(self, index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        self.start = 0
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={index}", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                       "-lms", "50"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None
            return
        # the sampler takes a moment to start: wait for its first sample (it
        # is started before the warm-up steps, so that it runs through them)
        t0 = time.time()
        while time.time() - t0 < 3.0 and self.p.poll() is None:
            if os.path.getsize(self.f.name) > 0:
                break
            time.sleep(0.01)

    def mark(self):
        """Start of the timed region: only the samples written after this count."""
        if self.p is not None:
            self.start = os.path.getsize(self.f.name)

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        self.p.wait()
        self.f.seek(self.start)
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
    from persistent_decode_megakernel_sm_b200.traffic import router_unions, step_bytes

    torch.cuda.set_device(local_rank)
    dev = f"cuda:{local_rank}"
    stream = torch.cuda.current_stream()
    peak, peak_kind = measured_peaks()

    prefill_s = {}

    def load(config):
        """The workload's model (seeded weights) and a cache of 8 sequences
        whose context is sequence 0's seeded prompt run through the model on
        the GPU (mk_prefill, 8 positions per launch), copied to the other
        sequences.  Returns the model, the cache and a function that puts the
        cache back to that context."""
        mc = synth.preset(config)
        model = Megakernel(mc, device=local_rank, max_batch=8)
        model.init_random(mc.seed, mc.w_sigma, mc.router_sigma, mc.gain_sigma, mc.fp8_block_base)
        kv = model.kv_cache(8, mc.max_ctx)
        prompt = torch.tensor(synth.seq_tokens(synth.SEED_TOKENS, 0, range(mc.context), mc.vocab), dtype=torch.int32,
                              device=dev)
        t0 = time.perf_counter()
        model.prefill(prompt, 0, 0, kv, stream=stream)
        torch.cuda.synchronize()
        prefill_s[config] = time.perf_counter() - t0
        assert model.sync_status() == 0, "device error in the prefill"
        snap = kv.copy_out()
        if mc.mla:
            v = snap.view(mc.layers, 8, -1)
            v[:, 1:] = v[:, :1]
        else:
            v = snap.view(2, mc.layers, 8, -1)
            v[:, :, 1:] = v[:, :, :1]
        kv.copy_in(snap)

        def restore():
            kv.copy_in(snap)

        return mc, model, kv, restore

    def decode_run(mc, model, kv, restore, B, steps, warmup, clocks=False):
        """Greedy decode of B sequences from the synthetic context: `warmup`
        untimed steps, then `steps` steps timed with CUDA events on the
        launching stream.  For MoE models the same steps are replayed
        afterwards (same cache state, same tokens) with the router trace on,
        to count the experts each timed step had to read."""
        total = warmup + steps
        assert mc.context + total <= mc.max_ctx
        pos = torch.tensor([[mc.context + i] * B for i in range(total)], dtype=torch.int32, device=dev)
        toks = torch.tensor(synth.tokens(synth.SEED_TOKENS, B, mc.vocab), dtype=torch.int32, device=dev)
        am = [torch.zeros(B, dtype=torch.int32, device=dev) for _ in range(total)]
        logits = torch.empty((B, mc.vocab), dtype=torch.float32, device=dev)
        restore()
        ck = Clocks(local_rank) if clocks else None
        cur = toks
        for i in range(warmup):
            model.decode_step(cur, pos[i], kv, logits, am[i], stream)
            cur = am[i]
        torch.cuda.synchronize()
        assert model.sync_status() == 0, "device error during warm-up"
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        if ck:
            ck.mark()
        ev[0].record(stream)
        for i in range(steps):
            model.decode_step(cur, pos[warmup + i], kv, logits, am[warmup + i], stream)
            cur = am[warmup + i]
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        clk = ck.stop() if ck else None
        assert model.sync_status() == 0, "device error in the timed region"
        per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
        ms = max_over_ranks(ev[0].elapsed_time(ev[steps]), world, dev)
        unions = None
        if mc.n_routed:
            restore()
            idx = torch.zeros((mc.layers, B, mc.top_k), dtype=torch.int32, device=dev)
            w = torch.zeros((mc.layers, B, mc.top_k), dtype=torch.float32, device=dev)
            unions = []
            cur = toks
            for i in range(total):
                model.set_router_trace(idx, w)
                model.decode_step(cur, pos[i], kv, logits, am[i], stream)
                model.set_router_trace(None, None)
                cur = am[i]
                if i >= warmup:
                    unions.append(router_unions(mc, idx))
        nbytes = [step_bytes(mc, [mc.context + warmup + i] * B, 1, unions[i] if unions else None)
                  for i in range(steps)]
        mean_bytes = statistics.mean(nbytes)
        launch_ms = statistics.mean(per)
        gbs = mean_bytes / (launch_ms / 1e3) / 1e9
        out = {"tokens_per_s": job_rate(B * steps, world, ms), "ms_per_step": ms / steps,
               "bytes_per_step": mean_bytes, "hbm_gbs": gbs, "frac_of_measured": gbs / peak, "frac_of_8tbs": gbs / 8000.0}
        if unions:
            out["routed_experts_per_layer_mean"] = statistics.mean(statistics.mean(u) for u in unions)
        return out, ms, per, clk, mean_bytes

    def verify_run(mc, model, kv, restore, steps, warmup):
        """Speculative verify on one sequence: each step checks an anchor and
        7 seeded uniform proposals at position P over the synthetic context;
        the next anchor is the greedy token after the accepted prefix and P
        advances by accepted + 1 (rewound to the context end when the cache
        would overflow).  Device time per launch from CUDA events."""
        def one_pass(record_unions):
            restore()
            anchor = int(synth.tokens(synth.SEED_TOKENS, 1, mc.vocab)[0])
            P = mc.context
            am = torch.zeros(8, dtype=torch.int32, device=dev)
            acc = torch.zeros(1, dtype=torch.int32, device=dev)
            idx = torch.zeros((mc.layers, 8, mc.top_k), dtype=torch.int32, device=dev)
            w = torch.zeros((mc.layers, 8, mc.top_k), dtype=torch.float32, device=dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            times, accepted, unions, starts = [], [], [], []
            for i in range(warmup + steps):
                props = synth.proposals(synth.SEED_PROPOSALS, i, 7, mc.vocab)
                toks = torch.tensor([anchor] + [int(x) for x in props], dtype=torch.int32, device=dev)
                if record_unions:
                    model.set_router_trace(idx, w)
                e0.record(stream)
                model.verify(toks, P, kv, None, am, acc, stream)
                e1.record(stream)
                torch.cuda.synchronize()
                if record_unions:
                    model.set_router_trace(None, None)
                a = int(acc.item())
                if i >= warmup:
                    times.append(e0.elapsed_time(e1))
                    accepted.append(a)
                    starts.append(P)
                    if record_unions:
                        unions.append(router_unions(mc, idx))
                anchor = int(am[a].item())
                P += a + 1
                if P + 8 > mc.max_ctx:
                    P = mc.context
            assert model.sync_status() == 0
            return times, accepted, unions, starts

        times, accepted, _, starts = one_pass(False)
        _, acc2, unions, _ = one_pass(True)
        assert acc2 == accepted, "verify replay diverged"
        nbytes = [step_bytes(mc, [starts[i]], 8, unions[i], write_logits=False) for i in range(steps)]
        ms = statistics.mean(times)
        gbs = statistics.mean(nbytes) / (ms / 1e3) / 1e9
        hist = {}
        for a in accepted:
            hist[str(a)] = hist.get(str(a), 0) + 1
        return {"verify_steps": steps, "ms_per_verify_step": ms, "accepted_hist": hist,
                "emitted_tokens_per_s": sum(a + 1 for a in accepted) / (sum(times) / 1e3),
                "bytes_per_step": statistics.mean(nbytes), "hbm_gbs": gbs, "frac_of_measured": gbs / peak,
                "frac_of_8tbs": gbs / 8000.0,
                "routed_experts_per_layer_mean": statistics.mean(statistics.mean(u) for u in unions),
                "proposals": "seeded uniform over the vocabulary"}

    def tiny_latency():
        """The small dense workload: 128 positions prefilled from seeded
        tokens, then 16 greedy steps at B = 1, each timed alone (CUDA events
        around each launch): step latency, no roofline claim (the model is
        resident in L2)."""
        tmc, tm, tkv, trestore = load("tiny")
        n = 16
        tok = torch.tensor(synth.seq_tokens(synth.SEED_TOKENS, 0, [tmc.context], tmc.vocab), dtype=torch.int32,
                           device=dev)
        ams = [torch.zeros(1, dtype=torch.int32, device=dev) for _ in range(n)]
        times = []
        for rep in range(2):  # the first pass warms up, the second is timed
            trestore()
            cur = tok
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * n)]
            for i in range(n):
                pos = torch.full((1,), tmc.context + i, dtype=torch.int32, device=dev)
                ev[2 * i].record(stream)
                tm.decode_step(cur, pos, tkv, None, ams[i], stream)
                ev[2 * i + 1].record(stream)
                cur = ams[i]
            torch.cuda.synchronize()
            times = [ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(n)]
        assert tm.sync_status() == 0
        tkv.close()
        tm.close()
        return {"greedy_steps": n, "ms_per_step_mean": statistics.mean(times), "ms_per_step_median": statistics.median(times),
                "ms_per_step_max": max(times), "tokens_per_s": 1e3 / statistics.mean(times),
                "note": "latency only: the 6 MB model is L2-resident, no roofline claim"}

    def step_times(mc, model, kv, restore, B, steps, warmup, multikernel):
        """Greedy decode of B sequences from the context: mean device time per
        step (CUDA events on the launching stream) of the single persistent
        kernel or of the multi-kernel comparison path (one kernel per phase in
        a CUDA graph with programmatic dependent launch)."""
        fn = model.decode_step_multikernel if multikernel else model.decode_step
        total = warmup + steps
        pos = torch.tensor([[mc.context + i] * B for i in range(total)], dtype=torch.int32, device=dev)
        am = [torch.zeros(B, dtype=torch.int32, device=dev) for _ in range(total)]
        restore()
        cur = torch.tensor(synth.tokens(synth.SEED_TOKENS, B, mc.vocab), dtype=torch.int32, device=dev)
        for i in range(warmup):
            fn(cur, pos[i], kv, None, am[i], stream)
            cur = am[i]
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(warmup, total):
            fn(cur, pos[i], kv, None, am[i], stream)
            cur = am[i]
        e1.record(stream)
        torch.cuda.synchronize()
        assert model.sync_status() == 0
        return e0.elapsed_time(e1) / steps, [int(a[0].item()) for a in am]

    def compare_multikernel(mc, model, kv, restore, batches=(1, 8), steps=32):
        out = {}
        for b in batches:
            one, t1 = step_times(mc, model, kv, restore, b, steps, 4, False)
            multi, t2 = step_times(mc, model, kv, restore, b, steps, 4, True)
            out[str(b)] = {"megakernel_ms_per_step": one, "multikernel_ms_per_step": multi,
                           "megakernel_speedup": multi / one, "same_tokens": t1 == t2}
        return out

    def spec_run(mc, model, kv, restore, n_out=64, targets=(3, 6)):
        """Speculative greedy generation (mk_spec_generate) on one sequence
        from the end of the context, with a synthetic draft that proposes the
        plain greedy chain (computed first by mk_decode_step) and corrupts
        each proposal with a seeded probability chosen so that the mean
        acceptance length (tokens emitted per verify launch) is the target.
        Each run is timed with CUDA events around the whole call (it reads
        every launch's accepted count on the host before the next launch)."""
        import random
        P = mc.context
        anchor = int(synth.seq_tokens(synth.SEED_TOKENS, 0, [P], mc.vocab)[0])
        restore()
        chain = []
        am = torch.zeros(1, dtype=torch.int32, device=dev)
        cur = torch.tensor([anchor], dtype=torch.int32, device=dev)
        for j in range(n_out + 8):
            model.decode_step(cur, torch.tensor([P + j], dtype=torch.int32, device=dev), kv, None, am, stream)
            cur = am.clone()
            chain.append(cur)
        chain = [int(x.item()) for x in chain]

        def err_for(length):
            # sum_{j=1..7} q^j = length - 1 (the mean of accepted + 1), q = 1 - err
            lo, hi = 0.0, 1.0
            for _ in range(60):
                q = (lo + hi) / 2
                if sum(q ** j for j in range(1, 8)) < length - 1:
                    lo = q
                else:
                    hi = q
            return 1.0 - lo

        out = {}
        for target in targets:
            err = err_for(target)
            rng = random.Random(1000 + target)

            def draft(history, max_k):
                e = len(history) - 1
                props = []
                for j in range(e, min(e + max_k, len(chain))):
                    t = chain[j]
                    if rng.random() < err:
                        t = (t + 1 + rng.randrange(mc.vocab - 1)) % mc.vocab
                    props.append(t)
                return props

            restore()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            toks, st = model.spec_generate(kv, anchor, P, n_out, draft, stream)
            e1.record(stream)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            out[f"acceptance_{target}"] = {
                "per_proposal_error": err, "emitted": st["emitted"], "launches": st["launches"],
                "acceptance_length_mean": st["emitted"] / st["launches"],
                "emitted_tokens_per_s": st["emitted"] / (ms / 1e3), "ms_per_launch": ms / st["launches"],
                "matches_plain_greedy": toks == chain[:n_out]}
        assert model.sync_status() == 0
        return out

    # ---- the headline workload ----
    mc, model, kv, restore = load(args.config)
    ctas, smem, threads = model.launch_info()
    B = args.batch
    head, ms, per, clk, abytes = decode_run(mc, model, kv, restore, B, args.steps, args.warmup, clocks=True)
    ms_step = ms / args.steps
    value = head["tokens_per_s"]
    launch_ms = statistics.mean(per)
    achieved = abytes / (launch_ms / 1e3) / 1e9

    multikernel = {args.config: compare_multikernel(mc, model, kv, restore)}

    # every timed run stays inside the cache: context + warm-up + steps <= max_ctx
    sweep_steps = min(args.sweep_steps, mc.max_ctx - mc.context - 3)
    by_batch = {str(B): head}
    for b in [int(x) for x in args.sweep.split(",") if x]:
        if b != B:
            by_batch[str(b)] = decode_run(mc, model, kv, restore, b, sweep_steps, 3)[0]

    # ---- end to end through the public API with host buffers ----
    restore()
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
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    assert model.sync_status() == 0
    e2e = {"value": job_rate(B * E, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": 2 * B * 4,
           "d2h_bytes_per_step": B * 4}
    kv.close()
    model.close()

    # ---- the other workloads of the study (one GPU each, rank-local) ----
    workloads = {}
    cur_base, cur = None, None
    for name in [w for w in args.workloads.split(",") if w]:
        if name == "tiny":
            workloads["tiny"] = tiny_latency()
            continue
        base = "moe" if name == "verify" else name
        if base != cur_base:
            if cur:  # one model on the device at a time
                cur[2].close()
                cur[1].close()
            cur, cur_base = load(base), base
        wmc, wm, wkv, wrestore = cur
        if name == "verify":
            workloads["verify_moe"] = verify_run(wmc, wm, wkv, wrestore, args.verify_steps, 4)
            workloads["spec_moe"] = spec_run(wmc, wm, wkv, wrestore)
        else:
            batches = (1, 2, 4, 8) if name == "moe" else (1, 8)
            steps_w = min(args.sweep_steps, wmc.max_ctx - wmc.context - 3)
            workloads[name] = {str(b): decode_run(wmc, wm, wkv, wrestore, b, steps_w, 3)[0] for b in batches}
            if name == "moe":
                multikernel["moe"] = compare_multikernel(wmc, wm, wkv, wrestore)
    if cur:
        cur[2].close()
        cur[1].close()

    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded random-init weights; context = a seeded prompt prefilled through the model)",
        "config": {"workload": f"{args.config} decode, B={B}, context {mc.context} (+ positions advancing)",
                   "model": args.config, "global_batch": B * world, "seq_len": mc.context, "parallelism": f"dp{world}",
                   "l2": "inputs larger than L2 (44 GB weights), no flush",
                   "context": "sequence 0's seeded prompt run through the model on the GPU, copied to the other sequences",
                   "prefill_s": prefill_s, "sweep_steps": sweep_steps},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": peak_kind,
                     "traffic": args.traffic if args.traffic is not None else recorded_traffic(args.config, B),
                     "frac_of_8tbs": achieved / 8000.0, "algorithmic_bytes_per_launch": abytes},
        "by_batch": by_batch,
        "workloads": workloads,
        "multikernel_comparison": multikernel,
        "e2e": e2e,
        "gpu_launches": args.steps,
        "launch": {"ctas": ctas, "threads": threads, "smem_bytes": smem},
        "clocks": clk,
    }
    return res


def oracle_steps(config: str, steps: int, warmup: int = 0):
    """Time the fp64 oracle (as it stands) on the host cores: `warmup`
    untimed, then `steps` timed full-depth B=1 decode steps of the workload
    (every layer, the LM head and the greedy argmax) at consecutive
    positions past a seeded synthetic context (the oracle's own fill: its
    prefill of thousands of positions would take hours, and the step's cost
    does not depend on the context's values).  Returns the seconds of each
    timed step."""
    import oracle
    import synth
    mc = synth.preset(config)
    om = oracle.OracleModel(mc.replace(max_seqs=1))
    om.kv_fill_synthetic(synth.SEED_KV, mc.context)
    tok = [int(synth.seq_tokens(synth.SEED_TOKENS, 0, [mc.context], mc.vocab)[0])]
    times = []
    for i in range(warmup + steps):
        t0 = time.perf_counter()
        r = om.step(tok, [mc.context + (i % 64)], want_logits=False, absorbed=mc.mla)
        dt = time.perf_counter() - t0
        tok = [int(r["argmax"][0])]
        if i >= warmup:
            times.append(dt)
    om.close()
    return times


def cpu_baseline(config: str, steps: int = 3):
    """The oracle timed over `steps` full-depth steps of the headline workload."""
    import oracle
    times = oracle_steps(config, steps)
    mean = statistics.mean(times)
    return {"value": 1.0 / mean, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{steps} full-depth B=1 decode steps of {config} (every layer, LM head, argmax) on a seeded "
                      f"synthetic context, timed one by one: mean {mean:.2f} s per step",
            "step_s": times}


def run_reference(args):
    """The reference arm: the fp64 CPU oracle on the host cores, W untimed
    and K timed full-depth B=1 decode steps of the headline workload (each
    step the whole model, as the GPU arm's)."""
    import oracle
    import synth
    mc = synth.preset(args.config)
    times = oracle_steps(args.config, args.steps, args.warmup)
    ms = 1e3 * statistics.mean(times)
    value = 1e3 / ms
    cpu = {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
           "sample": f"{args.steps} full-depth B=1 decode steps of {args.config} after {args.warmup} untimed ones "
                     f"(every layer, LM head, argmax), seeded synthetic context, timed one by one",
           "step_s": times}
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.config} decode, B=1, context {mc.context} (+ positions advancing)",
                   "model": args.config, "global_batch": 1, "seq_len": mc.context,
                   "parallelism": "none (host cores)",
                   "context": "a seeded synthetic cache (the oracle's own fill; the step's cost does not depend on "
                              "the cached values)"},
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
        res["cpu_baseline"] = cpu_baseline(args.config, args.oracle_steps)
    if world > 1:
        import torch
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
