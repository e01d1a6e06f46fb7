"""Task trace of the decode megakernel (the in-kernel %globaltimer records
written when mk_set_trace is enabled) and its summary: per phase, the time
CTAs spend waiting on dependencies, on weight tiles and on activation slices,
and the SM idle fraction between tasks.

    python -m persistent_decode_megakernel_sm_b200.trace --config dense27b --batch 1
"""
from __future__ import annotations

import argparse
import collections
import json
import os
import sys

import numpy as np

TYPE_NAMES = {1: "gemv", 2: "attn", 3: "moe_gu", 4: "moe_down", 5: "prefetch", 6: "embed", 7: "mla", 8: "mla_comb"}
FIELDS = 20
EPI_NAMES = {0: "store", 1: "resid", 2: "swiglu", 3: "logits", 4: "swiglu_moe"}


def record(model, kv, tokens, positions, logits, argmax, cap: int = 1024):
    import torch
    ctas, _, _ = model.launch_info()
    buf = torch.zeros((ctas, cap, FIELDS), dtype=torch.int64, device=tokens.device)
    model.set_trace(buf, cap)
    model.decode_step(tokens, positions, kv, logits, argmax)
    torch.cuda.synchronize()
    model.set_trace(None, 0)
    return buf.cpu().numpy()


def summarize(tr: np.ndarray, sm_clock_mhz: float = 0.0) -> dict:
    """tr: [ctas][cap][20] = t_begin, t_dep, t_end (ns), wait_full, wait_x (cycles),
    chunks, layer (+ phase << 16), type*16+epi, then cycles in fragment prep, mma, epilogue,
    release, [12..15] producer statistics (record 0: cycles blocked on a full
    ring, chunks issued, first and last issue time; record 1: producer cycles
    and ns, giving the SM clock), then cycles in the chunk loop, before it,
    after it and signalling (consumer thread 0)."""
    if sm_clock_mhz <= 0:
        # measured: SM cycles / ns over each producer's lifetime (record 1)
        cyc, ns = tr[:, 1, 12].astype(np.float64), tr[:, 1, 13].astype(np.float64)
        ok = ns > 0
        sm_clock_mhz = float(np.median(cyc[ok] / ns[ok]) * 1e3) if ok.any() else 1965.0
    valid = tr[:, :, 2] > 0
    t0 = tr[:, :, 0][valid].min()
    t1 = tr[:, :, 2][valid].max()
    # a prefetch record is an L2 request the weight producer issued ahead of
    # a task (no consumer work, no phase of its own): counted, kept out of the
    # phases and of the CTAs' busy time
    work = valid & (tr[:, :, 7] // 16 != 5)
    phases = collections.defaultdict(lambda: dict(n=0, dep_us=0.0, run_us=0.0, wf_us=0.0, wx_us=0.0, chunks=0,
                                                  frag_us=0.0, mma_us=0.0, epi_us=0.0, rel_us=0.0,
                                                  loop_us=0.0, pre_us=0.0, post_us=0.0, sig_us=0.0))
    busy = 0.0
    # wall span of each phase (the tasks between two dependency points):
    # first dependency met to last task end
    span = collections.defaultdict(lambda: [None, None])
    for c in range(tr.shape[0]):
        for k in range(tr.shape[1]):
            if not work[c, k]:
                continue
            tb, td, te, wf, wx, ch, layer, te16 = tr[c, k, :8]
            fr, mm, ep, rl = tr[c, k, 8:12]
            lo, pr, po, sg = tr[c, k, 16:20]
            name = TYPE_NAMES.get(int(te16) // 16, "?") + ("/" + EPI_NAMES[int(te16) % 16] if int(te16) // 16 in (1, 3) else "")
            p = phases[name]
            phase = int(layer) >> 16
            layer = int(layer) & 0xFFFF
            sp = span[(phase, name)]
            sp[0] = int(td) if sp[0] is None else min(sp[0], int(td))
            sp[1] = int(te) if sp[1] is None else max(sp[1], int(te))
            p["n"] += 1
            p["dep_us"] += (td - tb) / 1e3
            p["run_us"] += (te - td) / 1e3
            p["wf_us"] += wf / sm_clock_mhz
            p["wx_us"] += wx / sm_clock_mhz
            p["chunks"] += int(ch)
            p["frag_us"] += fr / sm_clock_mhz
            p["mma_us"] += mm / sm_clock_mhz
            p["epi_us"] += ep / sm_clock_mhz
            p["rel_us"] += rl / sm_clock_mhz
            p["loop_us"] += lo / sm_clock_mhz
            p["pre_us"] += pr / sm_clock_mhz
            p["post_us"] += po / sm_clock_mhz
            p["sig_us"] += sg / sm_clock_mhz
            busy += (te - td) / 1e3 - wf / sm_clock_mhz - wx / sm_clock_mhz
    ctas = tr.shape[0]
    step_us = (t1 - t0) / 1e3
    out = {"step_us": step_us, "ctas": ctas, "sm_clock_mhz": sm_clock_mhz, "phases": {}}
    for name, p in sorted(phases.items()):
        out["phases"][name] = {k: (v / ctas if k.endswith("_us") else v) for k, v in p.items()}
        out["phases"][name]["per_cta_us_note"] = "times summed over the CTA's tasks, averaged over CTAs"
        # wall time: per phase, the first CTA's dependency met to the last
        # CTA's end, summed over the step's phases of this kind
        out["phases"][name]["wall_us"] = sum((e - b) / 1e3 for (ph, nm), (b, e) in span.items() if nm == name)
    out["compute_fraction"] = busy / ctas / step_us
    # SM idle between tasks: the part of the step a CTA spends outside task
    # bodies (waiting for a task's dependency, or done before the step ends)
    run_ns = np.where(work, tr[:, :, 2] - tr[:, :, 1], 0).sum(axis=1).astype(np.float64)
    idle = 1.0 - run_ns / float(t1 - t0)
    out["idle_between_tasks_fraction"] = float(idle.mean())
    out["idle_between_tasks_fraction_max_cta"] = float(idle.max())
    out["prefetch_requests"] = int((valid & ~work).sum())
    out["producer_blocked_us_per_cta"] = float(tr[:, 0, 12].mean()) / sm_clock_mhz
    out["producer_chunks_per_cta"] = float(tr[:, 0, 13].mean())
    out["producer_span_us"] = float((tr[:, 0, 15] - tr[:, 0, 14]).mean()) / 1e3
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="dense27b")
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--out", default=None)
    a = ap.parse_args()
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch
    import synth
    from persistent_decode_megakernel_sm_b200 import Megakernel
    mc = synth.preset(a.config)
    m = Megakernel(mc, 0)
    m.init_random(mc.seed, mc.w_sigma, mc.router_sigma, mc.gain_sigma, mc.fp8_block_base)
    kv = m.kv_cache(8, mc.max_ctx)
    kv.fill_random(synth.SEED_KV, mc.kv_sigma, mc.context)
    B = a.batch
    tok = torch.arange(B, dtype=torch.int32, device="cuda:0") + 7
    lg = torch.empty((B, mc.vocab), dtype=torch.float32, device="cuda:0")
    am = torch.empty(B, dtype=torch.int32, device="cuda:0")
    for i in range(a.steps):
        pos = torch.full((B,), mc.context + i, dtype=torch.int32, device="cuda:0")
        m.decode_step(tok, pos, kv, lg, am)
    pos = torch.full((B,), mc.context + a.steps, dtype=torch.int32, device="cuda:0")
    tr = record(m, kv, tok, pos, lg, am)
    assert m.sync_status() == 0
    s = summarize(tr)
    if a.out:
        np.savez_compressed(a.out, tr=tr)
    print(json.dumps(s, indent=1))


if __name__ == "__main__":
    main()
