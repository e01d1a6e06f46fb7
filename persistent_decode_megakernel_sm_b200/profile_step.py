"""Run a few decode steps of a workload (optionally cut to fewer layers or a
smaller vocabulary) for an external profiler: seeded weights and context,
`warmup` steps, then `steps` more, all through the C ABI.

    python -m persistent_decode_megakernel_sm_b200.profile_step --config dense27b --layers 2 --vocab 32768

A cut keeps every per-layer shape of the workload, so the kernel's per-layer
behaviour (tiles, chunks, attention splits) is the full model's; only the
number of layers and the LM head / embedding rows shrink.  Prints the bytes
the last step must move (weights, cache rows, logits) for the cut, counted
as the benchmark counts them: for MoE models the routed experts are those the
last step's rows picked (a router trace of that step)."""
from __future__ import annotations

import argparse
import json
import os
import sys


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="dense27b")
    ap.add_argument("--layers", type=int, default=0, help="0 = the workload's own depth")
    ap.add_argument("--vocab", type=int, default=0, help="0 = the workload's own vocabulary")
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--verify", action="store_true",
                    help="launch verify steps (1 anchor + 7 seeded proposals on sequence 0) instead of decode steps")
    a = ap.parse_args()
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch
    import synth
    from persistent_decode_megakernel_sm_b200 import Megakernel
    from persistent_decode_megakernel_sm_b200.traffic import router_unions, step_bytes

    mc = synth.preset(a.config)
    if a.layers:
        mc = mc.replace(layers=a.layers)
    if a.vocab:
        mc = mc.replace(vocab=a.vocab)
    dev = "cuda:0"
    m = Megakernel(mc, 0)
    m.init_random(mc.seed, mc.w_sigma, mc.router_sigma, mc.gain_sigma, mc.fp8_block_base)
    kv = m.kv_cache(8, mc.max_ctx)
    kv.fill_random(synth.SEED_KV, mc.kv_sigma, mc.context)
    B = 8 if a.verify else a.batch
    tok = torch.tensor(synth.tokens(synth.SEED_TOKENS, B, mc.vocab), dtype=torch.int32, device=dev)
    lg = torch.empty((B, mc.vocab), dtype=torch.float32, device=dev)
    am = torch.empty(B, dtype=torch.int32, device=dev)
    acc = torch.empty(1, dtype=torch.int32, device=dev)
    n = a.warmup + a.steps
    k = max(mc.top_k, 1)
    idx = torch.full((mc.layers, B, k), -1, dtype=torch.int32, device=dev)
    wts = torch.zeros((mc.layers, B, k), dtype=torch.float32, device=dev)
    pos0 = None
    for i in range(n):
        last = i == n - 1
        if last and mc.n_routed:
            m.set_router_trace(idx, wts)
        if a.verify:
            props = synth.proposals(synth.SEED_PROPOSALS, i, 7, mc.vocab)
            toks8 = torch.tensor([int(tok[0].item())] + [int(x) for x in props], dtype=torch.int32, device=dev)
            m.verify(toks8, mc.context, kv, lg, am, acc)
            pos0 = [mc.context]
        else:
            pos = torch.full((B,), mc.context + i, dtype=torch.int32, device=dev)
            m.decode_step(tok, pos, kv, lg, am)
            tok = am.clone()
            pos0 = [mc.context + i] * B
        if last and mc.n_routed:
            m.set_router_trace(None, None)
    torch.cuda.synchronize()
    assert m.sync_status() == 0
    Q = 8 if a.verify else 1
    unions = router_unions(mc, idx) if mc.n_routed else None
    out = {"config": a.config, "layers": mc.layers, "vocab": mc.vocab, "batch": B,
           "launches": n, "algorithmic_bytes_last_step": step_bytes(mc, pos0, Q, unions, write_logits=True)}
    if unions:
        out["routed_experts_per_layer_last_step"] = unions
    print(json.dumps(out))
    kv.close()
    m.close()


if __name__ == "__main__":
    main()
