"""Run a few decode steps of a workload (optionally cut to fewer layers or a
smaller vocabulary) for an external profiler: seeded weights and context,
`warmup` steps, then `steps` more, all through the C ABI.

    python -m persistent_decode_megakernel_sm_b200.profile_step --config dense27b --layers 2 --vocab 32768

A cut keeps every per-layer shape of the workload, so the kernel's per-layer
behaviour (tiles, chunks, attention splits) is the full model's; only the
number of layers and the LM head / embedding rows shrink.  Prints the bytes
the step must move (weights, cache rows, logits) for the cut.  For MoE models
the weight figure counts every resident expert, an upper bound: a step reads
only the shared experts and the routed experts its rows pick."""
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
    for i in range(a.warmup + a.steps):
        if a.verify:
            props = synth.proposals(synth.SEED_PROPOSALS, i, 7, mc.vocab)
            toks8 = torch.tensor([int(tok[0].item())] + [int(x) for x in props], dtype=torch.int32, device=dev)
            m.verify(toks8, mc.context, kv, lg, am, acc)
        else:
            pos = torch.full((B,), mc.context + i, dtype=torch.int32, device=dev)
            m.decode_step(tok, pos, kv, lg, am)
            tok = am.clone()
    torch.cuda.synchronize()
    assert m.sync_status() == 0
    weights = m.weight_bytes() - mc.vocab * mc.hidden * 2 + B * mc.hidden * 2
    kvt = (mc.kv_lora_rank + mc.rope_dim) * 2 if mc.mla else 2 * mc.n_kv_heads * mc.head_dim * 2
    cache = (mc.context * kvt * mc.layers + 8 * kvt * mc.layers if a.verify
             else B * (mc.context + a.warmup) * kvt * mc.layers + B * kvt * mc.layers)
    key = "weight_bytes_resident_upper_bound" if mc.n_routed else "weight_bytes_streamed"
    print(json.dumps({"config": a.config, "layers": mc.layers, "vocab": mc.vocab, "batch": B,
                      key: weights, "cache_bytes": cache, "logit_bytes": B * mc.vocab * 4,
                      "bytes_per_step_first_profiled": weights + cache + B * mc.vocab * 4}))
    kv.close()
    m.close()


if __name__ == "__main__":
    main()
