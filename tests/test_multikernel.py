"""The multi-kernel comparison path (mk_decode_step_multikernel: one kernel
per phase of the step, recorded as a CUDA graph with programmatic dependent
launch) runs the persistent kernel's tasks one phase per launch, so its
logits and greedy tokens must be bit-identical to mk_decode_step's on the same
inputs; the persistent kernel itself is pinned to the oracle by the parity
tests.  Two steps in a row on identical caches, several batch sizes, every
model family, and the full per-layer sizes of the dense and MoE workloads."""
import numpy as np
import pytest
import torch

import synth
from harness import gpu_model, tokens_at

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _t(a):
    return torch.as_tensor(np.asarray(a), dtype=torch.int32, device=DEV)


def _both(mc, batches, steps=2, context=None):
    m = gpu_model(mc)
    ctx = mc.context if context is None else context
    kvs = [m.kv_cache(8, mc.max_ctx) for _ in range(2)]
    for B in batches:
        for kv in kvs:
            kv.fill_random(synth.SEED_KV, mc.kv_sigma, ctx)
        pos = [ctx - 3 * s for s in range(B)]
        for step in range(steps):
            pp = [p + step for p in pos]
            toks = _t([int(tokens_at(mc, s, [pp[s]])[0]) for s in range(B)])
            out = []
            for kv, fn in ((kvs[0], m.decode_step), (kvs[1], m.decode_step_multikernel)):
                lg = torch.empty((B, mc.vocab), dtype=torch.float32, device=DEV)
                am = torch.empty(B, dtype=torch.int32, device=DEV)
                fn(toks, _t(pp), kv, lg, am)
                torch.cuda.synchronize()
                assert m.sync_status() == 0
                out.append((lg.cpu().numpy(), am.cpu().numpy()))
            assert np.array_equal(out[0][0], out[1][0]), (mc.name, B, step)
            assert np.array_equal(out[0][1], out[1][1]), (mc.name, B, step)
        # the caches both paths wrote are identical too
        assert torch.equal(kvs[0].copy_out(), kvs[1].copy_out()), (mc.name, B)
    for kv in kvs:
        kv.close()
    m.close()


@pytest.mark.parametrize("name", ["tiny", "tiny_moe", "tiny_mla"])
def test_multikernel_bit_identical_small(name):
    _both(synth.preset(name, gain_sigma=0.1), (1, 3, 8))


@pytest.mark.parametrize("name", ["dense27b", "moe"])
def test_multikernel_bit_identical_full_layer_sizes(name):
    """Every per-layer shape of the workload, two layers."""
    _both(synth.preset(name, layers=2, gain_sigma=0.1), (1, 8), steps=1)
