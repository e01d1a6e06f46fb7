"""mk_decode_step_noalloc against mk_decode_step.

The no-allocation entry point serves callers that cannot call cudaMalloc
while they step the model: a process whose device memory is all owned by
its own allocator, or a stepping loop that must not be synchronised by an
allocation.  It runs the same kernel with its scratch in the library's
static device array, so its results must be bit-identical to
mk_decode_step's.  Kept in a file of its own, collected last.
"""
import numpy as np
import pytest
import torch

import synth
from harness import gpu_model, tokens_at

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _t(a):
    return torch.as_tensor(np.asarray(a), dtype=torch.int32, device=DEV)


class Pair:
    """One model with two identical caches: one stepped by mk_decode_step,
    the other by mk_decode_step_noalloc."""

    def __init__(self, name, **over):
        self.mc = mc = synth.preset(name, gain_sigma=0.1, **over)
        self.m = gpu_model(mc)
        self.kv = {}
        for key in ("ref", "noalloc"):
            kv = self.m.kv_cache(8, mc.max_ctx)
            kv.fill_random(synth.SEED_KV, mc.kv_sigma, 40)
            self.kv[key] = kv
        self.step_no = 0

    def step_and_compare(self, B):
        from persistent_decode_megakernel_sm_b200 import mk
        mc, m = self.mc, self.m
        pp = [40 - 4 * s + self.step_no for s in range(B)]
        toks = _t([int(tokens_at(mc, s, [pp[s]])[0]) for s in range(B)])
        out = {}
        for key, fn in (("ref", mk.mk_decode_step), ("noalloc", mk.mk_decode_step_noalloc)):
            lg = torch.empty((B, mc.vocab), dtype=torch.float32, device=DEV)
            am = torch.empty(B, dtype=torch.int32, device=DEV)
            fn(m.h, toks, _t(pp), B, self.kv[key].h, lg, am)
            torch.cuda.synchronize()
            assert m.sync_status() == 0
            out[key] = (lg.cpu().numpy(), am.cpu().numpy())
        self.step_no += 1
        assert np.array_equal(out["noalloc"][0], out["ref"][0]), (mc.name, B)
        assert np.array_equal(out["noalloc"][1], out["ref"][1]), (mc.name, B)

    def close(self):
        for kv in self.kv.values():
            kv.close()
        self.m.close()


# a dense model whose projections have more row tiles than CTAs, with a
# remainder (160 row tiles: some CTAs take one more)
MID = dict(layers=2, hidden=2560, n_q_heads=20, n_kv_heads=4, head_dim=128, ffn=6912, vocab=8192, max_ctx=600)


@pytest.mark.parametrize("name,B,over", [("tiny", 3, {}), ("tiny_moe", 8, {}), ("tiny", 3, MID)],
                         ids=["tiny", "tiny_moe", "mid_dense"])
def test_noalloc_matches_decode_step_two_calls(name, B, over):
    """Two calls in a row on one handle and batch size: bit-identical logits
    and greedy tokens to mk_decode_step."""
    p = Pair(name, **over)
    p.step_and_compare(B)
    p.step_and_compare(B)
    p.close()


def test_noalloc_alternating_handles_and_batch_sizes():
    """Calls that alternate between two handles and between batch sizes on
    one handle: each call installs its own task list in the shared array
    when another handle or batch size used it last, and still matches
    mk_decode_step bit for bit."""
    a, b = Pair("tiny"), Pair("tiny_moe")
    for p, B in ((a, 3), (b, 8), (a, 3), (a, 1), (b, 2), (a, 3), (b, 2)):
        p.step_and_compare(B)
    a.close()
    b.close()


def test_noalloc_rejects_scratch_beyond_the_static_array():
    """A shape whose per-step scratch is larger than MK_NOALLOC_SCRATCH_BYTES
    (16 MiB) is refused before anything is launched."""
    from persistent_decode_megakernel_sm_b200 import mk
    # FFN width 2^19: its fp32 SwiGLU activations for 8 rows alone fill 16 MiB
    mc = synth.preset("tiny", ffn=1 << 19, layers=1)
    m = gpu_model(mc)
    kv = m.kv_cache(1, mc.max_ctx)
    lg = torch.empty((1, mc.vocab), dtype=torch.float32, device=DEV)
    am = torch.empty(1, dtype=torch.int32, device=DEV)
    with pytest.raises(mk.MkError) as e:
        mk.mk_decode_step_noalloc(m.h, _t([1]), _t([0]), 1, kv.h, lg, am)
    assert e.value.code == mk.MK_ERR_INVALID
    assert "static array" in mk.mk_last_error(m.h)
    kv.close()
    m.close()
