"""mk_decode_step_noalloc against mk_decode_step.

The no-allocation entry point serves callers that cannot call cudaMalloc
while they step the model (their device memory is owned by their own
allocator, or the loop must not be synchronised by an allocation).  It runs
the same kernel with its scratch in the library's static device array; here
both entry points take two steps in a row on identical caches and must agree
within the decode-step tolerance.  Kept in a file of its own, collected last.
"""
import numpy as np
import pytest
import torch

import synth
from harness import gpu_model, logits_close, tokens_at

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _t(a):
    return torch.as_tensor(np.asarray(a), dtype=torch.int32, device=DEV)


@pytest.mark.parametrize("name,B", [("tiny", 3), ("tiny_moe", 8)])
def test_noalloc_matches_decode_step_two_calls(name, B):
    from persistent_decode_megakernel_sm_b200 import mk
    mc = synth.preset(name, gain_sigma=0.1)
    m = gpu_model(mc)
    kv_a = m.kv_cache(B, mc.max_ctx)
    kv_b = m.kv_cache(B, mc.max_ctx)
    for kv in (kv_a, kv_b):
        kv.fill_random(synth.SEED_KV, mc.kv_sigma, 40)
    pos = [40 - 4 * s for s in range(B)]
    for step in range(2):
        pp = [p + step for p in pos]
        toks = _t([int(tokens_at(mc, s, [pp[s]])[0]) for s in range(B)])
        out = {}
        for key, kv, fn in (("ref", kv_a, mk.mk_decode_step), ("noalloc", kv_b, mk.mk_decode_step_noalloc)):
            lg = torch.empty((B, mc.vocab), dtype=torch.float32, device=DEV)
            am = torch.empty(B, dtype=torch.int32, device=DEV)
            fn(m.h, toks, _t(pp), B, kv.h, lg, am)
            torch.cuda.synchronize()
            assert m.sync_status() == 0
            out[key] = (lg.cpu().numpy(), am.cpu().numpy())
        for b in range(B):
            ok, err, sc = logits_close(out["noalloc"][0][b], out["ref"][0][b].astype(np.float64))
            assert ok, (name, step, b, err, sc)
        assert np.array_equal(out["noalloc"][1], out["ref"][1])
    kv_a.close()
    kv_b.close()
    m.close()


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
