"""GPU parity of whole decode steps of the benchmarked workloads at their full
depth, against the fp64 oracle, through the C ABI.

Each workload is the benchmark's model with every layer (dense 27B-shaped:
64 layers; MoE: 32; latent attention with fp8 experts: 48), its vocabulary
and its context length.  The context is sequence 0's seeded prompt run
through the model by the GPU itself (mk_prefill, 8 positions per launch) and
copied to the other sequences; that cache is handed to the oracle as input.
Every row's logits and greedy token and every layer's router decision are
compared; where the oracle's own router margin is a near-tie (< DELTA) it
adopts the GPU's selection if that is correct at the tolerance, so later
layers stay comparable.  Multi-step runs feed both sides the GPU's greedy
token (teacher forcing).  The cache rows the step writes are compared code
by code."""
import numpy as np
import pytest
import torch

import oracle
import synth
from harness import (CODE_MISMATCH_MAX_DEEP, DELTA, check_router, code_mismatch, compare_rows, gpu_model,
                     tokens_at)

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
NSEQ = 8


def _t(a):
    return torch.as_tensor(np.asarray(a), dtype=torch.int32, device=DEV)


def _replicate_seq0(snap: torch.Tensor, mc, nseq: int) -> None:
    """Copy sequence 0 of a logical cache image to sequences 1..nseq-1 in place."""
    L = mc.layers
    if mc.mla:
        v = snap.view(L, nseq, -1)
        v[:, 1:] = v[:, :1]
    else:
        v = snap.view(2, L, nseq, -1)
        v[:, :, 1:] = v[:, :, :1]


class Full:
    def __init__(self, name):
        self.mc = mc = synth.preset(name, gain_sigma=0.1)
        self.m = gpu_model(mc)
        self.kv = self.m.kv_cache(NSEQ, mc.max_ctx)
        prompt = tokens_at(mc, 0, range(mc.context))
        self.m.prefill(_t(prompt), 0, 0, self.kv)
        torch.cuda.synchronize()
        assert self.m.sync_status() == 0
        snap = self.kv.copy_out()
        _replicate_seq0(snap, mc, NSEQ)
        self.kv.copy_in(snap)
        self.snap = snap
        self.host = snap.cpu().numpy()

    def restore(self):
        self.kv.copy_in(self.snap)

    def oracle(self):
        o = oracle.OracleModel(self.mc.replace(max_seqs=NSEQ))
        o.set_kv(self.host)
        return o

    def close(self):
        self.kv.close()
        self.m.close()


@pytest.fixture(scope="module", params=["dense27b", "moe", "mla_fp8"])
def full(request):
    f = Full(request.param)
    yield f
    f.close()


def _step(f, orc, toks, pos, Q=1):
    """One GPU step (decode for Q = 1, verify for Q > 1) and the oracle's
    step on the same tokens, following the GPU's router at near-ties."""
    mc, m = f.mc, f.m
    M = len(toks)
    logits = torch.empty((M, mc.vocab), dtype=torch.float32, device=DEV)
    am = torch.empty(M, dtype=torch.int32, device=DEV)
    acc = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    k = max(mc.top_k, 1)
    idx = torch.full((mc.layers, M, k), -1, dtype=torch.int32, device=DEV)
    w = torch.zeros((mc.layers, M, k), dtype=torch.float32, device=DEV)
    if mc.n_routed:
        m.set_router_trace(idx, w)
    if Q == 1:
        m.decode_step(_t(toks), _t(pos), f.kv, logits, am)
    else:
        m.verify(_t(toks), pos[0], f.kv, logits, am, acc)
    m.set_router_trace(None, None)
    torch.cuda.synchronize()
    assert m.sync_status() == 0
    gidx = idx.cpu().numpy()
    ref = orc.step(toks, pos, Q=Q, absorbed=mc.mla, follow=gidx if mc.n_routed else None, delta=DELTA)
    out = dict(logits=logits.cpu().numpy(), argmax=am.cpu().numpy(), accepted=int(acc.item()), ref=ref)
    if mc.n_routed:
        out["followed"] = check_router(mc, gidx, w.cpu().numpy(), ref, M)
    return out


def _cache_rows(f, orc, seq_pos):
    """Fraction of differing codes in the cache rows at (sequence, position)
    pairs, GPU against oracle, over every layer (and kv head)."""
    mc = f.mc
    dev = f.kv.copy_out().cpu().numpy().view(np.uint16)
    if mc.mla:
        lat = orc.kv_arrays()
        g = dev.reshape(lat.shape)
        a = np.stack([g[:, s, p] for s, p in seq_pos])
        b = np.stack([lat[:, s, p] for s, p in seq_pos])
    else:
        kk, vv = orc.kv_arrays()
        half = dev.size // 2
        gk, gv = dev[:half].reshape(kk.shape), dev[half:].reshape(vv.shape)
        a = np.stack([x[:, s, :, p] for s, p in seq_pos for x in (gk, gv)])
        b = np.stack([x[:, s, :, p] for s, p in seq_pos for x in (kk, vv)])
    return code_mismatch(a, b)


@pytest.mark.parametrize("B", [1, NSEQ])
def test_full_depth_decode(full, B):
    """B = 1: two teacher-forced greedy steps of sequence 0 past its
    context.  B = 8: one step of 8 sequences at ragged positions."""
    f = full
    mc = f.mc
    f.restore()
    orc = f.oracle()
    fp8 = bool(mc.expert_fp8)
    if B == 1:
        pos = [mc.context]
        tok = [int(tokens_at(mc, 0, pos)[0])]
        written = []
        for step in range(2):
            r = _step(f, orc, tok, pos)
            compare_rows(r["logits"], r["argmax"], r["ref"], range(1), fp8, f"{mc.name} B=1 step {step}")
            written.append((0, pos[0]))
            tok, pos = [int(r["argmax"][0])], [pos[0] + 1]
    else:
        pos = [mc.context - 3 * s for s in range(B)]
        tok = [int(tokens_at(mc, s, [pos[s]])[0]) for s in range(B)]
        r = _step(f, orc, tok, pos)
        compare_rows(r["logits"], r["argmax"], r["ref"], range(B), fp8, f"{mc.name} B={B}")
        written = [(s, pos[s]) for s in range(B)]
    rate = _cache_rows(f, orc, written)
    assert rate <= CODE_MISMATCH_MAX_DEEP, (mc.name, B, rate)
    orc.close()


def test_full_depth_verify_planted_chain(full):
    """1 anchor + 7 proposals in one launch, the proposals being the GPU's
    own greedy decode chain from the same position: the verify logits match
    the oracle on all 8 rows, and all 7 proposals are accepted wherever the
    chain is also the oracle's greedy chain."""
    f = full
    mc, m = f.mc, f.m
    if mc.name != "moe":
        pytest.skip("the verify workload runs on the MoE model")
    f.restore()
    P = mc.context
    chain = [int(tokens_at(mc, 0, [P])[0])]
    am = torch.empty(1, dtype=torch.int32, device=DEV)
    for j in range(7):
        m.decode_step(_t([chain[-1]]), _t([P + j]), f.kv, None, am)
        torch.cuda.synchronize()
        chain.append(int(am.item()))
    orc = f.oracle()
    r = _step(f, orc, chain, [P], Q=8)
    ref = r["ref"]
    compare_rows(r["logits"], r["argmax"], ref, range(8), False, "moe verify")
    exact = all(int(r["argmax"][j]) == int(ref["argmax"][j]) for j in range(8))
    if exact:
        assert r["accepted"] == oracle.accept(chain, ref["argmax"])
        if all(int(ref["argmax"][j]) == chain[j + 1] for j in range(7)):
            assert r["accepted"] == 7
    rate = _cache_rows(f, orc, [(0, P + j) for j in range(8)])
    assert rate <= CODE_MISMATCH_MAX_DEEP, rate
    orc.close()


def test_full_depth_verify_random_proposals(full):
    """The verify workload's own input: 1 anchor + 7 seeded uniform proposals."""
    f = full
    mc = f.mc
    if mc.name != "moe":
        pytest.skip("the verify workload runs on the MoE model")
    f.restore()
    P = mc.context
    toks = [int(tokens_at(mc, 0, [P])[0])] + [int(x) for x in synth.proposals(synth.SEED_PROPOSALS, 0, 7, mc.vocab)]
    orc = f.oracle()
    r = _step(f, orc, toks, [P], Q=8)
    ref = r["ref"]
    compare_rows(r["logits"], r["argmax"], ref, range(8), False, "moe verify random")
    if all(int(r["argmax"][j]) == int(ref["argmax"][j]) for j in range(8)):
        assert r["accepted"] == oracle.accept(toks, ref["argmax"])
    orc.close()
