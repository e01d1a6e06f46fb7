"""Speculative greedy generation (mk_spec_generate: a verify launch of the
anchor and up to 7 proposals, keep the accepted prefix and the bonus token,
rewind the rest) emits exactly the tokens plain greedy decoding emits,
whatever the draft proposes.  Checked on the three model families with a
draft that proposes the plain greedy chain (all accepted), one that corrupts
each proposal with a set probability, and one that proposes random tokens.
Comparisons stop at the first position whose plain-decode top-2 logit gap is
below DELTA (a near-tie, where either token is a correct greedy choice)."""
import random

import numpy as np
import pytest
import torch

import synth
from harness import DELTA, gpu_model, tokens_at

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
N_OUT = 40


def _t(a):
    return torch.as_tensor(np.asarray(a), dtype=torch.int32, device=DEV)


def chain_draft(chain, err=0.0, seed=0, vocab=2):
    """Proposes the continuation of `chain` (the plain greedy tokens), each
    proposal replaced with probability `err` by another seeded token."""
    rng = random.Random(seed)

    def draft(history, max_k):
        e = len(history) - 1  # tokens emitted so far
        out = []
        for j in range(e, min(e + max_k, len(chain))):
            t = chain[j]
            if err > 0 and rng.random() < err:
                t = (t + 1 + rng.randrange(vocab - 1)) % vocab
            out.append(t)
        return out

    return draft


def random_draft(vocab, seed=0):
    rng = random.Random(seed)
    return lambda history, max_k: [rng.randrange(vocab) for _ in range(max_k)]


@pytest.fixture(scope="module", params=["tiny", "tiny_moe", "tiny_mla"])
def setup(request):
    mc = synth.preset(request.param, gain_sigma=0.1)
    m = gpu_model(mc)
    kv = m.kv_cache(1, mc.max_ctx)
    P = mc.max_ctx - N_OUT - 10  # room for the last launch's 8 positions
    prompt = tokens_at(mc, 0, range(P))
    m.prefill(_t(prompt), 0, 0, kv)
    torch.cuda.synchronize()
    snap = kv.copy_out()
    anchor = int(tokens_at(mc, 0, [P])[0])
    # plain greedy decode from the anchor, with each step's top-2 gap
    chain, gaps = [], []
    logits = torch.empty((1, mc.vocab), dtype=torch.float32, device=DEV)
    am = torch.empty(1, dtype=torch.int32, device=DEV)
    cur = anchor
    for j in range(N_OUT + 8):
        m.decode_step(_t([cur]), _t([P + j]), kv, logits, am)
        torch.cuda.synchronize()
        g = np.sort(logits.cpu().numpy()[0])
        gaps.append(float(g[-1] - g[-2]))
        cur = int(am.item())
        chain.append(cur)
    assert m.sync_status() == 0
    yield mc, m, kv, snap, P, anchor, chain, gaps
    kv.close()
    m.close()


def _check(setup, draft):
    mc, m, kv, snap, P, anchor, chain, gaps = setup
    kv.copy_in(snap)
    out, stats = m.spec_generate(kv, anchor, P, N_OUT, draft)
    assert m.sync_status() == 0
    n = N_OUT
    for j, g in enumerate(gaps[:N_OUT]):
        if g < DELTA:
            n = j + 1  # token j itself may be either choice; later ones follow from it
            break
    agree = out[:n - 1] == chain[:n - 1] if n < N_OUT else out == chain[:N_OUT]
    assert agree, (mc.name, out[:n], chain[:n])
    assert stats["emitted"] >= N_OUT and stats["accepted"] <= stats["proposed"]
    assert stats["emitted"] == stats["launches"] + stats["accepted"]
    return stats


def test_spec_perfect_draft_matches_greedy(setup):
    """The draft proposes the greedy chain itself: every proposal is accepted
    (8 tokens per launch)."""
    mc, _, _, _, _, _, chain, gaps = setup
    stats = _check(setup, chain_draft(chain))
    if min(gaps[:N_OUT]) >= DELTA:
        assert stats["launches"] == -(-N_OUT // 8)
        assert stats["accepted"] == stats["proposed"]


def test_spec_noisy_draft_matches_greedy(setup):
    """Each proposal is wrong with probability 0.3: fewer accepted per launch,
    the same emitted tokens."""
    mc, _, _, _, _, _, chain, _ = setup
    stats = _check(setup, chain_draft(chain, err=0.3, seed=7, vocab=mc.vocab))
    assert stats["launches"] > -(-N_OUT // 8)


def test_spec_random_draft_matches_greedy(setup):
    """Random proposals are (almost) never accepted: one token per launch."""
    mc = setup[0]
    stats = _check(setup, random_draft(mc.vocab, seed=3))
    assert stats["launches"] >= N_OUT - 2
