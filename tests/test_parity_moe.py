"""GPU parity of the MoE decoder path (router -> shared expert -> routed
experts -> down projection, all in the one persistent launch) against the
fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import synth
from harness import (CODE_MISMATCH_MAX, DELTA, check_router, code_mismatch, compare_rows, gpu_model,
                     tokens_at)

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _t(a, dtype=torch.int32):
    return torch.as_tensor(np.asarray(a), dtype=dtype, device=DEV)


def _router_buffers(mc, M):
    idx = torch.full((mc.layers, M, mc.top_k), -1, dtype=torch.int32, device=DEV)
    w = torch.zeros((mc.layers, M, mc.top_k), dtype=torch.float32, device=DEV)
    return idx, w


def _gpu_step(m, mc, toks, pos, kv, Q=1):
    """A traced GPU step: logits, greedy tokens, accepted (verify), router."""
    M = len(toks)
    logits = torch.empty((M, mc.vocab), dtype=torch.float32, device=DEV)
    am = torch.empty(M, dtype=torch.int32, device=DEV)
    acc = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    idx, w = _router_buffers(mc, M)
    m.set_router_trace(idx, w)
    if Q == 1:
        m.decode_step(_t(toks), _t(pos), kv, logits, am)
    else:
        m.verify(_t(toks), pos[0], kv, logits, am, acc)
    m.set_router_trace(None, None)
    torch.cuda.synchronize()
    return logits.cpu().numpy(), am.cpu().numpy(), int(acc.item()), idx.cpu().numpy(), w.cpu().numpy()


def _compare(mc, orc, m, kv, toks, pos, Q=1, fp8=False, what=""):
    """GPU step against the oracle's step on the same tokens (the oracle
    follows the GPU's router at its own near-ties)."""
    g, am, acc, gidx, gw = _gpu_step(m, mc, toks, pos, kv, Q)
    ref = orc.step(toks, pos, Q=Q, follow=gidx, delta=DELTA)
    check_router(mc, gidx, gw, ref, len(toks))
    compare_rows(g, am, ref, range(len(toks)), fp8, what)
    return g, am, acc, ref


@pytest.fixture(scope="module")
def tiny_moe():
    mc = synth.preset("tiny_moe")
    m = gpu_model(mc)
    yield mc, m
    m.close()


@pytest.mark.parametrize("B", [1, 3, 8])
def test_tiny_moe_batched_ragged(tiny_moe, B):
    """B sequences at ragged positions over a synthetic context: logits,
    greedy tokens and every layer's router choice and weights."""
    mc, m = tiny_moe
    kv = m.kv_cache(8, mc.max_ctx)
    kv.fill_random(synth.SEED_KV, mc.kv_sigma, mc.context)
    orc = oracle.OracleModel(mc.replace(max_seqs=8))
    orc.kv_fill_synthetic(synth.SEED_KV, mc.context)
    pos = [mc.context - 5 * s for s in range(B)]
    for step in range(3):
        pp = [p + step for p in pos]
        toks = [int(tokens_at(mc, s, [pp[s]])[0]) for s in range(B)]
        _compare(mc, orc, m, kv, toks, pp, what=f"B={B} step {step}")
    assert m.sync_status() == 0
    kv.close()


def test_tiny_moe_prefill_and_greedy(tiny_moe):
    """Pre-fill from seeded tokens through the model on both sides, then
    teacher-forced greedy steps (both sides consume the GPU's token); also
    compares the K/V both sides wrote."""
    mc, m = tiny_moe
    kv = m.kv_cache(1, mc.max_ctx)
    orc = oracle.OracleModel(mc.replace(max_seqs=1))
    toks = tokens_at(mc, 0, range(mc.context))
    for p in range(mc.context):
        _compare(mc, orc, m, kv, [toks[p]], [p], what=f"prefill {p}")
    tok = int(tokens_at(mc, 0, [mc.context])[0])
    for step in range(8):
        p = mc.context + step
        g, am, _, _ = _compare(mc, orc, m, kv, [tok], [p], what=f"greedy {step}")
        tok = int(am[0])
    assert m.sync_status() == 0
    kk, vv = orc.kv_arrays()
    dev = kv.copy_out().cpu().numpy().view(np.uint16)
    half = dev.size // 2
    n = mc.context + 8
    rate = code_mismatch(np.stack([dev[:half].reshape(kk.shape)[:, :, :, :n], dev[half:].reshape(vv.shape)[:, :, :, :n]]),
                         np.stack([kk[:, :, :, :n], vv[:, :, :, :n]]))
    assert rate <= CODE_MISMATCH_MAX, rate
    kv.close()


def test_tiny_moe_verify(tiny_moe):
    """1 anchor + 7 proposals on the MoE model: the 8 rows share one router
    union; planted proposals (the oracle's greedy chain) are all accepted."""
    mc, m = tiny_moe
    P = mc.context
    kv = m.kv_cache(1, mc.max_ctx)
    kv.fill_random(synth.SEED_KV, mc.kv_sigma, P)
    orc = oracle.OracleModel(mc.replace(max_seqs=1))
    orc.kv_fill_synthetic(synth.SEED_KV, P)
    chain_model = oracle.OracleModel(mc.replace(max_seqs=1))
    chain_model.kv_fill_synthetic(synth.SEED_KV, P)
    anchor = int(tokens_at(mc, 0, [P])[0])
    chain = [anchor]
    for j in range(7):
        r = chain_model.step([chain[-1]], [P + j], want_logits=False)
        chain.append(int(r["argmax"][0]))
    for case, props in (("planted", chain[1:]),
                        ("random", list(synth.proposals(synth.SEED_PROPOSALS, 0, 7, mc.vocab)))):
        toks = [anchor] + [int(x) for x in props]
        g, ga, acc, ref = _compare(mc, orc, m, kv, toks, [P], Q=8, what=case)
        if all(int(ga[j]) == int(ref["argmax"][j]) for j in range(8)):
            assert acc == oracle.accept(toks, ref["argmax"]), case
            if case == "planted":
                assert acc == 7
    assert m.sync_status() == 0
    kv.close()


def test_moe_no_shared_expert_and_top1():
    """Degenerate MoE shapes: no shared expert, top-1 routing, one layer."""
    mc = synth.preset("tiny_moe", n_shared=0, top_k=1, layers=1)
    m = gpu_model(mc)
    kv = m.kv_cache(4, mc.max_ctx)
    kv.fill_random(synth.SEED_KV, mc.kv_sigma, 20)
    orc = oracle.OracleModel(mc.replace(max_seqs=4))
    orc.kv_fill_synthetic(synth.SEED_KV, 20)
    toks, pos = [3, 99, 1500, 7], [20, 19, 18, 0]
    _, _, _, gidx, gw = _gpu_step(m, mc, toks, pos, kv)
    ref = orc.step(toks, pos, follow=gidx, delta=DELTA)
    check_router(mc, gidx, gw, ref, 4)
    assert np.allclose(gw, 1.0)
    g2, am2, _, ref2 = _compare(mc, orc, m, kv, toks, pos, what="top1")
    assert m.sync_status() == 0
    kv.close()
    m.close()


@pytest.mark.parametrize("B", [1, 2, 8])
def test_tiny_moe_fp8_experts(B):
    """Shared and routed expert weights as e4m3 codes with one fp32 scale per
    128 x 128 block (expert_ffn 192 gives a ragged second block)."""
    mc = synth.preset("tiny_moe", expert_fp8=1)
    m = gpu_model(mc)
    kv = m.kv_cache(8, mc.max_ctx)
    kv.fill_random(synth.SEED_KV, mc.kv_sigma, mc.context)
    orc = oracle.OracleModel(mc.replace(max_seqs=8))
    orc.kv_fill_synthetic(synth.SEED_KV, mc.context)
    pp = [mc.context - 3 * s for s in range(B)]
    toks = [int(tokens_at(mc, s, [pp[s]])[0]) for s in range(B)]
    _compare(mc, orc, m, kv, toks, pp, fp8=True, what=f"fp8 B={B}")
    assert m.sync_status() == 0
    kv.close()
    m.close()

