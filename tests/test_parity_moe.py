"""GPU parity of the MoE decoder path (router -> shared expert -> routed
experts -> down projection, all in the one persistent launch) against the
fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import synth
from harness import DELTA, argmax_agrees, gpu_model, logits_close, tokens_at

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _t(a, dtype=torch.int32):
    return torch.as_tensor(np.asarray(a), dtype=dtype, device=DEV)


def _router_buffers(mc, M):
    idx = torch.full((mc.layers, M, mc.top_k), -1, dtype=torch.int32, device=DEV)
    w = torch.zeros((mc.layers, M, mc.top_k), dtype=torch.float32, device=DEV)
    return idx, w


def _check_router(mc, idx, w, ref, rows):
    """Expert choices are exact unless the oracle's own k-th / (k+1)-th logit
    gap is below DELTA (a near-tie).  Returns the rows whose choice is a
    near-tie somewhere (their logits are then not comparable)."""
    gi = idx.cpu().numpy()
    gw = w.cpu().numpy()
    tied = set()
    for l in range(mc.layers):
        for r in range(rows):
            if ref["router_margin"][l, r] < DELTA:
                tied.add(r)
                continue
            assert list(gi[l, r]) == list(ref["router_idx"][l, r]), (l, r, gi[l, r], ref["router_idx"][l, r])
            assert np.allclose(gw[l, r], ref["router_w"][l, r], atol=5e-3), (l, r)
    return tied


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
        logits = torch.empty((B, mc.vocab), dtype=torch.float32, device=DEV)
        am = torch.empty(B, dtype=torch.int32, device=DEV)
        idx, w = _router_buffers(mc, B)
        m.set_router_trace(idx, w)
        m.decode_step(_t(toks), _t(pp), kv, logits, am)
        m.set_router_trace(None, None)
        ref = orc.step(toks, pp)
        torch.cuda.synchronize()
        tied = _check_router(mc, idx, w, ref, B)
        g = logits.cpu().numpy()
        for b in range(B):
            if b in tied:
                continue
            ok, err, sc = logits_close(g[b], ref["logits"][b])
            assert ok, (step, b, err, sc)
            assert argmax_agrees(int(am[b].item()), ref["logits"][b], int(ref["argmax"][b]),
                                 ref["argmax_margin"][b])
    assert m.sync_status() == 0
    kv.close()


def test_tiny_moe_prefill_and_greedy(tiny_moe):
    """Pre-fill from seeded tokens through the model on both sides, then
    greedy steps; also compares the K/V both sides wrote."""
    mc, m = tiny_moe
    kv = m.kv_cache(1, mc.max_ctx)
    orc = oracle.OracleModel(mc.replace(max_seqs=1))
    toks = tokens_at(mc, 0, range(mc.context))
    logits = torch.empty((1, mc.vocab), dtype=torch.float32, device=DEV)
    am = torch.empty(1, dtype=torch.int32, device=DEV)
    for p in range(mc.context):
        m.decode_step(_t([toks[p]]), _t([p]), kv, logits, am)
        ref = orc.step([toks[p]], [p], want_logits=(p % 16 == 15))
        if p % 16 == 15:
            torch.cuda.synchronize()
            ok, err, sc = logits_close(logits.cpu().numpy()[0], ref["logits"][0])
            if not (ref["router_margin"][:, 0] < DELTA).any():
                assert ok, (p, err, sc)
    tok_g = tok_o = int(tokens_at(mc, 0, [mc.context])[0])
    for step in range(8):
        p = mc.context + step
        m.decode_step(_t([tok_g]), _t([p]), kv, logits, am)
        ref = orc.step([tok_o], [p])
        torch.cuda.synchronize()
        g = logits.cpu().numpy()[0]
        if (ref["router_margin"][:, 0] < DELTA).any():
            break
        ok, err, sc = logits_close(g, ref["logits"][0])
        assert ok, (step, err, sc)
        ga = int(am.item())
        assert argmax_agrees(ga, ref["logits"][0], int(ref["argmax"][0]), ref["argmax_margin"][0]), step
        if ga != int(ref["argmax"][0]):
            break
        tok_g, tok_o = ga, int(ref["argmax"][0])
    assert m.sync_status() == 0
    kk, vv = orc.kv_arrays()
    dev = kv.copy_out().cpu().numpy().view(np.uint16)
    half = dev.size // 2
    n = mc.context
    for a, b in ((dev[:half].reshape(kk.shape)[:, :, :, :n], kk[:, :, :, :n]),
                 (dev[half:].reshape(vv.shape)[:, :, :, :n], vv[:, :, :, :n])):
        fa = synth.bf16_to_f32(np.ascontiguousarray(a)).astype(np.float64)
        fb = synth.bf16_to_f32(np.ascontiguousarray(b)).astype(np.float64)
        scale = np.max(np.abs(fb))
        assert np.all(np.abs(fa - fb) <= 2.0 ** -7 * np.maximum(np.abs(fa), np.abs(fb)) + 1e-3 * scale)
        assert np.mean(a != b) < 0.1
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
        logits = torch.empty((8, mc.vocab), dtype=torch.float32, device=DEV)
        am = torch.empty(8, dtype=torch.int32, device=DEV)
        acc = torch.full((1,), -1, dtype=torch.int32, device=DEV)
        idx, w = _router_buffers(mc, 8)
        m.set_router_trace(idx, w)
        m.verify(_t(toks), P, kv, logits, am, acc)
        m.set_router_trace(None, None)
        ref = orc.step(toks, [P], Q=8)
        torch.cuda.synchronize()
        tied = _check_router(mc, idx, w, ref, 8)
        g = logits.cpu().numpy()
        for j in range(8):
            if j in tied:
                continue
            ok, err, sc = logits_close(g[j], ref["logits"][j])
            assert ok, (case, j, err, sc)
        ga = am.cpu().numpy()
        if not tied and all(int(ga[j]) == int(ref["argmax"][j]) for j in range(8)):
            assert int(acc.item()) == oracle.accept(toks, ref["argmax"]), case
            if case == "planted":
                assert int(acc.item()) == 7
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
    logits = torch.empty((4, mc.vocab), dtype=torch.float32, device=DEV)
    am = torch.empty(4, dtype=torch.int32, device=DEV)
    idx, w = _router_buffers(mc, 4)
    m.set_router_trace(idx, w)
    m.decode_step(_t(toks), _t(pos), kv, logits, am)
    ref = orc.step(toks, pos)
    torch.cuda.synchronize()
    tied = _check_router(mc, idx, w, ref, 4)
    assert np.allclose(w.cpu().numpy(), 1.0)
    g = logits.cpu().numpy()
    for b in range(4):
        if b not in tied:
            ok, err, sc = logits_close(g[b], ref["logits"][b])
            assert ok, (b, err, sc)
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
    logits = torch.empty((B, mc.vocab), dtype=torch.float32, device=DEV)
    am = torch.empty(B, dtype=torch.int32, device=DEV)
    idx, w = _router_buffers(mc, B)
    m.set_router_trace(idx, w)
    m.decode_step(_t(toks), _t(pp), kv, logits, am)
    ref = orc.step(toks, pp)
    torch.cuda.synchronize()
    tied = _check_router(mc, idx, w, ref, B)
    g = logits.cpu().numpy()
    for b in range(B):
        if b in tied:
            continue
        ok, err, sc = logits_close(g[b], ref["logits"][b], fp8=True)
        assert ok, (b, err, sc)
        assert argmax_agrees(int(am[b].item()), ref["logits"][b], int(ref["argmax"][b]), ref["argmax_margin"][b])
    assert m.sync_status() == 0
    kv.close()
    m.close()

