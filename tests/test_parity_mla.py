"""GPU parity of the latent-attention (MLA) decoder with fp8 block-scaled
experts against the fp64 oracle, through the C ABI.

The oracle evaluates latent attention in its explicit form (per-position
key and value up-projections); the GPU path absorbs W_uk into the query and
applies W_uv after the attention, so these tests also check that
associativity on the real step."""
import numpy as np
import pytest
import torch

import oracle
import synth
from harness import DELTA, argmax_agrees, gpu_model, logits_close, tokens_at

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _t(a):
    return torch.as_tensor(np.asarray(a), dtype=torch.int32, device=DEV)


def _tied_rows(mc, ref, rows):
    return {r for r in range(rows) if (ref["router_margin"][:, r] < DELTA).any()}


def _check_router(mc, idx, w, ref, rows):
    gi, gw = idx.cpu().numpy(), w.cpu().numpy()
    for l in range(mc.layers):
        for r in range(rows):
            if ref["router_margin"][l, r] < DELTA:
                continue
            assert list(gi[l, r]) == list(ref["router_idx"][l, r]), (l, r)
            assert np.allclose(gw[l, r], ref["router_w"][l, r], atol=5e-3), (l, r)


@pytest.fixture(scope="module")
def tiny_mla():
    mc = synth.preset("tiny_mla")
    m = gpu_model(mc)
    yield mc, m
    m.close()


@pytest.mark.parametrize("B", [1, 3, 8])
def test_tiny_mla_batched_ragged(tiny_mla, B):
    mc, m = tiny_mla
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
        idx = torch.full((mc.layers, B, mc.top_k), -1, dtype=torch.int32, device=DEV)
        w = torch.zeros((mc.layers, B, mc.top_k), dtype=torch.float32, device=DEV)
        m.set_router_trace(idx, w)
        m.decode_step(_t(toks), _t(pp), kv, logits, am)
        m.set_router_trace(None, None)
        ref = orc.step(toks, pp)
        torch.cuda.synchronize()
        _check_router(mc, idx, w, ref, B)
        tied = _tied_rows(mc, ref, B)
        g = logits.cpu().numpy()
        for b in range(B):
            if b in tied:
                continue
            ok, err, sc = logits_close(g[b], ref["logits"][b], fp8=True)
            assert ok, (step, b, err, sc)
            assert argmax_agrees(int(am[b].item()), ref["logits"][b], int(ref["argmax"][b]),
                                 ref["argmax_margin"][b])
    assert m.sync_status() == 0
    kv.close()


def test_tiny_mla_prefill_greedy_and_latent_cache(tiny_mla):
    """Pre-fill through the model on both sides, greedy steps, and the latent
    rows [c | RoPE(k_rope)] both sides appended (bf16, at most one code apart)."""
    mc, m = tiny_mla
    kv = m.kv_cache(1, mc.max_ctx)
    orc = oracle.OracleModel(mc.replace(max_seqs=1))
    toks = tokens_at(mc, 0, range(mc.context))
    logits = torch.empty((1, mc.vocab), dtype=torch.float32, device=DEV)
    am = torch.empty(1, dtype=torch.int32, device=DEV)
    for p in range(mc.context):
        m.decode_step(_t([toks[p]]), _t([p]), kv, logits, am)
        ref = orc.step([toks[p]], [p], want_logits=(p % 16 == 15))
        if p % 16 == 15 and not _tied_rows(mc, ref, 1):
            torch.cuda.synchronize()
            ok, err, sc = logits_close(logits.cpu().numpy()[0], ref["logits"][0], fp8=True)
            assert ok, (p, err, sc)
    tok_g = tok_o = int(tokens_at(mc, 0, [mc.context])[0])
    for step in range(8):
        p = mc.context + step
        m.decode_step(_t([tok_g]), _t([p]), kv, logits, am)
        ref = orc.step([tok_o], [p])
        torch.cuda.synchronize()
        if _tied_rows(mc, ref, 1):
            break
        g = logits.cpu().numpy()[0]
        ok, err, sc = logits_close(g, ref["logits"][0], fp8=True)
        assert ok, (step, err, sc)
        ga = int(am.item())
        assert argmax_agrees(ga, ref["logits"][0], int(ref["argmax"][0]), ref["argmax_margin"][0]), step
        if ga != int(ref["argmax"][0]):
            break
        tok_g, tok_o = ga, int(ref["argmax"][0])
    assert m.sync_status() == 0
    lat = orc.kv_arrays()
    dev = kv.copy_out().cpu().numpy().view(np.uint16).reshape(lat.shape)
    n = mc.context
    a, b = dev[:, :, :n], lat[:, :, :n]
    fa = synth.bf16_to_f32(np.ascontiguousarray(a)).astype(np.float64)
    fb = synth.bf16_to_f32(np.ascontiguousarray(b)).astype(np.float64)
    scale = np.max(np.abs(fb))
    assert np.all(np.abs(fa - fb) <= 2.0 ** -7 * np.maximum(np.abs(fa), np.abs(fb)) + 1e-3 * scale)
    assert np.mean(a != b) < 0.1
    kv.close()


def test_tiny_mla_verify(tiny_mla):
    """1 anchor + 7 proposals: 8 query rows of one sequence, causal over the
    chunk, planted proposals (the oracle's greedy chain) all accepted."""
    mc, m = tiny_mla
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
        m.verify(_t(toks), P, kv, logits, am, acc)
        ref = orc.step(toks, [P], Q=8)
        torch.cuda.synchronize()
        tied = _tied_rows(mc, ref, 8)
        g = logits.cpu().numpy()
        for j in range(8):
            if j not in tied:
                ok, err, sc = logits_close(g[j], ref["logits"][j], fp8=True)
                assert ok, (case, j, err, sc)
        ga = am.cpu().numpy()
        if not tied and all(int(ga[j]) == int(ref["argmax"][j]) for j in range(8)):
            assert int(acc.item()) == oracle.accept(toks, ref["argmax"]), case
            if case == "planted":
                assert int(acc.item()) == 7
    assert m.sync_status() == 0
    kv.close()


def test_mla_bf16_experts_dense_heads():
    """Latent attention with bf16 experts and 32 heads (two m-tiles per item),
    one layer, R = 128."""
    mc = synth.preset("tiny_mla", layers=1, n_q_heads=32, kv_lora_rank=128, expert_fp8=0)
    m = gpu_model(mc)
    kv = m.kv_cache(2, mc.max_ctx)
    kv.fill_random(synth.SEED_KV, mc.kv_sigma, 70)
    orc = oracle.OracleModel(mc.replace(max_seqs=2))
    orc.kv_fill_synthetic(synth.SEED_KV, 70)
    toks, pos = [5, 1999], [70, 33]
    logits = torch.empty((2, mc.vocab), dtype=torch.float32, device=DEV)
    am = torch.empty(2, dtype=torch.int32, device=DEV)
    m.decode_step(_t(toks), _t(pos), kv, logits, am)
    ref = orc.step(toks, pos)
    torch.cuda.synchronize()
    tied = _tied_rows(mc, ref, 2)
    g = logits.cpu().numpy()
    for b in range(2):
        if b not in tied:
            ok, err, sc = logits_close(g[b], ref["logits"][b])
            assert ok, (b, err, sc)
    assert m.sync_status() == 0
    kv.close()
    m.close()
