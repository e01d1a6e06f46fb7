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
from harness import (CODE_MISMATCH_MAX, DELTA, check_router, code_mismatch, compare_rows, gpu_model,
                     tokens_at)

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _t(a):
    return torch.as_tensor(np.asarray(a), dtype=torch.int32, device=DEV)


def _compare(mc, orc, m, kv, toks, pos, Q=1, what=""):
    """A traced GPU step against the oracle's step on the same tokens (the
    oracle follows the GPU's router at its own near-ties): logits, greedy
    tokens, router choices and weights.  Returns (argmax, accepted, ref)."""
    M = len(toks)
    logits = torch.empty((M, mc.vocab), dtype=torch.float32, device=DEV)
    am = torch.empty(M, dtype=torch.int32, device=DEV)
    acc = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    idx = torch.full((mc.layers, M, mc.top_k), -1, dtype=torch.int32, device=DEV)
    w = torch.zeros((mc.layers, M, mc.top_k), dtype=torch.float32, device=DEV)
    m.set_router_trace(idx, w)
    if Q == 1:
        m.decode_step(_t(toks), _t(pos), kv, logits, am)
    else:
        m.verify(_t(toks), pos[0], kv, logits, am, acc)
    m.set_router_trace(None, None)
    torch.cuda.synchronize()
    gidx = idx.cpu().numpy()
    ref = orc.step(toks, pos, Q=Q, follow=gidx, delta=DELTA)
    check_router(mc, gidx, w.cpu().numpy(), ref, M)
    ga = am.cpu().numpy()
    compare_rows(logits.cpu().numpy(), ga, ref, range(M), bool(mc.expert_fp8), what)
    return ga, int(acc.item()), ref


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
        _compare(mc, orc, m, kv, toks, pp, what=f"B={B} step {step}")
    assert m.sync_status() == 0
    kv.close()


def test_tiny_mla_prefill_greedy_and_latent_cache(tiny_mla):
    """Pre-fill through the model on both sides, teacher-forced greedy steps
    (both sides consume the GPU's token), and the latent rows
    [c | RoPE(k_rope)] both sides appended (bf16, at most one code apart)."""
    mc, m = tiny_mla
    kv = m.kv_cache(1, mc.max_ctx)
    orc = oracle.OracleModel(mc.replace(max_seqs=1))
    toks = tokens_at(mc, 0, range(mc.context))
    for p in range(mc.context):
        _compare(mc, orc, m, kv, [toks[p]], [p], what=f"prefill {p}")
    tok = int(tokens_at(mc, 0, [mc.context])[0])
    for step in range(8):
        ga, _, _ = _compare(mc, orc, m, kv, [tok], [mc.context + step], what=f"greedy {step}")
        tok = int(ga[0])
    assert m.sync_status() == 0
    lat = orc.kv_arrays()
    dev = kv.copy_out().cpu().numpy().view(np.uint16).reshape(lat.shape)
    n = mc.context + 8
    rate = code_mismatch(dev[:, :, :n], lat[:, :, :n])
    assert rate <= CODE_MISMATCH_MAX, rate
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
        ga, acc, ref = _compare(mc, orc, m, kv, toks, [P], Q=8, what=case)
        if all(int(ga[j]) == int(ref["argmax"][j]) for j in range(8)):
            assert acc == oracle.accept(toks, ref["argmax"]), case
            if case == "planted":
                assert acc == 7
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
    _compare(mc, orc, m, kv, toks, pos, what="bf16 experts")
    assert m.sync_status() == 0
    kv.close()
    m.close()
