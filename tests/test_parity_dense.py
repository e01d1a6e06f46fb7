"""GPU parity of the dense decoder path (C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from harness import (CODE_MISMATCH_MAX, argmax_agrees, check_router, code_mismatch, compare_rows, gpu_model,
                     logits_close, tokens_at)

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _t(a, dtype=torch.int32):
    return torch.as_tensor(np.asarray(a), dtype=dtype, device=DEV)


@pytest.fixture(scope="module")
def tiny():
    mc = synth.preset("tiny")
    m = gpu_model(mc)
    yield mc, m
    m.close()


def test_tiny_prefill_and_greedy_decode(tiny):
    """The small dense workload: 128 positions pre-filled from seeded tokens
    (both sides run the model over them), then 16 greedy steps; logits,
    greedy tokens and the whole KV cache are compared."""
    mc, m = tiny
    kv = m.kv_cache(1, mc.max_ctx)
    orc = oracle.OracleModel(mc.replace(max_seqs=1))
    toks = tokens_at(mc, 0, range(mc.context))
    logits = torch.empty((1, mc.vocab), dtype=torch.float32, device=DEV)
    am = torch.empty(1, dtype=torch.int32, device=DEV)
    for p in range(mc.context):
        m.decode_step(_t([toks[p]]), _t([p]), kv, logits, am)
        ref = orc.step([toks[p]], [p], want_logits=(p % 32 == 31))
        if p % 32 == 31:
            torch.cuda.synchronize()
            ok, err, sc = logits_close(logits.cpu().numpy()[0], ref["logits"][0])
            assert ok, (p, err, sc)
    assert m.sync_status() == 0
    # greedy decode, teacher-forced: both sides consume the GPU's token, so
    # a near-tie (where the two greedy choices may differ) does not end the run
    tok = int(tokens_at(mc, 0, [mc.context])[0])
    for step in range(16):
        p = mc.context + step
        m.decode_step(_t([tok]), _t([p]), kv, logits, am)
        ref = orc.step([tok], [p])
        torch.cuda.synchronize()
        g = logits.cpu().numpy()[0]
        ga = int(am.item())
        assert ga == int(np.argmax(g)) or g[ga] == g.max()
        compare_rows(logits.cpu().numpy(), am.cpu().numpy(), ref, range(1), False, f"greedy step {step}")
        tok = ga
    assert m.sync_status() == 0
    # KV cache: bf16 values written by both sides, one code apart at most
    kk, vv = orc.kv_arrays()
    dev = kv.copy_out().cpu().numpy().view(np.uint16)
    half = dev.size // 2
    n_pos = mc.context + 16
    gk = dev[:half].reshape(kk.shape)[:, :, :, :n_pos]
    gv = dev[half:].reshape(vv.shape)[:, :, :, :n_pos]
    rate = code_mismatch(np.stack([gk, gv]), np.stack([kk[:, :, :, :n_pos], vv[:, :, :, :n_pos]]))
    assert rate <= CODE_MISMATCH_MAX, rate
    kv.close()


@pytest.mark.parametrize("name", ["tiny", "tiny_moe", "tiny_mla"])
def test_prefill_in_chunks_matches_oracle(name):
    """mk_prefill runs a prompt 8 positions per launch (the verify form), for
    cache sequence 0 and, in a second call, sequence 1.  The cache it writes
    matches the oracle's position-by-position prefill code for code (within
    the mismatch bound), its last greedy tokens are the oracle's, and a decode
    step over the GPU-written cache (handed to the oracle) matches."""
    mc = synth.preset(name, gain_sigma=0.1)
    m = gpu_model(mc)
    n = mc.context + 5  # a ragged last chunk
    kv = m.kv_cache(2, mc.max_ctx)
    toks = [tokens_at(mc, s, range(n + 1)) for s in range(2)]
    last = [torch.full((1,), -1, dtype=torch.int32, device=DEV) for _ in range(2)]
    for s in range(2):
        m.prefill(_t(toks[s][:n]), s, 0, kv, last[s])
    orc = oracle.OracleModel(mc.replace(max_seqs=2))
    for p in range(n):
        r = orc.step([toks[0][p], toks[1][p]], [p, p], want_logits=(p == n - 1))
    torch.cuda.synchronize()
    assert m.sync_status() == 0
    for s in range(2):
        assert argmax_agrees(int(last[s].item()), r["logits"][s], int(r["argmax"][s]), r["argmax_margin"][s]), s
    dev = kv.copy_out().cpu().numpy().view(np.uint16)
    if mc.mla:
        lat = orc.kv_arrays()
        rate = code_mismatch(dev.reshape(lat.shape)[:, :, :n], lat[:, :, :n])
    else:
        kk, vv = orc.kv_arrays()
        half = dev.size // 2
        gk, gv = dev[:half].reshape(kk.shape), dev[half:].reshape(vv.shape)
        rate = code_mismatch(np.stack([gk[:, :, :, :n], gv[:, :, :, :n]]),
                             np.stack([kk[:, :, :, :n], vv[:, :, :, :n]]))
    assert rate <= CODE_MISMATCH_MAX, (name, rate)
    orc.close()
    # one decode step of both sequences over the GPU-written context
    orc = oracle.OracleModel(mc.replace(max_seqs=2))
    orc.set_kv(dev)
    logits = torch.empty((2, mc.vocab), dtype=torch.float32, device=DEV)
    am = torch.empty(2, dtype=torch.int32, device=DEV)
    k = max(mc.top_k, 1)
    idx = torch.full((mc.layers, 2, k), -1, dtype=torch.int32, device=DEV)
    w = torch.zeros((mc.layers, 2, k), dtype=torch.float32, device=DEV)
    if mc.n_routed:
        m.set_router_trace(idx, w)
    step_toks = [toks[0][n], toks[1][n]]
    m.decode_step(_t(step_toks), _t([n, n]), kv, logits, am)
    m.set_router_trace(None, None)
    torch.cuda.synchronize()
    assert m.sync_status() == 0
    gidx = idx.cpu().numpy()
    ref = orc.step(step_toks, [n, n], follow=gidx if mc.n_routed else None)
    if mc.n_routed:
        check_router(mc, gidx, w.cpu().numpy(), ref, 2)
    compare_rows(logits.cpu().numpy(), am.cpu().numpy(), ref, range(2), bool(mc.expert_fp8), name)
    orc.close()
    kv.close()
    m.close()


def test_kv_copy_in_round_trip(tiny):
    """mk_kv_copy_in is the inverse of mk_kv_copy_out (logical order in and
    out), and a step over a copied-in cache equals the step over the original."""
    mc, m = tiny
    a = m.kv_cache(3, mc.max_ctx)
    b = m.kv_cache(3, mc.max_ctx)
    a.fill_random(synth.SEED_KV, mc.kv_sigma, 77)
    img = a.copy_out()
    b.copy_in(img)
    assert torch.equal(b.copy_out(), img)
    outs = []
    for kv in (a, b):
        lg = torch.empty((3, mc.vocab), dtype=torch.float32, device=DEV)
        am = torch.empty(3, dtype=torch.int32, device=DEV)
        m.decode_step(_t([4, 5, 6]), _t([77, 60, 10]), kv, lg, am)
        torch.cuda.synchronize()
        outs.append(lg.cpu().numpy().copy())
    assert np.array_equal(outs[0], outs[1])
    assert m.sync_status() == 0
    a.close()
    b.close()


@pytest.mark.parametrize("B", [1, 2, 3, 4, 8])
def test_tiny_batched_ragged_positions(tiny, B):
    """B sequences at different positions over a synthetic context, gains != 1."""
    mc = synth.preset("tiny", gain_sigma=0.1)
    m = gpu_model(mc)
    kv = m.kv_cache(8, mc.max_ctx)
    kv.fill_random(synth.SEED_KV, mc.kv_sigma, 100)
    orc = oracle.OracleModel(mc.replace(max_seqs=8))
    orc.kv_fill_synthetic(synth.SEED_KV, 100)
    pos = [100 - 7 * s for s in range(B)]
    for step in range(3):
        pp = [p + step for p in pos]
        toks = [int(tokens_at(mc, s, [pp[s]])[0]) for s in range(B)]
        logits = torch.empty((B, mc.vocab), dtype=torch.float32, device=DEV)
        am = torch.empty(B, dtype=torch.int32, device=DEV)
        m.decode_step(_t(toks), _t(pp), kv, logits, am)
        ref = orc.step(toks, pp)
        torch.cuda.synchronize()
        g = logits.cpu().numpy()
        for b in range(B):
            ok, err, sc = logits_close(g[b], ref["logits"][b])
            assert ok, (step, b, err, sc)
            assert argmax_agrees(int(am[b].item()), ref["logits"][b], int(ref["argmax"][b]),
                                 ref["argmax_margin"][b])
    assert m.sync_status() == 0
    kv.close()
    m.close()


def test_tiny_verify_planted_and_random(tiny):
    """1 anchor + 7 proposals in one launch: logits of all 8 positions, greedy
    tokens and the accepted length; planted proposals (the oracle's greedy
    chain) are all accepted."""
    mc, m = tiny
    kv = m.kv_cache(1, mc.max_ctx)
    kv.fill_random(synth.SEED_KV, mc.kv_sigma, 64)
    orc = oracle.OracleModel(mc.replace(max_seqs=1))
    orc.kv_fill_synthetic(synth.SEED_KV, 64)
    P = 64
    # greedy chain from the oracle (a separate copy, so orc's cache stays at the prefix)
    chain_model = oracle.OracleModel(mc.replace(max_seqs=1))
    chain_model.kv_fill_synthetic(synth.SEED_KV, 64)
    anchor = int(tokens_at(mc, 0, [P])[0])
    chain = [anchor]
    for j in range(7):
        r = chain_model.step([chain[-1]], [P + j], want_logits=False)
        chain.append(int(r["argmax"][0]))
    for case, props in (("planted", chain[1:]), ("random", list(synth.proposals(synth.SEED_PROPOSALS, 0, 7, mc.vocab)))):
        toks = [anchor] + [int(x) for x in props]
        logits = torch.empty((8, mc.vocab), dtype=torch.float32, device=DEV)
        am = torch.empty(8, dtype=torch.int32, device=DEV)
        acc = torch.full((1,), -1, dtype=torch.int32, device=DEV)
        m.verify(_t(toks), P, kv, logits, am, acc)
        ref = orc.step(toks, [P], Q=8)
        torch.cuda.synchronize()
        g = logits.cpu().numpy()
        for j in range(8):
            ok, err, sc = logits_close(g[j], ref["logits"][j])
            assert ok, (case, j, err, sc)
        ga = am.cpu().numpy()
        exact = all(int(ga[j]) == int(ref["argmax"][j]) for j in range(8))
        if exact:
            assert int(acc.item()) == oracle.accept(toks, ref["argmax"]), case
        if case == "planted" and exact:
            assert int(acc.item()) == 7
    assert m.sync_status() == 0
    kv.close()


def test_determinism(tiny):
    mc, m = tiny
    kv = m.kv_cache(4, mc.max_ctx)
    kv.fill_random(synth.SEED_KV, mc.kv_sigma, 50)
    toks, pos = _t([5, 6, 7, 8]), _t([50, 40, 30, 20])
    outs = []
    for _ in range(2):
        kv.fill_random(synth.SEED_KV, mc.kv_sigma, 50)
        lg = torch.empty((4, mc.vocab), dtype=torch.float32, device=DEV)
        am = torch.empty(4, dtype=torch.int32, device=DEV)
        m.decode_step(toks, pos, kv, lg, am)
        torch.cuda.synchronize()
        outs.append(lg.cpu().numpy().copy())
    assert np.array_equal(outs[0], outs[1])
    kv.close()


def test_load_weights_equals_init_random():
    """Weights passed in from host buffers (logical layout) re-tile to the
    same device bytes as the seeded fill: identical logits."""
    from persistent_decode_megakernel_sm_b200 import Megakernel, mk
    mc = synth.preset("tiny", gain_sigma=0.1, layers=1)
    a = gpu_model(mc)
    b = Megakernel(mc, device=0)
    H, V, hd, Hq, G, I = mc.hidden, mc.vocab, mc.head_dim, mc.n_q_heads, mc.n_kv_heads, mc.ffn
    keep = []

    def T(kind, layer, rows, cols, sigma, gain=False):
        arr = synth.bf16_gain(mc.seed, kind, layer, rows * cols, sigma) if gain else \
            synth.bf16_normal(mc.seed, kind, layer, 0, (rows, cols), sigma)
        arr = np.ascontiguousarray(arr)
        keep.append(arr)
        return mk.mk_tensor_src(kind, layer, 0, rows, cols, arr.ctypes.data, None, 0)

    ts = [T(synth.EMBED, 0, V, H, mc.w_sigma), T(synth.FINAL_NORM, 0, 1, H, mc.gain_sigma, True),
          T(synth.LM_HEAD, 0, V, H, mc.w_sigma)]
    for l in range(mc.layers):
        ts += [T(synth.ATTN_NORM, l, 1, H, mc.gain_sigma, True), T(synth.FFN_NORM, l, 1, H, mc.gain_sigma, True),
               T(synth.WQKV, l, (Hq + 2 * G) * hd, H, mc.w_sigma), T(synth.WO, l, H, Hq * hd, mc.w_sigma),
               T(synth.WGATE, l, I, H, mc.w_sigma), T(synth.WUP, l, I, H, mc.w_sigma),
               T(synth.WDOWN, l, H, I, mc.w_sigma)]
    b.load_weights(ts)
    outs = []
    for m in (a, b):
        kv = m.kv_cache(2, mc.max_ctx)
        kv.fill_random(synth.SEED_KV, mc.kv_sigma, 30)
        lg = torch.empty((2, V), dtype=torch.float32, device=DEV)
        am = torch.empty(2, dtype=torch.int32, device=DEV)
        m.decode_step(_t([11, 12]), _t([30, 29]), kv, lg, am)
        torch.cuda.synchronize()
        outs.append(lg.cpu().numpy().copy())
        kv.close()
    assert np.array_equal(outs[0], outs[1])
    a.close()
    b.close()


def test_device_bounds_error_and_reset(tiny):
    from persistent_decode_megakernel_sm_b200 import mk
    mc, m = tiny
    kv = m.kv_cache(1, mc.max_ctx)
    lg = torch.empty((1, mc.vocab), dtype=torch.float32, device=DEV)
    am = torch.empty(1, dtype=torch.int32, device=DEV)
    m.decode_step(_t([mc.vocab + 5]), _t([3]), kv, lg, am)  # token out of range, checked on the device
    torch.cuda.synchronize()
    assert m.sync_status() == mk.MK_ERR_DEVICE_BOUNDS
    with pytest.raises(mk.MkError) as e:
        m.decode_step(_t([1]), _t([3]), kv, lg, am)
    assert e.value.code == mk.MK_ERR_STATE
    m.reset()
    m.decode_step(_t([1]), _t([3]), kv, lg, am)
    torch.cuda.synchronize()
    assert m.sync_status() == 0
    kv.close()


def test_dependency_timeout_returns_status(tiny):
    """A wait on a counter that nothing signals ends after the limit with
    MK_ERR_DEVICE_TIMEOUT; the context stays usable after mk_reset."""
    from persistent_decode_megakernel_sm_b200 import mk
    mc, m = tiny
    kv = m.kv_cache(1, mc.max_ctx)
    lg = torch.empty((1, mc.vocab), dtype=torch.float32, device=DEV)
    am = torch.empty(1, dtype=torch.int32, device=DEV)
    m.inject_stall(20_000_000)  # 20 ms
    m.decode_step(_t([1]), _t([3]), kv, lg, am)
    torch.cuda.synchronize()
    assert m.sync_status() == mk.MK_ERR_DEVICE_TIMEOUT
    m.reset()
    m.decode_step(_t([1]), _t([3]), kv, lg, am)
    torch.cuda.synchronize()
    assert m.sync_status() == 0
    kv.close()


def test_host_argument_errors(tiny):
    from persistent_decode_megakernel_sm_b200 import mk
    mc, m = tiny
    kv = m.kv_cache(2, mc.max_ctx)
    am = torch.empty(8, dtype=torch.int32, device=DEV)
    with pytest.raises(mk.MkError):
        m.decode_step(_t([1, 2, 3]), _t([1, 2, 3]), kv, None, am)  # B > kv max_seqs
    with pytest.raises(mk.MkError):
        m.verify(_t([1] * 8), mc.max_ctx - 4, kv, None, am, am)   # positions past the cache
    kv.close()


def test_task_trace_same_results_and_records(tiny):
    """A step with the task trace on (the instrumented kernel instance) gives
    bit-identical logits to the plain instance, and writes one record per
    task: begin <= dependency met <= end, on every CTA."""
    from persistent_decode_megakernel_sm_b200 import trace
    mc, m = tiny
    kv = m.kv_cache(2, mc.max_ctx)
    toks, pos = _t([9, 10]), _t([40, 33])
    outs = []
    for traced in (False, True):
        kv.fill_random(synth.SEED_KV, mc.kv_sigma, 40)
        lg = torch.empty((2, mc.vocab), dtype=torch.float32, device=DEV)
        am = torch.empty(2, dtype=torch.int32, device=DEV)
        if traced:
            tr = trace.record(m, kv, toks, pos, lg, am, cap=64)
        else:
            m.decode_step(toks, pos, kv, lg, am)
            torch.cuda.synchronize()
        outs.append(lg.cpu().numpy().copy())
    assert np.array_equal(outs[0], outs[1])
    assert m.sync_status() == 0
    valid = tr[:, :, 2] > 0
    assert valid[:, 0].all()  # every CTA ran at least its first task
    tb, td, te = tr[:, :, 0][valid], tr[:, :, 1][valid], tr[:, :, 2][valid]
    assert (tb <= td).all() and (td <= te).all()
    for c in range(tr.shape[0]):  # each CTA runs its tasks in phase order
        ph = tr[c, :, 6][valid[c]] >> 16
        assert (np.diff(ph) >= 0).all(), c
    s = trace.summarize(tr)
    assert s["step_us"] > 0 and 0.0 < s["compute_fraction"] <= 1.0
    walls = [p["wall_us"] for p in s["phases"].values()]
    assert min(walls) >= 0 and sum(walls) > 0
    kv.close()
