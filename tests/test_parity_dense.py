"""GPU parity of the dense decoder path (C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from harness import argmax_agrees, gpu_model, logits_close, tokens_at

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
    # greedy decode: each side feeds its own argmax
    tok_g = tok_o = int(tokens_at(mc, 0, [mc.context])[0])
    for step in range(16):
        p = mc.context + step
        m.decode_step(_t([tok_g]), _t([p]), kv, logits, am)
        ref = orc.step([tok_o], [p])
        torch.cuda.synchronize()
        g = logits.cpu().numpy()[0]
        ok, err, sc = logits_close(g, ref["logits"][0])
        assert ok, (step, err, sc)
        ga = int(am.item())
        assert ga == int(np.argmax(g)) or g[ga] == g.max()
        assert argmax_agrees(ga, ref["logits"][0], int(ref["argmax"][0]), ref["argmax_margin"][0]), step
        if ga != int(ref["argmax"][0]):
            break  # near-tie: the two greedy chains legitimately diverge here
        tok_g, tok_o = ga, int(ref["argmax"][0])
    assert m.sync_status() == 0
    # KV cache: bf16 values written by both sides
    kk, vv = orc.kv_arrays()
    dev = kv.copy_out().cpu().numpy().view(np.uint16)
    half = dev.size // 2
    n_pos = mc.context + 16
    gk = dev[:half].reshape(kk.shape)[:, :, :, :n_pos]
    gv = dev[half:].reshape(vv.shape)[:, :, :, :n_pos]
    for a, b in ((gk, kk[:, :, :, :n_pos]), (gv, vv[:, :, :, :n_pos])):
        # Both sides round their own K/V to bf16 (fp32 on the GPU, fp64 in the
        # oracle): a value within ~1e-5 of a rounding boundary may land on the
        # neighbouring bf16 code.  Require at most one code apart, and rarely.
        fa = synth.bf16_to_f32(np.ascontiguousarray(a)).astype(np.float64)
        fb = synth.bf16_to_f32(np.ascontiguousarray(b)).astype(np.float64)
        scale = np.max(np.abs(fb))
        ulp = 2.0 ** -7 * np.maximum(np.abs(fa), np.abs(fb))
        assert np.all(np.abs(fa - fb) <= ulp + 1e-3 * scale)
        assert np.mean(a != b) < 0.1
    kv.close()


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
    s = trace.summarize(tr)
    assert s["step_us"] > 0 and 0.0 < s["compute_fraction"] <= 1.0
    kv.close()
