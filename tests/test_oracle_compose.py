"""The oracle's whole decode step against an independent composition of the
textbook definition, written here in float64 numpy from the seeded weights.

The building blocks of the oracle are pinned one by one elsewhere; this pins
their composition: a dropped residual, a norm gain applied to the wrong
phase, RoPE at the wrong position, the new position's K/V not rounded to bf16
or left out of the attention, a mis-indexed or missing expert, a routed
weight that is not renormalised, or latent attention with a swapped
up-projection all change the logits here by far more than the tolerance.
Source of the definition: "700 TPS on Kimi K3: A Case for TPU Megakernels",
sections "Why megakernels?" (the megakernel evaluates the ordinary decoder
step) and "Our Kimi K3 megakernel" (attention, router, shared expert, routed
experts; MLA layers)."""
import numpy as np
import pytest
import torch

import oracle
import synth


def _w(mc, kind, layer, expert, rows, cols, sigma=None):
    s = mc.w_sigma if sigma is None else sigma
    return synth.bf16_to_f32(synth.bf16_normal(mc.seed, kind, layer, expert, (rows, cols), s)).astype(np.float64)


def _w_expert(mc, kind, layer, expert, rows, cols):
    if not mc.expert_fp8:
        return _w(mc, kind, layer, expert, rows, cols)
    codes = synth.e4m3_normal(mc.seed, kind, layer, expert, (rows, cols))
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy().astype(np.float64)
    nbr, nbc = -(-rows // 128), -(-cols // 128)
    sc = synth.block_scales(mc.seed, kind, layer, expert, nbr * nbc, mc.fp8_block_base).reshape(nbr, nbc)
    return vals * np.kron(sc.astype(np.float64), np.ones((128, 128)))[:rows, :cols]


def _gain(mc, kind, layer, n):
    return synth.bf16_to_f32(synth.bf16_gain(mc.seed, kind, layer, n, mc.gain_sigma)).astype(np.float64)


def _rmsnorm(x, g, eps):
    return x / np.sqrt(np.mean(x * x) + eps) * g


def _rope(v, pos, theta):
    d = v.shape[-1]
    half = d // 2
    inv = theta ** (-2.0 * np.arange(half) / d)
    ang = pos * inv
    c, s = np.cos(ang), np.sin(ang)
    a, b = v[..., :half], v[..., half:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def _bf16(v):
    """Round float64 to the nearest bf16 value (ties to even)."""
    m, e = np.frexp(v)
    return np.ldexp(np.round(m * 256.0) / 256.0, e)


def _softmax(s):
    p = np.exp(s - s.max())
    return p / p.sum()


def _silu(z):
    return z / (1.0 + np.exp(-z))


def _swiglu(mc, kinds, layer, expert, h, width, expert_weights):
    get = _w_expert if expert_weights else _w
    g = get(mc, kinds[0], layer, expert, width, mc.hidden) @ h
    u = get(mc, kinds[1], layer, expert, width, mc.hidden) @ h
    return get(mc, kinds[2], layer, expert, mc.hidden, width) @ (_silu(g) * u)


def _bits(a):
    return synth.bf16_to_f32(np.ascontiguousarray(a)).astype(np.float64)


def _step(mc, cache, seq, tok, pos):
    """One decode step of one sequence; `cache` holds the oracle's bf16 cache
    before the step.  Returns (logits, router picks per layer)."""
    H, L = mc.hidden, mc.layers
    x = _bits(synth.bf16_normal(mc.seed, synth.EMBED, 0, 0, (mc.vocab, H), mc.w_sigma)[tok])
    picks = []
    for l in range(L):
        h = _rmsnorm(x, _gain(mc, synth.ATTN_NORM, l, H), mc.rms_eps)
        if not mc.mla:
            Hq, G, d = mc.n_q_heads, mc.n_kv_heads, mc.head_dim
            qkv = _w(mc, synth.WQKV, l, 0, (Hq + 2 * G) * d, H) @ h
            q = _rope(qkv[:Hq * d].reshape(Hq, d), pos, mc.rope_theta)
            k = _bf16(_rope(qkv[Hq * d:(Hq + G) * d].reshape(G, d), pos, mc.rope_theta))
            v = _bf16(qkv[(Hq + G) * d:].reshape(G, d))
            kk, vv = cache
            o = np.zeros((Hq, d))
            for hq in range(Hq):
                g = hq // (Hq // G)
                K = np.vstack([_bits(kk[l, seq, g, :pos]), k[g][None]])
                V = np.vstack([_bits(vv[l, seq, g, :pos]), v[g][None]])
                o[hq] = _softmax(K @ q[hq] / np.sqrt(d)) @ V
            x = x + _w(mc, synth.WO, l, 0, H, Hq * d) @ o.reshape(-1)
        else:
            Hq, dn, dr, R = mc.n_q_heads, mc.head_dim, mc.rope_dim, mc.kv_lora_rank
            dv = dn
            q = (_w(mc, synth.MLA_WQ, l, 0, Hq * (dn + dr), H) @ h).reshape(Hq, dn + dr)
            ckr = _w(mc, synth.MLA_WDKV, l, 0, R + dr, H) @ h
            q_rope = _rope(q[:, dn:], pos, mc.rope_theta)
            row = _bf16(np.concatenate([ckr[:R], _rope(ckr[R:], pos, mc.rope_theta)]))
            lat = np.vstack([_bits(cache[l, seq, :pos]), row[None]])
            Wuk = _w(mc, synth.MLA_WUK, l, 0, Hq * dn, R)
            Wuv = _w(mc, synth.MLA_WUV, l, 0, Hq * dv, R)
            o = np.zeros((Hq, dv))
            for hq in range(Hq):
                k_nope = lat[:, :R] @ Wuk[hq * dn:(hq + 1) * dn].T      # per-position keys, explicit
                s = (k_nope @ q[hq, :dn] + lat[:, R:] @ q_rope[hq]) / np.sqrt(dn + dr)
                values = lat[:, :R] @ Wuv[hq * dv:(hq + 1) * dv].T       # per-position values, explicit
                o[hq] = _softmax(s) @ values
            x = x + _w(mc, synth.WO, l, 0, H, Hq * dv) @ o.reshape(-1)
        h = _rmsnorm(x, _gain(mc, synth.FFN_NORM, l, H), mc.rms_eps)
        if mc.n_routed == 0:
            x = x + _swiglu(mc, (synth.WGATE, synth.WUP, synth.WDOWN), l, 0, h, mc.ffn, False)
        else:
            lg = _w(mc, synth.ROUTER, l, 0, mc.n_routed, H, mc.router_sigma) @ h
            p = _softmax(lg)
            sel = np.argsort(-lg, kind="stable")[:mc.top_k]
            w = p[sel] / p[sel].sum()
            picks.append(list(sel))
            y = np.zeros(H)
            for j in range(mc.n_shared):
                y += _swiglu(mc, (synth.SH_GATE, synth.SH_UP, synth.SH_DOWN), l, j, h, mc.expert_ffn, True)
            for j, e in enumerate(sel):
                y += w[j] * _swiglu(mc, (synth.EX_GATE, synth.EX_UP, synth.EX_DOWN), l, int(e), h, mc.expert_ffn,
                                    True)
            x = x + y
    hf = _rmsnorm(x, _gain(mc, synth.FINAL_NORM, 0, H), mc.rms_eps)
    return _w(mc, synth.LM_HEAD, 0, 0, mc.vocab, H) @ hf, picks


@pytest.mark.parametrize("name", ["tiny", "tiny_moe", "tiny_mla"])
def test_oracle_step_equals_textbook_composition(name):
    mc = synth.preset(name, gain_sigma=0.1, max_seqs=2)
    orc = oracle.OracleModel(mc)
    orc.kv_fill_synthetic(synth.SEED_KV, 24)
    before = orc.kv_arrays()
    cache = tuple(a.copy() for a in before) if isinstance(before, tuple) else before.copy()
    toks, pos = [17, 1500], [24, 9]
    ref = orc.step(toks, pos)
    for b in range(2):
        want, picks = _step(mc, cache, b, toks[b], pos[b])
        got = ref["logits"][b]
        assert np.max(np.abs(got - want)) <= 1e-9 * np.max(np.abs(want)), (name, b)
        for l, sel in enumerate(picks):
            assert list(ref["router_idx"][l, b]) == sel, (name, b, l)
