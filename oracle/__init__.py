"""TEST INFRASTRUCTURE ONLY: ctypes bindings to the fp64 CPU oracle.

Only the test-suite, the smoke check and the bench's CPU-baseline leg may
import this package.  The product library never loads it.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import numpy as np

from . import build as _build

_lib: Optional[ctypes.CDLL] = None


class OrcCfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "ffn", "vocab",
        "n_routed", "n_shared", "top_k", "expert_ffn", "kv_lora_rank", "rope_dim", "expert_fp8",
        "max_seqs", "max_ctx")] + [(n, ctypes.c_double) for n in (
        "rope_theta", "rms_eps", "w_sigma", "router_sigma", "gain_sigma", "kv_sigma", "fp8_block_base")] + [
        ("seed", ctypes.c_uint64)]


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(_build.build())
        vp, i32, dbl = ctypes.c_void_p, ctypes.c_int32, ctypes.c_double
        L.orc_create.argtypes = [ctypes.POINTER(OrcCfg)]
        L.orc_create.restype = vp
        L.orc_destroy.argtypes = [vp]
        for f in ("orc_kv_k", "orc_kv_v", "orc_kv_lat"):
            getattr(L, f).argtypes = [vp]
            getattr(L, f).restype = vp
        L.orc_kv_fill_synthetic.argtypes = [vp, ctypes.c_uint64, i32]
        L.orc_step.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int,
                               vp, dbl, vp]
        L.orc_step.restype = ctypes.c_int
        L.orc_forward_full.argtypes = [ctypes.POINTER(OrcCfg), ctypes.c_int, vp, vp]
        L.orc_forward_full.restype = ctypes.c_int
        L.orc_rmsnorm.argtypes = [ctypes.c_int, vp, vp, dbl, vp]
        L.orc_rope_apply.argtypes = [ctypes.c_int, vp, i32, dbl]
        L.orc_softmax.argtypes = [ctypes.c_int, vp, vp]
        L.orc_attention_head.argtypes = [ctypes.c_int, ctypes.c_int, vp, vp, vp, dbl, vp]
        L.orc_silu.argtypes = [dbl]
        L.orc_silu.restype = dbl
        L.orc_router_select.argtypes = [ctypes.c_int, ctypes.c_int, vp, vp, vp, vp]
        L.orc_router_select_follow.argtypes = [ctypes.c_int, ctypes.c_int, vp, vp, dbl, vp, vp, vp]
        L.orc_router_select_follow.restype = ctypes.c_int
        L.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_value.restype = dbl
        L.orc_bf16_round.argtypes = [dbl]
        L.orc_bf16_round.restype = ctypes.c_uint16
        L.orc_matvec_dense.argtypes = [ctypes.c_int64, ctypes.c_int64, vp, ctypes.c_int, vp, vp]
        L.orc_swiglu_dense.argtypes = [ctypes.c_int, ctypes.c_int, vp, vp, vp, ctypes.c_int, vp, vp]
        L.orc_moe_ffn_dense.argtypes = [ctypes.c_int] * 5 + [vp] * 11
        L.orc_mla_attention.argtypes = [ctypes.c_int] * 6 + [vp] * 4 + [ctypes.c_int, vp]
        L.orc_accept.argtypes = [ctypes.c_int, vp, vp]
        L.orc_accept.restype = i32
        L.orc_num_threads.restype = ctypes.c_int
        L.orc_argmax.argtypes = [ctypes.c_int64, vp, vp]
        L.orc_argmax.restype = i32
        L.orc_gqa_attend_row.argtypes = [vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp]
        L.orc_debug_mat_row.argtypes = [ctypes.POINTER(OrcCfg), ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32,
                                        ctypes.c_int64, ctypes.c_int64, ctypes.c_int, dbl, ctypes.c_int64, vp]
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle buffers must be C-contiguous"
    return a.ctypes.data


def _d(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def make_cfg(mc) -> OrcCfg:
    c = OrcCfg()
    for name, _ in OrcCfg._fields_:
        setattr(c, name, getattr(mc, name))
    return c


# --------------------------------------------------------------------------
# building blocks
# --------------------------------------------------------------------------

def rmsnorm(x, g, eps):
    x, g = _d(x), _d(g)
    y = np.empty_like(x)
    lib().orc_rmsnorm(len(x), _p(x), _p(g), eps, _p(y))
    return y


def rope(x, pos, theta=1e4):
    y = _d(x).copy()
    lib().orc_rope_apply(len(y), _p(y), int(pos), theta)
    return y


def softmax(x):
    x = _d(x)
    y = np.empty_like(x)
    lib().orc_softmax(len(x), _p(x), _p(y))
    return y


def attention_head(q, K, V, scale):
    q, K, V = _d(q), _d(K), _d(V)
    out = np.empty(K.shape[1], dtype=np.float64)
    lib().orc_attention_head(K.shape[0], K.shape[1], _p(q), _p(K), _p(V), scale, _p(out))
    return out


def silu(z: float) -> float:
    return lib().orc_silu(z)


def router_select(logits, k):
    lg = _d(logits)
    idx = np.empty(k, dtype=np.int32)
    w = np.empty(k, dtype=np.float64)
    mg = np.empty(1, dtype=np.float64)
    lib().orc_router_select(len(lg), k, _p(lg), _p(idx), _p(w), _p(mg))
    return idx, w, float(mg[0])


def router_select_follow(logits, k, follow, delta):
    """Router selection with the near-tie protocol: `follow` is adopted only
    when the oracle's own k-th / (k+1)-th gap is below delta and `follow` is a
    valid choice at that tolerance.  Returns (idx, w, margin, followed)."""
    lg = _d(logits)
    fo = np.ascontiguousarray(follow, dtype=np.int32)
    idx = np.empty(k, dtype=np.int32)
    w = np.empty(k, dtype=np.float64)
    mg = np.empty(1, dtype=np.float64)
    fl = lib().orc_router_select_follow(len(lg), k, _p(lg), _p(fo), delta, _p(idx), _p(w), _p(mg))
    return idx, w, float(mg[0]), bool(fl)


def e4m3_value(code: int) -> float:
    return lib().orc_e4m3_value(code)


def bf16_round(v: float) -> int:
    return lib().orc_bf16_round(v)


def matvec(W, x):
    W, x = _d(W), _d(np.atleast_2d(x))
    y = np.empty((x.shape[0], W.shape[0]), dtype=np.float64)
    lib().orc_matvec_dense(W.shape[0], W.shape[1], _p(W), x.shape[0], _p(x), _p(y))
    return y


def swiglu(Wg, Wu, Wd, x):
    Wg, Wu, Wd, x = _d(Wg), _d(Wu), _d(Wd), _d(np.atleast_2d(x))
    y = np.empty((x.shape[0], Wd.shape[0]), dtype=np.float64)
    lib().orc_swiglu_dense(Wg.shape[1], Wg.shape[0], _p(Wg), _p(Wu), _p(Wd), x.shape[0], _p(x), _p(y))
    return y


def moe_ffn(Wr, g, u, d, shg, shu, shd, x, k):
    E, I, H = g.shape
    ns = shg.shape[0]
    args = [_d(a) for a in (Wr, g, u, d, shg, shu, shd, x)]
    y = np.empty(H, dtype=np.float64)
    idx = np.empty(k, dtype=np.int32)
    w = np.empty(k, dtype=np.float64)
    lib().orc_moe_ffn_dense(H, I, E, k, ns, *[_p(a) for a in args], _p(y), _p(idx), _p(w))
    return y, idx, w


def mla_attention(q_full, lat, Wuk, Wuv, Hq, dn, dr, dv, R, absorbed):
    q_full, lat, Wuk, Wuv = _d(q_full), _d(lat), _d(Wuk), _d(Wuv)
    out = np.empty(Hq * dv, dtype=np.float64)
    T = lat.shape[0]
    lib().orc_mla_attention(Hq, dn, dr, dv, R, T, _p(q_full), _p(lat), _p(Wuk), _p(Wuv), int(absorbed), _p(out))
    return out


def accept(tokens, greedy) -> int:
    t = np.ascontiguousarray(tokens, dtype=np.int32)
    g = np.ascontiguousarray(greedy, dtype=np.int32)
    return lib().orc_accept(len(t), _p(t), _p(g))


def argmax(x):
    x = _d(x)
    mg = np.empty(1, dtype=np.float64)
    i = lib().orc_argmax(len(x), _p(x), _p(mg))
    return int(i), float(mg[0])


def debug_mat_row(mc, kind, layer, expert, rows, cols, r, fp8=False, sigma=None):
    cfg = make_cfg(mc)
    out = np.empty(cols, dtype=np.float64)
    lib().orc_debug_mat_row(ctypes.byref(cfg), kind, layer, expert, rows, cols, int(fp8),
                            mc.w_sigma if sigma is None else sigma, r, _p(out))
    return out


def num_threads() -> int:
    return lib().orc_num_threads()


# --------------------------------------------------------------------------
# model
# --------------------------------------------------------------------------

class OracleModel:
    """fp64 decoder with seeded synthetic weights and a host bf16 KV cache."""

    def __init__(self, mc):
        self.mc = mc
        self.cfg = make_cfg(mc)
        self.h = lib().orc_create(ctypes.byref(self.cfg))
        if not self.h:
            raise MemoryError("oracle: cache allocation failed")

    def close(self):
        if getattr(self, "h", None) and _lib is not None:
            _lib.orc_destroy(self.h)
            self.h = None

    def __del__(self):
        self.close()

    def attend_row(self, layer, seq, pos, q):
        """GQA attention of one query row (all heads) over cached positions 0..pos."""
        mc = self.mc
        q = _d(q).reshape(-1)
        out = np.empty(mc.n_q_heads * mc.head_dim, dtype=np.float64)
        lib().orc_gqa_attend_row(self.h, layer, seq, pos, _p(q), _p(out))
        return out

    def kv_fill_synthetic(self, kv_seed: int, T: int):
        lib().orc_kv_fill_synthetic(self.h, kv_seed, T)

    def kv_arrays(self):
        mc = self.mc
        if mc.mla:
            n = mc.layers * mc.max_seqs * mc.max_ctx * (mc.kv_lora_rank + mc.rope_dim)
            p = lib().orc_kv_lat(self.h)
            lat = np.ctypeslib.as_array(ctypes.cast(p, ctypes.POINTER(ctypes.c_uint16)), shape=(n,))
            return lat.reshape(mc.layers, mc.max_seqs, mc.max_ctx, mc.kv_lora_rank + mc.rope_dim)
        n = mc.layers * mc.max_seqs * mc.n_kv_heads * mc.max_ctx * mc.head_dim
        shape = (mc.layers, mc.max_seqs, mc.n_kv_heads, mc.max_ctx, mc.head_dim)
        k = np.ctypeslib.as_array(ctypes.cast(lib().orc_kv_k(self.h), ctypes.POINTER(ctypes.c_uint16)), shape=(n,))
        v = np.ctypeslib.as_array(ctypes.cast(lib().orc_kv_v(self.h), ctypes.POINTER(ctypes.c_uint16)), shape=(n,))
        return k.reshape(shape), v.reshape(shape)

    def set_kv(self, gpu_logical: np.ndarray):
        """Take a cache written elsewhere as this model's input (the layout of
        the GPU library's logical copy-out: GQA keys then values, or latent
        rows), for contexts prefilled by the GPU."""
        flat = np.ascontiguousarray(gpu_logical).view(np.uint16).reshape(-1)
        if self.mc.mla:
            lat = self.kv_arrays()
            assert flat.size == lat.size, (flat.size, lat.size)
            lat.reshape(-1)[:] = flat
        else:
            k, v = self.kv_arrays()
            assert flat.size == k.size + v.size, (flat.size, k.size, v.size)
            k.reshape(-1)[:] = flat[:k.size]
            v.reshape(-1)[:] = flat[k.size:]

    def step(self, tokens, pos0, Q: int = 1, want_logits: bool = True, absorbed: bool = False,
             follow=None, delta: float = 1e-3):
        """One decode (Q=1) or verify (Q>1) step for S = len(pos0) sequences.
        follow: router choices [layers][S*Q][top_k] of the implementation
        under test, adopted only at near-ties (margin < delta)."""
        mc = self.mc
        tokens = np.ascontiguousarray(tokens, dtype=np.int32).reshape(-1)
        pos0 = np.ascontiguousarray(pos0, dtype=np.int32).reshape(-1)
        S = len(pos0)
        M = S * Q
        assert len(tokens) == M
        logits = np.empty((M, mc.vocab), dtype=np.float64) if want_logits else None
        amax = np.empty(M, dtype=np.int32)
        amargin = np.empty(M, dtype=np.float64)
        k = max(mc.top_k, 1)
        ridx = np.zeros((mc.layers, M, k), dtype=np.int32)
        rw = np.zeros((mc.layers, M, k), dtype=np.float64)
        rmargin = np.full((mc.layers, M), np.inf, dtype=np.float64)
        fo = None
        if follow is not None and mc.n_routed:
            fo = np.ascontiguousarray(follow, dtype=np.int32).reshape(mc.layers, M, k)
        followed = np.zeros((mc.layers, M), dtype=np.int32)
        rc = lib().orc_step(self.h, S, Q, _p(tokens), _p(pos0), _p(logits), _p(amax), _p(amargin),
                            _p(ridx), _p(rw), _p(rmargin), int(absorbed), _p(fo), float(delta), _p(followed))
        if rc != 0:
            raise ValueError("oracle: bad step arguments")
        return dict(logits=logits, argmax=amax, argmax_margin=amargin,
                    router_idx=ridx, router_w=rw, router_margin=rmargin, router_followed=followed.astype(bool))


def forward_full(mc, tokens):
    cfg = make_cfg(mc)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    logits = np.empty((len(tokens), mc.vocab), dtype=np.float64)
    rc = lib().orc_forward_full(ctypes.byref(cfg), len(tokens), _p(tokens), _p(logits))
    assert rc == 0
    return logits
