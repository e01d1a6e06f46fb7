"""Seeded synthetic inputs shared by the GPU path's tests/bench and the oracle.

This package holds the workload definitions (model shapes and the input
recipe) and ctypes bindings to libsynth.so, the host copy of the counter-based
generator in synth.h.  It contains none of the decoder's arithmetic.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
from typing import Optional

import numpy as np

from . import build as _build

# Tensor kinds (must match synth.h).
EMBED, ATTN_NORM, WQKV, WO, FFN_NORM, WGATE, WUP, WDOWN, ROUTER = 1, 2, 3, 4, 5, 6, 7, 8, 9
SH_GATE, SH_UP, SH_DOWN, EX_GATE, EX_UP, EX_DOWN = 10, 11, 12, 13, 14, 15
FINAL_NORM, LM_HEAD, MLA_WQ, MLA_WDKV, MLA_WUK, MLA_WUV = 16, 17, 18, 19, 20, 21
FP8_SCALE, KV_K, KV_V, KV_LAT, TOKENS, PROPOSALS = 22, 23, 24, 25, 26, 27

# Seeds of the input recipe.
SEED_WEIGHTS, SEED_TOKENS, SEED_PROPOSALS, SEED_KV = 1, 2, 3, 4

_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        u64, u32, vp = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_void_p
        L.syn_fill_bf16_normal.argtypes = [u64, u32, u32, u32, u64, u64, ctypes.c_double, vp]
        L.syn_fill_bf16_gain.argtypes = [u64, u32, u32, u64, ctypes.c_double, vp]
        L.syn_fill_e4m3_normal.argtypes = [u64, u32, u32, u32, u64, u64, vp]
        L.syn_fill_block_scales.argtypes = [u64, u32, u32, u32, u64, ctypes.c_float, vp]
        L.syn_fill_tokens.argtypes = [u64, u32, u64, u64, u32, vp]
        L.syn_e4m3_encode.argtypes = [ctypes.c_float]
        L.syn_e4m3_encode.restype = ctypes.c_uint8
        L.syn_bf16_encode.argtypes = [ctypes.c_float]
        L.syn_bf16_encode.restype = ctypes.c_uint16
        L.syn_raw_u64.argtypes = [u64, u32, u32, u32, u64]
        L.syn_raw_u64.restype = u64
        _lib = L
    return _lib


@dataclasses.dataclass
class ModelConfig:
    """Shape of a synthetic decoder and its input recipe."""
    name: str
    layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    rope_theta: float = 1e4
    rms_eps: float = 1e-6
    n_routed: int = 0
    n_shared: int = 0
    top_k: int = 0
    expert_ffn: int = 0
    kv_lora_rank: int = 0
    rope_dim: int = 0
    expert_fp8: int = 0
    max_seqs: int = 8
    max_ctx: int = 256
    w_sigma: float = 0.02
    router_sigma: float = 0.0
    gain_sigma: float = 0.0
    kv_sigma: float = 0.0
    fp8_block_base: float = 0.02 / 16
    seed: int = SEED_WEIGHTS
    context: int = 0          # pre-filled positions per sequence
    prefill: str = "synthetic"  # "tokens": run the model over seeded tokens; "synthetic": seeded KV values

    def __post_init__(self):
        if self.router_sigma == 0.0:
            self.router_sigma = 1.0 / math.sqrt(self.hidden)
        if self.kv_sigma == 0.0:
            self.kv_sigma = self.w_sigma * math.sqrt(self.hidden)

    @property
    def mla(self) -> bool:
        return self.kv_lora_rank > 0

    def replace(self, **kw) -> "ModelConfig":
        return dataclasses.replace(self, **kw)


def preset(name: str, **overrides) -> ModelConfig:
    """The five workloads of the decode-step study, by name."""
    p = {
        # 2 layers, hidden 256, 4/2 heads x 64, SwiGLU 1024, vocab 4096; 128 prefilled positions, 16 greedy steps.
        "tiny": ModelConfig("tiny", layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=1024,
                            vocab=4096, max_seqs=8, max_ctx=160, context=128, prefill="tokens"),
        # Dense 27B-shaped: 64 layers, hidden 5120, 40/8 heads x 128, SwiGLU 17408, vocab 151936, context 2048.
        "dense27b": ModelConfig("dense27b", layers=64, hidden=5120, n_q_heads=40, n_kv_heads=8, head_dim=128,
                                ffn=17408, vocab=151936, max_seqs=8, max_ctx=2048 + 80, context=2048),
        # MoE: 32 layers, hidden 4096, 32/8 heads x 128, 1 shared + 64 routed experts of width 1408, top-4, vocab 65536.
        "moe": ModelConfig("moe", layers=32, hidden=4096, n_q_heads=32, n_kv_heads=8, head_dim=128, ffn=0,
                           vocab=65536, n_routed=64, n_shared=1, top_k=4, expert_ffn=1408,
                           max_seqs=8, max_ctx=4096 + 80, context=4096),
        # MLA + fp8 experts: 48 layers, hidden 4096, 32 heads, latent 512 + 64 rope, 1 + 64 experts of 1536, top-8, vocab 131072.
        "mla_fp8": ModelConfig("mla_fp8", layers=48, hidden=4096, n_q_heads=32, n_kv_heads=1, head_dim=128, ffn=0,
                               vocab=131072, n_routed=64, n_shared=1, top_k=8, expert_ffn=1536,
                               kv_lora_rank=512, rope_dim=64, expert_fp8=1, max_seqs=8, max_ctx=8192 + 80,
                               context=8192),
        # Small shapes of the same families, for parity at sizes the oracle finishes in seconds.
        "tiny_moe": ModelConfig("tiny_moe", layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=0,
                                vocab=2048, n_routed=8, n_shared=1, top_k=2, expert_ffn=192,
                                max_seqs=8, max_ctx=96, context=48, gain_sigma=0.1),
        "tiny_mla": ModelConfig("tiny_mla", layers=2, hidden=256, n_q_heads=4, n_kv_heads=1, head_dim=32, ffn=0,
                                vocab=2048, n_routed=8, n_shared=1, top_k=3, expert_ffn=192,
                                kv_lora_rank=64, rope_dim=16, expert_fp8=1, max_seqs=8, max_ctx=96,
                                context=48, gain_sigma=0.1),
    }[name]
    return p.replace(**overrides) if overrides else p


# ---------------------------------------------------------------------------
# host-side fills
# ---------------------------------------------------------------------------

def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def bf16_normal(seed: int, kind: int, layer: int, expert: int, shape, sigma: float, start: int = 0) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    lib().syn_fill_bf16_normal(seed, kind, layer, expert, start, n, sigma, _ptr(out))
    return out.reshape(shape)


def bf16_gain(seed: int, kind: int, layer: int, n: int, sigma: float) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    lib().syn_fill_bf16_gain(seed, kind, layer, n, sigma, _ptr(out))
    return out


def e4m3_normal(seed: int, kind: int, layer: int, expert: int, shape, start: int = 0) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint8)
    lib().syn_fill_e4m3_normal(seed, kind, layer, expert, start, n, _ptr(out))
    return out.reshape(shape)


def block_scales(seed: int, kind: int, layer: int, expert: int, n: int, base: float) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    lib().syn_fill_block_scales(seed, kind, layer, expert, n, base, _ptr(out))
    return out


def tokens(seed: int, n: int, vocab: int, start: int = 0, kind: int = TOKENS) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    lib().syn_fill_tokens(seed, kind, start, n, vocab, _ptr(out))
    return out


def seq_tokens(seed: int, seq: int, positions, vocab: int) -> np.ndarray:
    """Token of sequence `seq` at each position (index seq << 24 | pos)."""
    out = np.empty(len(positions), dtype=np.int32)
    for i, p in enumerate(positions):
        out[i] = tokens(seed, 1, vocab, start=(seq << 24) + int(p))[0]
    return out


def proposals(seed: int, step: int, n: int, vocab: int) -> np.ndarray:
    return tokens(seed, n, vocab, start=step * n, kind=PROPOSALS)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)
