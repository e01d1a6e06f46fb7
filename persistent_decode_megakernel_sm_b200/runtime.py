"""Convenience wrapper over the C ABI for Python callers (argument
marshalling and ownership only; every computation runs in libmk.so)."""
from __future__ import annotations

from typing import Optional

import torch

from . import mk


def desc_from(cfg, max_batch: int = 8) -> mk.mk_model_desc:
    """Build an mk_model_desc from any object with the decoder's shape fields."""
    d = mk.mk_model_desc()
    for name in ("layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "ffn", "vocab", "n_routed", "n_shared",
                 "top_k", "expert_ffn", "kv_lora_rank", "rope_dim", "expert_fp8", "max_ctx"):
        setattr(d, name, int(getattr(cfg, name)))
    d.rope_theta = float(cfg.rope_theta)
    d.rms_eps = float(cfg.rms_eps)
    d.max_batch = int(max_batch)
    return d


class KVCache:
    def __init__(self, model: "Megakernel", max_seqs: int, max_ctx: int):
        self.model = model
        self.h = mk.mk_kv_create(model.h, max_seqs, max_ctx)
        self.max_seqs, self.max_ctx = max_seqs, max_ctx

    def fill_random(self, seed: int, sigma: float, length: int):
        mk.mk_kv_fill_random(self.model.h, self.h, seed, sigma, length)

    def nbytes(self) -> int:
        return mk.mk_kv_bytes(self.h)

    def copy_out(self) -> torch.Tensor:
        out = torch.empty(self.nbytes() // 2, dtype=torch.int16, device=f"cuda:{self.model.device}")
        mk.mk_kv_copy_out(self.model.h, self.h, out)
        return out

    def copy_in(self, src: torch.Tensor):
        """Replace the cache with `src` (device, logical order, nbytes() bytes)."""
        assert src.is_cuda and src.numel() * src.element_size() == self.nbytes()
        mk.mk_kv_copy_in(self.model.h, self.h, src)

    def close(self):
        if self.h:
            mk.mk_kv_destroy(self.h)
            self.h = None


class Megakernel:
    """One decoder model resident on one GPU."""

    def __init__(self, cfg, device: int = 0, max_batch: int = 8):
        self.cfg = cfg
        self.device = device
        self.desc = desc_from(cfg, max_batch)
        self.h = mk.mk_create(self.desc, device)

    def init_random(self, seed: int, w_sigma: float, router_sigma: float, gain_sigma: float, fp8_block_base: float):
        mk.mk_init_random(self.h, seed, w_sigma, router_sigma, gain_sigma, fp8_block_base)

    def load_weights(self, tensors):
        mk.mk_load_weights(self.h, tensors)

    def kv_cache(self, max_seqs: int, max_ctx: int) -> KVCache:
        return KVCache(self, max_seqs, max_ctx)

    def decode_step(self, tokens: torch.Tensor, positions: torch.Tensor, kv: KVCache,
                    logits: Optional[torch.Tensor], argmax: torch.Tensor, stream=None):
        B = tokens.numel()
        mk.mk_decode_step(self.h, tokens, positions, B, kv.h, logits, argmax, stream)

    def decode_step_multikernel(self, tokens: torch.Tensor, positions: torch.Tensor, kv: KVCache,
                                logits: Optional[torch.Tensor], argmax: torch.Tensor, stream=None):
        """The same step as one kernel per phase in a CUDA graph (comparison path)."""
        mk.mk_decode_step_multikernel(self.h, tokens, positions, tokens.numel(), kv.h, logits, argmax, stream)

    def verify(self, tokens: torch.Tensor, position: int, kv: KVCache, logits: Optional[torch.Tensor],
               argmax: torch.Tensor, accepted: torch.Tensor, stream=None):
        mk.mk_verify(self.h, tokens, tokens.numel() - 1, position, kv.h, logits, argmax, accepted, stream)

    def prefill(self, tokens: torch.Tensor, seq: int, start: int, kv: KVCache,
                argmax_last: Optional[torch.Tensor] = None, stream=None):
        """Write the K/V of tokens (positions start ..) of cache sequence seq."""
        mk.mk_prefill(self.h, tokens, tokens.numel(), seq, start, kv.h, argmax_last, stream)

    def spec_generate(self, kv: KVCache, anchor: int, position: int, n_out: int, draft, stream=None):
        """Speculative greedy generation on cache sequence 0 (mk_spec_generate):
        draft(history, max_k) -> proposals.  Returns (tokens, stats)."""
        return mk.mk_spec_generate(self.h, kv.h, anchor, position, n_out, draft, stream)

    def set_router_trace(self, idx: Optional[torch.Tensor], w: Optional[torch.Tensor]):
        mk.mk_set_router_trace(self.h, idx, w)

    def set_trace(self, trace: Optional[torch.Tensor], max_tasks_per_cta: int = 0):
        """trace: int64 CUDA tensor [ctas, max_tasks_per_cta, 8] or None."""
        mk.mk_set_trace(self.h, trace, max_tasks_per_cta)

    def sync_status(self) -> int:
        return mk.mk_sync_status(self.h)

    def reset(self):
        mk.mk_reset(self.h)

    def launch_info(self):
        return mk.mk_launch_info(self.h)

    def weight_bytes(self) -> int:
        return mk.mk_weight_bytes(self.h)

    def inject_stall(self, timeout_ns: int):
        mk.mk_debug_inject_stall(self.h, timeout_ns)

    def close(self):
        if self.h:
            mk.mk_destroy(self.h)
            self.h = None
