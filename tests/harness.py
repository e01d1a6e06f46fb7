"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the fp64 oracle on the same seeded inputs, and compare."""
from __future__ import annotations

import numpy as np

import synth

# Tolerances of the decode-step contract: bf16 weights with fp32 accumulation
# must give max |dlogit| <= 2e-2 absolute or <= 1e-2 relative to max |logit|;
# fp8 expert weights 5e-2.  Integer outputs (router indices, greedy tokens) are
# exact unless the oracle's own margin at that decision is below DELTA
# (a near-tie, where both choices are correct to the arithmetic's precision).
ATOL_BF16, RTOL_BF16, ATOL_FP8 = 2e-2, 1e-2, 5e-2
DELTA = 1e-3


def logits_close(gpu: np.ndarray, ref: np.ndarray, fp8: bool = False):
    err = float(np.max(np.abs(gpu.astype(np.float64) - ref)))
    scale = float(np.max(np.abs(ref)))
    atol = ATOL_FP8 if fp8 else ATOL_BF16
    ok = err <= atol or err <= RTOL_BF16 * scale
    return ok, err, scale


def argmax_agrees(gpu_tok: int, ref_logits: np.ndarray, ref_tok: int, ref_margin: float) -> bool:
    """Exact match, or a near-tie in the oracle where the GPU's token is
    within DELTA of the oracle's maximum (both are valid greedy choices)."""
    if gpu_tok == ref_tok:
        return True
    return ref_margin < DELTA and ref_logits[ref_tok] - ref_logits[gpu_tok] < DELTA


def gpu_model(mc, max_batch: int = 8):
    from persistent_decode_megakernel_sm_b200 import Megakernel
    m = Megakernel(mc, device=0, max_batch=max_batch)
    m.init_random(mc.seed, mc.w_sigma, mc.router_sigma, mc.gain_sigma, mc.fp8_block_base)
    return m


def tokens_at(mc, seq: int, positions):
    return synth.seq_tokens(synth.SEED_TOKENS, seq, positions, mc.vocab)
