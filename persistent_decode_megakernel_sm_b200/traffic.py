"""Algorithmic bytes of one decode or verify step: what the method must move
between HBM and the SMs, the numerator of the HBM roofline.

Counted per step: every weight the step needs once (for MoE layers the
router, the shared experts and only the union of routed experts the step's
rows picked), the embedding rows of the step's tokens, the cached KV (or
compressed latent) rows attended, read once per sequence even when several
query positions attend them (verify), the rows the step appends, and the
logits written.  fp8 matrices count one byte per weight plus one fp32 scale
per 128 x 128 block.  Activations and scratch that stay on chip or in L2 are
not counted."""
from __future__ import annotations


def mat_bytes(rows: int, cols: int, fp8: bool = False) -> int:
    if not fp8:
        return rows * cols * 2
    return rows * cols + (-(-rows // 128)) * (-(-cols // 128)) * 4


def expert_bytes(mc) -> int:
    """One expert's gate, up and down matrices."""
    f8 = bool(mc.expert_fp8)
    return 2 * mat_bytes(mc.expert_ffn, mc.hidden, f8) + mat_bytes(mc.hidden, mc.expert_ffn, f8)


def router_unions(mc, idx) -> list[int]:
    """Per layer, how many distinct routed experts a step's rows picked, from
    a router trace `idx` of shape [layers, rows, top_k]."""
    a = idx.cpu().numpy() if hasattr(idx, "cpu") else idx
    return [len(set(a[l].reshape(-1).tolist())) for l in range(mc.layers)]


def step_bytes(mc, pos0, Q: int = 1, unions=None, write_logits: bool = True) -> int:
    """Algorithmic bytes of one step.  pos0: first position of each sequence
    (positions 0..p-1 are attended from the cache); Q positions per sequence;
    unions[l]: routed experts read at layer l (default: the most the rows can
    pick)."""
    H, L, V = mc.hidden, mc.layers, mc.vocab
    Hq, d = mc.n_q_heads, mc.head_dim
    M = len(pos0) * Q
    total = mat_bytes(V, H) + H * 2 + M * H * 2          # LM head, final norm, embedding rows
    for l in range(L):
        total += 2 * H * 2                                # norm gains
        if mc.mla:
            R, dr = mc.kv_lora_rank, mc.rope_dim
            total += (mat_bytes(Hq * (d + dr) + R + dr, H) + mat_bytes(Hq * R, d) + mat_bytes(Hq * d, R)
                      + mat_bytes(H, Hq * d))
        else:
            total += mat_bytes((Hq + 2 * mc.n_kv_heads) * d, H) + mat_bytes(H, Hq * d)
        if mc.n_routed == 0:
            total += mat_bytes(2 * mc.ffn, H) + mat_bytes(H, mc.ffn)
        else:
            u = unions[l] if unions is not None else min(mc.n_routed, M * mc.top_k)
            total += mat_bytes(mc.n_routed, H) + (mc.n_shared + u) * expert_bytes(mc)
    kvt = (mc.kv_lora_rank + mc.rope_dim) * 2 if mc.mla else 2 * mc.n_kv_heads * d * 2
    total += sum(int(p) for p in pos0) * kvt * L          # cached rows read
    total += M * kvt * L                                  # new rows written
    if write_logits:
        total += M * V * 4
    return total
