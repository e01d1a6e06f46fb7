"""The benchmark's algorithmic byte count (the HBM roofline's numerator),
checked against sums written out by hand for the dense 27B-shaped model and
against properties that hold for any configuration."""
import numpy as np

import synth
from persistent_decode_megakernel_sm_b200.traffic import expert_bytes, mat_bytes, router_unions, step_bytes


def test_dense27b_step_bytes_by_hand():
    mc = synth.preset("dense27b")
    H, V, L = 5120, 151936, 64
    per_layer = (40 + 2 * 8) * 128 * H * 2 + H * 40 * 128 * 2 + 2 * 17408 * H * 2 + H * 17408 * 2 + 2 * H * 2
    weights = L * per_layer + V * H * 2 + H * 2 + H * 2  # layers, LM head, final norm, one embedding row
    p = 2048
    kv = p * 2 * 8 * 128 * 2 * L + 2 * 8 * 128 * 2 * L  # rows read + the row written
    assert step_bytes(mc, [p]) == weights + kv + V * 4
    assert weights == 43835740160


def test_fp8_matrix_counts_block_scales():
    assert mat_bytes(128, 128, fp8=True) == 128 * 128 + 4
    assert mat_bytes(129, 256, fp8=True) == 129 * 256 + 2 * 2 * 4
    assert mat_bytes(3, 5) == 30


def test_moe_unions_bound_and_monotone():
    mc = synth.preset("moe")
    full = step_bytes(mc, [mc.context] * 8)
    u = [min(mc.n_routed, 8 * mc.top_k)] * mc.layers
    assert step_bytes(mc, [mc.context] * 8, 1, u) == full
    fewer = [x - 1 for x in u]
    assert full - step_bytes(mc, [mc.context] * 8, 1, fewer) == mc.layers * expert_bytes(mc)


def test_verify_reads_the_cache_once():
    """Q positions of one sequence read its cached rows once: only the
    appended rows, embedding rows and logits grow with Q."""
    mc = synth.preset("moe")
    u = [8] * mc.layers
    a = step_bytes(mc, [mc.context], 8, u, write_logits=False)
    b = step_bytes(mc, [mc.context], 1, u, write_logits=False)
    kvt = 2 * mc.n_kv_heads * mc.head_dim * 2
    assert a - b == 7 * (kvt * mc.layers + mc.hidden * 2)


def test_router_unions_counts_distinct_experts():
    mc = synth.preset("tiny_moe")
    assert mc.layers == 2 and mc.top_k == 2
    idx = np.zeros((2, 3, 2), dtype=np.int32)
    idx[0] = [[0, 1], [1, 2], [2, 0]]
    idx[1] = [[5, 4], [4, 5], [5, 4]]
    assert router_unions(mc, idx) == [3, 2]
