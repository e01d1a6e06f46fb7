"""The trace summary (persistent_decode_megakernel_sm_b200.trace.summarize),
which the committed SM-idle and per-phase figures come from, checked on a
hand-built record set whose figures follow from the definitions: step span,
per-phase wall time (first dependency met to last end), per-CTA averages,
the idle fraction between tasks, and prefetch records kept out of all of
them."""
import numpy as np
import pytest

from persistent_decode_megakernel_sm_b200.trace import FIELDS, summarize


def _rec(tr, c, k, tb, td, te, typ, epi, phase, layer=0):
    tr[c, k, 0:3] = (tb, td, te)
    tr[c, k, 6] = layer | (phase << 16)
    tr[c, k, 7] = typ * 16 + epi


@pytest.fixture
def trace():
    tr = np.zeros((2, 4, FIELDS), dtype=np.int64)
    # CTA 0: a QKV-like GEMV (phase 0), a prefetch record, an attention item (phase 1)
    _rec(tr, 0, 0, 1000, 1000, 5000, 1, 0, 0)
    _rec(tr, 0, 1, 5000, 5000, 5100, 5, 0, 0)
    _rec(tr, 0, 2, 5100, 6000, 9000, 2, 0, 1)
    # CTA 1: the same two phases, later dependencies
    _rec(tr, 1, 0, 1000, 1500, 4000, 1, 0, 0)
    _rec(tr, 1, 1, 4000, 6500, 10000, 2, 0, 1)
    # producer statistics of record 1: 2 SM cycles per ns
    tr[:, 1, 12] = 2000
    tr[:, 1, 13] = 1000
    return tr


def test_step_and_clock(trace):
    s = summarize(trace)
    assert s["step_us"] == pytest.approx(9.0)
    assert s["sm_clock_mhz"] == pytest.approx(2000.0)
    assert s["ctas"] == 2


def test_phase_wall_and_per_cta_times(trace):
    ph = summarize(trace)["phases"]
    assert set(ph) == {"gemv/store", "attn"}
    g, a = ph["gemv/store"], ph["attn"]
    assert g["n"] == 2 and a["n"] == 2
    assert g["wall_us"] == pytest.approx(4.0)  # 1000 -> 5000
    assert a["wall_us"] == pytest.approx(4.0)  # 6000 -> 10000
    assert g["dep_us"] == pytest.approx((0.0 + 0.5) / 2)
    assert g["run_us"] == pytest.approx((4.0 + 2.5) / 2)
    assert a["dep_us"] == pytest.approx((0.9 + 2.5) / 2)
    assert a["run_us"] == pytest.approx((3.0 + 3.5) / 2)


def test_idle_fraction_and_prefetch(trace):
    s = summarize(trace)
    idle = [1 - 7000 / 9000, 1 - 6000 / 9000]
    assert s["idle_between_tasks_fraction"] == pytest.approx(np.mean(idle))
    assert s["idle_between_tasks_fraction_max_cta"] == pytest.approx(max(idle))
    assert s["prefetch_requests"] == 1
