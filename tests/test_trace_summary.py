"""The benchmark's per-phase trace summary (bench.summarize_trace) on a hand-built trace whose
waits, compute times and tails are known, so that the fractions it reports can be checked
by hand. CPU only."""

import numpy as np
import pytest

import bench


def _trace(grid: int, steps: int, layers: int, scale: int):
    """Rows of a launch where every phase takes: 2 units waiting for inputs, 5 computing
    (1 of them waiting for stages), 1 tail; 3 units between the LM head and the next step."""
    rows_per_cta = 5 * layers * steps + steps + 2
    tr = np.zeros((grid, rows_per_cta, 8), np.int64)
    for c in range(grid):
        t0 = 1000 + 7 * c
        r = 0
        for s in range(steps):
            if s > 0:
                t0 += 3 * scale  # step boundary
            phases = [(l, ph) for l in range(layers) for ph in range(5)] + [(layers - 1, 5)]
            for l, ph in phases:
                tr[c, r] = [(s << 16) | (l << 4) | ph, t0, t0 + 2 * scale, t0 + 7 * scale, t0 + 8 * scale, scale,
                            t0 + 3 * scale, t0 + 6 * scale]
                t0 += 8 * scale
                r += 1
    return tr


def test_summary_of_a_known_trace():
    grid, steps, layers, scale = 3, 4, 2, 100
    tr = _trace(grid, steps, layers, scale)
    # whole-launch span per CTA in cycles, and a launch time that makes 1 unit = 1 microsecond
    span_cyc = (5 * layers + 1) * 8 * scale * steps + 3 * scale * (steps - 1)
    traced_ms = span_cyc / scale / 1e3
    out = bench.summarize_trace(tr, traced_ms)
    assert out["sm_cycles_per_us"] == pytest.approx(scale)
    for n in bench.PHASES:
        p = out["us_per_phase"][n]
        assert p["wait"] == pytest.approx(2.0)
        assert p["compute"] == pytest.approx(5.0)
        assert p["tail"] == pytest.approx(1.0)
        assert p["stage_wait"] == pytest.approx(1.0)
        assert p["total"] == pytest.approx(8.0)
        if n != "qkv":
            assert p["gap_before"] == pytest.approx(0.0)
    # steps 1..3: 11 phases each; sync-gated waits: Q/K/V of layer >= 1, gate/up, LM head
    nph = 5 * layers + 1
    span = 3 * nph * 8 + 2 * 3
    n_sync = (layers - 1) + layers + 1
    f = out["fraction_of_time"]
    assert f["cross_cta_sync_wait"] == pytest.approx((3 * n_sync * 2 + 2 * 3) / span)
    assert f["kv_head_exchange_wait"] == pytest.approx(3 * 2 * layers * 2 / span)
    assert f["stage_wait_in_compute"] == pytest.approx(3 * nph / span)
    assert f["phase_tails"] == pytest.approx(3 * nph / span)
    assert out["step_boundary_us"] == pytest.approx(3.0)
    assert out["between_phases_us_per_step"] == pytest.approx(0.0)
