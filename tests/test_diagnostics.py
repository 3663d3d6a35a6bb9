"""Pins of the Appendix-A diagnostics (host-side numpy, no GPU): hand-worked
cases and the uniform-attention closed form with full-history masses from the
oracle."""

import numpy as np
import pytest

from oracle import statekv_oracle as O
from kv_cache_selection_b200 import diagnostics as Dg


def test_top_b_and_concentration_hand_cases():
    mass = np.array([0.1, 0.5, 0.1, 0.3])
    assert list(Dg.top_b(mass, 1)) == [1]
    assert list(Dg.top_b(mass, 3)) == [0, 1, 3]          # tie 0.1/0.1 -> lower index
    assert Dg.concentration(mass, 1) == pytest.approx(0.5)
    assert Dg.concentration(mass, 2) == pytest.approx(0.8)
    assert Dg.concentration(mass, 10) == pytest.approx(1.0)


def test_pool_recall_and_retention_hand_case():
    pos_next = np.arange(6)
    mass_next = np.array([0.10, 0.40, 0.05, 0.30, 0.10, 0.05])
    # O_{n+1} = {1, 3}; the pool O_n u frame = {1, 2} u {4, 5} covers only 1
    w, u, o_next = Dg.pool_recall(mass_next, pos_next, np.array([1, 2]), np.array([4, 5]), 2)
    assert list(o_next) == [1, 3]
    assert w == pytest.approx(0.40 / 0.70)
    assert u == pytest.approx(0.5)
    assert Dg.retention(np.array([1, 2]), o_next) == pytest.approx(0.5)
    assert Dg.captured_mass(mass_next, pos_next, np.array([1, 3])) == pytest.approx(0.70)


def _full_history_steps(frames):
    """Oracle run without eviction: pool scores are the full-attention masses."""
    n_tok = sum(len(f[3]) for f in frames)
    st = O.LayerState.empty(frames[0][1].shape[1], frames[0][1].shape[2])
    steps = []
    for f in frames:
        st, res = O.statekv_step(st, *f, B=n_tok)
        steps.append(dict(pos=res["pool_pos"][0], mass=res["score"][0], frame_pos=np.asarray(f[3])))
    return steps


def test_uniform_attention_closed_form():
    """q = 0: every visible key of a row gets the same weight, so every earlier
    token carries the same historical mass.  Concentration at B is then B / m
    for m historical tokens; ties go to the lower position, so the oracle
    state is always the first B tokens: recall and retention are 1."""
    T, Hq, Hkv, d, n_frames = 4, 3, 1, 8, 6
    g = np.random.default_rng(1)
    frames = []
    for n in range(n_frames):
        q = np.zeros((T, Hq, d))
        k = g.standard_normal((T, Hkv, d))
        v = g.standard_normal((T, Hkv, d))
        frames.append((q, k, v, np.arange(n * T, (n + 1) * T)))
    steps = _full_history_steps(frames)
    for n, st in enumerate(steps[1:], start=1):
        hist = ~np.isin(st["pos"], st["frame_pos"])
        m = int(hist.sum())
        assert m == n * T
        np.testing.assert_allclose(st["mass"][hist], st["mass"][hist][0], rtol=1e-13)
        for B in (1, 3, m):
            assert Dg.concentration(st["mass"][hist], B) == pytest.approx(B / m, rel=1e-12)
    rep = Dg.stream_report(steps, budgets=[2, 5])
    for B in (2, 5):
        assert rep["weighted_recall"][B] == pytest.approx(1.0)
        assert rep["retention"][B] == pytest.approx(1.0)


def test_stream_report_recency_capture():
    """Captured mass of 'the last B historical tokens' under uniform attention
    is B / m, and of all history is 1."""
    T, Hq, Hkv, d, n_frames, B = 4, 2, 1, 8, 5, 6
    g = np.random.default_rng(2)
    frames = [(np.zeros((T, Hq, d)), g.standard_normal((T, Hkv, d)), g.standard_normal((T, Hkv, d)),
               np.arange(n * T, (n + 1) * T)) for n in range(n_frames)]
    steps = _full_history_steps(frames)
    last_b = [np.arange(max(0, n * T - B), n * T) for n in range(n_frames)]
    everything = [np.arange(0, n * T) for n in range(n_frames)]
    rep = Dg.stream_report(steps, budgets=[B], retained={"recency": last_b, "all": everything})
    want = np.mean([min(B, n * T) / (n * T) for n in range(1, n_frames)])
    assert rep["captured"]["recency"] == pytest.approx(want)
    assert rep["captured"]["all"] == pytest.approx(1.0)
