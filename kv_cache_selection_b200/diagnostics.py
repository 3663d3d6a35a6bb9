"""Appendix-A diagnostics of the temporal state, computed from what the library
reports (host-side numpy on step statistics; no kernels of its own).

"Linear Scaling Video VLMs for Long Video Understanding", section-by-section
summary, Appendix A:

  * A.1 concentration: the fraction of the current frame's historical attention
    mass (attention of the frame's queries, summed over query heads and rows,
    onto tokens of earlier frames, with every available token as a key) that
    the top-B historical tokens capture;
  * A.2 candidate-pool recall: the oracle state O_n is the top-B set over every
    token seen through frame n; the incremental pool O_n u frame n+1 should
    cover O_{n+1}.  Weighted recall weighs the covered tokens of O_{n+1} by
    their mass; retention is the share of O_n that is still in O_{n+1};
  * A.3 recency comparison: the historical mass captured by a retained set (the
    score-based C or the last-B-tokens C) at a given budget.

The full-history masses come from a library handle whose capacity exceeds the
stream, so that C holds every earlier token: its pool scores at frame n are
then exactly the full-attention masses of frame n's queries on all tokens seen
through frame n (earlier tokens first, in position order, then the frame).
"""

from __future__ import annotations

import numpy as np


def top_b(mass: np.ndarray, B: int) -> np.ndarray:
    """Indices of the B largest masses (ties to the lower index), ascending."""
    L = mass.shape[0]
    if B >= L:
        return np.arange(L)
    order = np.lexsort((np.arange(L), -mass))
    return np.sort(order[:B])


def concentration(hist_mass: np.ndarray, B: int) -> float:
    """A.1: share of the historical mass captured by the top-B historical tokens."""
    total = float(hist_mass.sum())
    if total <= 0.0:
        return float("nan")
    return float(hist_mass[top_b(hist_mass, B)].sum()) / total


def captured_mass(hist_mass: np.ndarray, hist_pos: np.ndarray, kept_pos: np.ndarray) -> float:
    """A.3: share of the historical mass on the tokens whose positions are kept."""
    total = float(hist_mass.sum())
    if total <= 0.0:
        return float("nan")
    sel = np.isin(hist_pos, kept_pos)
    return float(hist_mass[sel].sum()) / total


def pool_recall(mass_next: np.ndarray, pos_next: np.ndarray, oracle_prev_pos: np.ndarray,
                frame_next_pos: np.ndarray, B: int):
    """A.2 for one step n -> n+1.

    mass_next / pos_next: masses and positions of every token seen through frame
    n+1 (full attention of frame n+1's queries).  oracle_prev_pos: positions of
    O_n.  frame_next_pos: positions of frame n+1's tokens.  Returns
    (weighted recall, unweighted recall, O_{n+1} positions)."""
    idx = top_b(mass_next, B)
    o_next = pos_next[idx]
    w = mass_next[idx]
    covered = np.isin(o_next, np.union1d(oracle_prev_pos, frame_next_pos))
    wsum = float(w.sum())
    weighted = float(w[covered].sum()) / wsum if wsum > 0 else float("nan")
    unweighted = float(covered.mean()) if len(o_next) else float("nan")
    return weighted, unweighted, o_next


def retention(prev_pos: np.ndarray, next_pos: np.ndarray) -> float:
    """A.2: share of O_n that is still in O_{n+1}."""
    if len(prev_pos) == 0:
        return float("nan")
    return float(np.isin(prev_pos, next_pos).mean())


def stream_report(full_steps, budgets, retained=None):
    """Diagnostics over a stream.

    full_steps: per frame n, a dict with `pos` (positions of every token seen
    through frame n: earlier tokens, then the frame), `mass` (their
    full-attention masses) and `frame_pos` (the frame's positions).
    budgets: the B values.  retained: optional {name: per-frame list of kept
    positions of C_{n-1} (the state the frame attends to)} for A.3.
    Returns means over the frames that have history."""
    rep = {"concentration": {}, "weighted_recall": {}, "recall": {}, "retention": {}, "captured": {}}
    for B in budgets:
        conc, wrec, rec, ret = [], [], [], []
        o_prev = None
        for n, st in enumerate(full_steps):
            hist = ~np.isin(st["pos"], st["frame_pos"])
            if hist.any():
                conc.append(concentration(st["mass"][hist], B))
            o_n = st["pos"][top_b(st["mass"], B)]
            if o_prev is not None:
                w, u, _ = pool_recall(st["mass"], st["pos"], o_prev, st["frame_pos"], B)
                wrec.append(w)
                rec.append(u)
                ret.append(retention(o_prev, o_n))
            o_prev = o_n
        rep["concentration"][B] = float(np.nanmean(conc)) if conc else float("nan")
        rep["weighted_recall"][B] = float(np.nanmean(wrec)) if wrec else float("nan")
        rep["recall"][B] = float(np.nanmean(rec)) if rec else float("nan")
        rep["retention"][B] = float(np.nanmean(ret)) if ret else float("nan")
    for name, kept_per_frame in (retained or {}).items():
        vals = []
        for st, kept in zip(full_steps, kept_per_frame):
            hist = ~np.isin(st["pos"], st["frame_pos"])
            if hist.any() and kept is not None:
                vals.append(captured_mass(st["mass"][hist], st["pos"][hist], kept))
        rep["captured"][name] = float(np.nanmean(vals)) if vals else float("nan")
    return rep
