"""Comparison helpers shared by the GPU parity tests (test infrastructure).

Tolerances:
  * detailed state D, positions, and the rows of C: bit-exact;
  * attention output: bf16 rel-L2 <= 1e-2 and max-abs <= 3e-2; f32 rel-L2
    <= 1e-5 and max-abs <= 1e-5;
  * lse (natural log): bf16 abs <= 2e-3; f32 abs <= 1e-5 (both sides see the
    same bf16 inputs, so the only differences are float32 accumulation order and
    the rounding of P to bf16 before P.V, which lse does not see);
  * scores: relative 1e-3 with an absolute floor of 1e-6 x the mean candidate
    score (Hq*T/L, or G*T/L per KV head);
  * kept set: identical except for candidates whose oracle score lies within
    1e-4 relative of the B-th largest oracle score.
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import statekv_oracle as O

OUT_TOL = {"bf16": (1e-2, 3e-2), "f32": (1e-5, 1e-5)}
LSE_TOL = {"bf16": 2e-3, "f32": 1e-5}
SCORE_RTOL = 1e-3
BOUNDARY_RTOL = 1e-4


def to_np(t):
    return O.to_f64(t)


def check_out(got, want, dtype, what="out"):
    got = to_np(got)
    want = np.asarray(want, dtype=np.float64)
    rel_l2 = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300)
    max_abs = np.abs(got - want).max() if want.size else 0.0
    rtol, atol = OUT_TOL[dtype]
    assert rel_l2 <= rtol and max_abs <= atol, f"{what}: rel_l2={rel_l2:.3e} max_abs={max_abs:.3e}"
    return rel_l2, max_abs


def check_lse(got, want, dtype):
    got = to_np(got)
    err = np.abs(got - want).max() if want.size else 0.0
    assert err <= LSE_TOL[dtype], f"lse max abs err {err:.3e}"
    return err


def check_scores(got, want, total_mass):
    """got/want [rows][L]; total_mass: per-row sum of scores (Hq*T or G*T)."""
    got = to_np(got)
    L = want.shape[-1]
    floor = 1e-6 * total_mass / max(L, 1)
    err = np.abs(got - want)
    ok = err <= SCORE_RTOL * np.abs(want) + floor
    assert ok.all(), (f"scores: {int((~ok).sum())} of {ok.size} out of tolerance; worst rel "
                      f"{(err / np.maximum(np.abs(want), floor)).max():.3e}")
    return (err / np.maximum(np.abs(want), floor)).max() if want.size else 0.0


def check_selection(got_pos, want_kept, score, pool_pos, B):
    """got_pos: positions the GPU kept for one selection group (ascending);
    want_kept: oracle kept pool indices; score/pool_pos: oracle pool scores and
    positions.  Returns the number of near-boundary candidates."""
    got_pos = np.asarray(got_pos, dtype=np.int64)
    L = len(score)
    assert np.all(np.diff(got_pos) > 0), "C positions must ascend"
    assert len(got_pos) == min(B, L), f"kept {len(got_pos)} expected {min(B, L)}"
    want_pos = set(int(p) for p in pool_pos[want_kept])
    got = set(int(p) for p in got_pos)
    assert got <= set(int(p) for p in pool_pos), "kept a position outside the pool"
    if L <= B:
        assert got == want_pos
        return 0
    tau = np.sort(score)[::-1][B - 1]
    near = np.abs(score - tau) <= BOUNDARY_RTOL * tau
    for j in range(L):
        if near[j]:
            continue
        p = int(pool_pos[j])
        assert (p in got) == (p in want_pos), (
            f"candidate pos {p} score {score[j]:.6g} (tau {tau:.6g}): gpu {p in got}, oracle {p in want_pos}")
    return int(near.sum())


def oracle_state_from_gpu(C, S_idx=0):
    """Oracle LayerState rebuilt from the GPU's compressed state of stream S_idx."""
    m = C["len"]
    K = C["k"][S_idx, :, :m].cpu()
    V = C["v"][S_idx, :, :m].cpu()
    pos = C["pos"][S_idx, :, :m].cpu().numpy()
    return O.LayerState.from_compressed(K, V, pos)
