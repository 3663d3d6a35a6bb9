"""Pins for the CPU oracle: facts fixed by the pages and by mathematics.

None of these tests compares the oracle with itself.  Each pin is one of:
  * an identity with an independent library routine (torch's
    scaled_dot_product_attention in float64) that holds when nothing is evicted;
  * a closed form (uniform attention, score mass);
  * hand-worked cases with exact rational weights (tests/golden/);
  * brute-force enumeration of top-B sets on tiny pools;
  * the detailed-state concatenation identity.
The mutation tests at the end plant plausible mistakes in the oracle and check
that at least one pin fails for each.

Source: "Linear Scaling Video VLMs for Long Video Understanding" summaries —
P1 §方法步骤详情 (the step), P2 §3.2-3.3 (C is the only prior-frame context;
virtual positions), P3 §2 "Het Proces".
"""

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import statekv_oracle as O
from kv_cache_selection_b200 import synthetic as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers ---
def sdpa_f64(q, k, v, attn_mask=None, is_causal=False):
    """torch SDPA in float64 on [N][H][d] inputs; GQA by repeating KV heads
    (query head h reads KV head h // G)."""
    q = torch.as_tensor(O.to_f64(q)).permute(1, 0, 2)  # [Hq][N][d]
    k = torch.as_tensor(O.to_f64(k)).permute(1, 0, 2)
    v = torch.as_tensor(O.to_f64(v)).permute(1, 0, 2)
    G = q.shape[0] // k.shape[0]
    k = k.repeat_interleave(G, dim=0)
    v = v.repeat_interleave(G, dim=0)
    out = F.scaled_dot_product_attention(q[None], k[None], v[None],
                                         attn_mask=attn_mask, is_causal=is_causal)
    return out[0].permute(1, 0, 2).numpy()


def random_frames(n_frames, T, Hq, Hkv, d, seed):
    g = np.random.default_rng(seed)
    frames = []
    for n in range(n_frames):
        q = g.standard_normal((T, Hq, d))
        k = g.standard_normal((T, Hkv, d))
        v = g.standard_normal((T, Hkv, d))
        pos = np.arange(n * T, (n + 1) * T)
        frames.append((q, k, v, pos))
    return frames


def concat(frames, i):
    return np.concatenate([np.asarray(O.to_f64(f[i])) for f in frames], axis=0)


# ------------------------------------------- no-eviction identity (SDPA) ---
@pytest.mark.parametrize("shape", [
    # (n_frames, T, Hq, Hkv, d)
    (8, 16, 2, 1, 64),   # the tiny workload shape
    (5, 7, 6, 2, 8),     # GQA group of 3, ragged T
    (4, 5, 7, 1, 4),     # group of 7 (the 1B/8B backbones' G)
])
def test_no_eviction_equals_causal_attention(shape):
    """B >= all tokens: nothing is evicted, C_{n-1} holds all history, so the
    frame's attention is exactly causal self-attention over the whole video
    (P2 §3.2: C is the only prior-frame context; P1 §方法步骤详情)."""
    n_frames, T, Hq, Hkv, d = shape
    frames = random_frames(n_frames, T, Hq, Hkv, d, seed=sum(shape))
    N = n_frames * T
    _, res = O.run_stream(frames, B=N)
    out = np.concatenate([r["out"] for r in res], axis=0)
    ref = sdpa_f64(concat(frames, 0), concat(frames, 1), concat(frames, 2), is_causal=True)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    # the quadratic comparator of the oracle agrees too
    full_out, full_lse = O.causal_attention(concat(frames, 0), concat(frames, 1), concat(frames, 2))
    np.testing.assert_allclose(full_out, ref, rtol=0, atol=1e-12)
    lse = np.concatenate([r["lse"] for r in res], axis=1)
    np.testing.assert_allclose(lse, full_lse, rtol=0, atol=1e-12)


def test_no_eviction_tiny_workload():
    """The tiny workload at B=128 (8 frames x 16 tokens) must equal full causal
    attention over its 128 tokens."""
    wl = S.workload("tiny_noevict")
    frames = S.gen_frames(wl)
    _, res = O.run_stream(frames, B=wl.B)
    out = np.concatenate([r["out"] for r in res], axis=0)
    ref = sdpa_f64(concat(frames, 0), concat(frames, 1), concat(frames, 2), is_causal=True)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_bidir_no_eviction_equals_block_causal():
    """Frame-bidirectional mask, nothing evicted: every query of frame b sees all
    tokens of frames a <= b (a block-causal mask)."""
    n_frames, T, Hq, Hkv, d = 4, 6, 4, 2, 8
    frames = random_frames(n_frames, T, Hq, Hkv, d, seed=5)
    _, res = O.run_stream(frames, B=n_frames * T, mask_mode=O.MASK_FRAME_BIDIR)
    out = np.concatenate([r["out"] for r in res], axis=0)
    fr = np.arange(n_frames * T) // T
    mask = torch.as_tensor(fr[None, :] <= fr[:, None])
    ref = sdpa_f64(concat(frames, 0), concat(frames, 1), concat(frames, 2), attn_mask=mask)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_zero_budget_is_per_frame_attention():
    """B = 0: no compressed state, each frame attends only to itself (causal)."""
    n_frames, T, Hq, Hkv, d = 3, 9, 4, 2, 8
    frames = random_frames(n_frames, T, Hq, Hkv, d, seed=9)
    _, res = O.run_stream(frames, B=0)
    for f, r in zip(frames, res):
        ref = sdpa_f64(f[0], f[1], f[2], is_causal=True)
        np.testing.assert_allclose(r["out"], ref, rtol=0, atol=1e-12)
        assert all(len(kk) == 0 for kk in r["kept"])


# ------------------------------------------------------ score-mass identity ---
@pytest.mark.parametrize("select", [O.SELECT_GLOBAL, O.SELECT_PER_KV_HEAD, O.SELECT_RECENCY])
@pytest.mark.parametrize("mask", [O.MASK_FRAME_CAUSAL, O.MASK_FRAME_BIDIR])
def test_score_mass(select, mask):
    """Each softmax row sums to 1, so the scores of one step sum to Hq*T
    (global) or G*T per KV head (per-KV-head)."""
    n_frames, T, Hq, Hkv, d, B = 6, 8, 6, 2, 16, 20
    frames = random_frames(n_frames, T, Hq, Hkv, d, seed=3)
    _, res = O.run_stream(frames, B=B, mask_mode=mask, select_mode=select)
    G = Hq // Hkv
    for r in res:
        sums = r["score"].sum(axis=1)
        want = G * T if select == O.SELECT_PER_KV_HEAD else Hq * T
        np.testing.assert_allclose(sums, want, rtol=1e-13)


# ------------------------------------------- uniform attention closed form ---
def test_uniform_attention_closed_form():
    """q = 0 makes every visible key equally weighted.  With m entries in C and
    frame-causal masking, query i sees m + i + 1 keys, so
        sigma_C       = Hq * sum_{i=0}^{T-1} 1/(m+i+1)   (every C entry)
        sigma_frame_t = Hq * sum_{i=t}^{T-1} 1/(m+i+1)
    and lse_i = log(m + i + 1).  Frame token 0 ties the C entries and loses on
    position, so once C is full it never changes."""
    T, Hq, Hkv, d, B, n_frames = 4, 3, 1, 8, 8, 6
    g = np.random.default_rng(0)
    frames = []
    for n in range(n_frames):
        q = np.zeros((T, Hq, d))
        k = g.standard_normal((T, Hkv, d))
        v = g.standard_normal((T, Hkv, d))
        frames.append((q, k, v, np.arange(n * T, (n + 1) * T)))
    _, res = O.run_stream(frames, B=B)
    m = 0
    prev_kept_pos = None
    for n, r in enumerate(res):
        Hs = [sum(Fraction(1, m + i + 1) for i in range(t, T)) for t in range(T + 1)]
        want_C = float(Hq * Hs[0])
        want_f = [float(Hq * Hs[t]) for t in range(T)]
        np.testing.assert_allclose(r["score"][0, :m], want_C, rtol=1e-13)
        np.testing.assert_allclose(r["score"][0, m:], want_f, rtol=1e-13)
        np.testing.assert_allclose(r["lse"], np.log(m + np.arange(T) + 1)[None, :].repeat(Hq, 0),
                                   rtol=0, atol=1e-13)
        kept_pos = r["pool_pos"][0][r["kept"][0]]
        if m + T <= B:
            np.testing.assert_array_equal(kept_pos, r["pool_pos"][0])
        else:
            # C entries (tied with frame token 0, lower positions) all stay
            np.testing.assert_array_equal(kept_pos, prev_kept_pos)
        prev_kept_pos = kept_pos
        m = min(B, m + T)


def test_uniform_attention_bidir_closed_form():
    """q = 0 with the bidirectional frame mask: every query sees all m + T keys,
    so every candidate scores Hq*T/(m+T)."""
    T, Hq, Hkv, d, B = 5, 2, 1, 4, 7
    g = np.random.default_rng(1)
    frames = [(np.zeros((T, Hq, d)), g.standard_normal((T, Hkv, d)),
               g.standard_normal((T, Hkv, d)), np.arange(n * T, (n + 1) * T))
              for n in range(4)]
    _, res = O.run_stream(frames, B=B, mask_mode=O.MASK_FRAME_BIDIR)
    m = 0
    for r in res:
        np.testing.assert_allclose(r["score"][0], Hq * T / (m + T), rtol=1e-13)
        m = min(B, m + T)


# ------------------------------------------------ hand-worked golden cases ---
def _frac(s):
    return float(Fraction(s))


def _lse_value(e):
    assert e[0] == "ln"
    return math.log(float(Fraction(e[1])))


def _handworked_frames(case, T, d):
    Hq, Hkv = case["Hq"], case["Hkv"]
    frames = []
    for n, expo in enumerate(case["key_exponents"]):
        pos = np.arange(n * T, (n + 1) * T)
        q = np.zeros((T, Hq, d))
        q[:, :, 0] = math.sqrt(2.0) * math.log(2.0)
        k = np.zeros((T, Hkv, d))
        v = np.zeros((T, Hkv, d))
        for t in range(T):
            for g in range(Hkv):
                k[t, g, 0] = expo[t][g]
                v[t, g, 0] = pos[t]
                v[t, g, 1] = 1.0
        frames.append((q, k, v, pos))
    return frames


def test_handworked_golden_cases():
    with open(os.path.join(GOLDEN, "handworked_three_frames.json")) as f:
        gold = json.load(f)
    T, d, B = gold["T"], gold["d"], gold["B"]
    for case in gold["cases"]:
        frames = _handworked_frames(case, T, d)
        _, res = O.run_stream(frames, B=B, select_mode=case["select"])
        for fexp, r in zip(case["frames"], res):
            for gi, row in enumerate(fexp["score"]):
                np.testing.assert_allclose(r["score"][gi], [_frac(s) for s in row],
                                           rtol=1e-12, err_msg=case["name"])
            for gi, kp in enumerate(fexp["kept_pos"]):
                got = r["pool_pos"][gi][r["kept"][gi]]
                np.testing.assert_array_equal(got, kp, err_msg=case["name"])
            if "lse" in fexp:
                want = [_lse_value(e) for e in fexp["lse"]]
                np.testing.assert_allclose(r["lse"][0], want, rtol=0, atol=1e-12)
            if "out_x" in fexp:
                want = [_frac(e[0]) for e in fexp["out_x"]]
                np.testing.assert_allclose(r["out"][:, 0, 0], want, rtol=0, atol=1e-12)
                np.testing.assert_allclose(r["out"][:, 0, 1], 1.0, rtol=0, atol=1e-12)


# ------------------------------------------------ brute-force top-B sets ---
def _brute_top_b(score, pos, B):
    """The kept set is the unique B-subset whose members all beat all
    non-members under (score desc, position asc); enumerate every subset."""
    L = len(score)
    if L <= B:
        return sorted(range(L), key=lambda j: pos[j])
    winners = []
    for sub in itertools.combinations(range(L), B):
        inside = set(sub)
        ok = all((score[a] > score[b]) or (score[a] == score[b] and pos[a] < pos[b])
                 for a in inside for b in range(L) if b not in inside)
        if ok:
            winners.append(sub)
    assert len(winners) == 1
    return sorted(winners[0], key=lambda j: pos[j])


@pytest.mark.parametrize("seed", range(40))
def test_select_matches_brute_force(seed):
    g = np.random.default_rng(seed)
    L = int(g.integers(1, 10))
    B = int(g.integers(0, 9))
    score = g.integers(0, 4, size=L).astype(np.float64) * 0.25   # many ties
    pos = g.permutation(100)[:L]
    got = O.select_top_b(score, pos, B)
    assert list(got) == _brute_top_b(score, pos, B)


# ------------------------------------------------- recency-based retention ---
def test_recency_keeps_the_last_b_tokens():
    """Recency retention (P2 Appendix A.3): after frame n, C holds exactly the
    last min(B, (n+1)T) tokens of the stream, for every KV head, as copies of
    those tokens' K/V rows."""
    n_frames, T, Hq, Hkv, d, B = 7, 8, 6, 2, 16, 20
    frames = random_frames(n_frames, T, Hq, Hkv, d, seed=5)
    Kall, Vall = concat(frames, 1), concat(frames, 2)
    st = O.LayerState.empty(Hkv, d)
    for n, f in enumerate(frames):
        st, res = O.statekv_step(st, *f, B=B, select_mode=O.SELECT_RECENCY)
        seen = (n + 1) * T
        want = np.arange(max(0, seen - B), seen)
        for g in range(Hkv):
            np.testing.assert_array_equal(st.pos_C[g], want)
            np.testing.assert_array_equal(st.K_C[g], Kall[want, g])
            np.testing.assert_array_equal(st.V_C[g], Vall[want, g])


@pytest.mark.parametrize("seed", range(20))
def test_recency_select_matches_brute_force(seed):
    """Largest positions first, on pools whose positions arrive in any order."""
    g = np.random.default_rng(seed)
    L = int(g.integers(1, 12))
    B = int(g.integers(0, 12))
    pos = g.permutation(50)[:L]
    got = list(O.select_recent_b(pos, B))
    best = sorted(range(L), key=lambda j: -pos[j])[:B]
    assert got == sorted(best, key=lambda j: pos[j])


def test_recency_changes_only_the_kept_set():
    """For one and the same state, recency and global steps compute identical
    attention outputs, row statistics and scores; only C_n differs."""
    n_frames, T, Hq, Hkv, d, B = 5, 8, 6, 2, 16, 12
    frames = random_frames(n_frames, T, Hq, Hkv, d, seed=9)
    st, _ = O.run_stream(frames[:-1], B=B)
    _, r_g = O.statekv_step(st, *frames[-1], B=B, select_mode=O.SELECT_GLOBAL)
    _, r_r = O.statekv_step(st, *frames[-1], B=B, select_mode=O.SELECT_RECENCY)
    for key in ("out", "lse", "score", "pool_pos"):
        np.testing.assert_array_equal(r_g[key], r_r[key])
    assert not all(np.array_equal(a, b) for a, b in zip(r_g["kept"], r_r["kept"]))


# ------------------------------------------------ decode over the detailed state ---
@pytest.mark.parametrize("n_text", [1, 5])
def test_decode_attention_equals_causal_over_the_whole_sequence(n_text):
    """Text tokens after the video attend over D (every frame token) and
    causally over the text: the rows of a library causal attention over the
    concatenated sequence [video; text]."""
    n_frames, T, Hq, Hkv, d, B = 4, 6, 6, 2, 16, 8
    frames = random_frames(n_frames, T, Hq, Hkv, d, seed=21)
    st, _ = O.run_stream(frames, B=B)
    DK, DV, _ = st.detailed()
    g = np.random.default_rng(22)
    q = g.standard_normal((n_text, Hq, d))
    k = g.standard_normal((n_text, Hkv, d))
    v = g.standard_normal((n_text, Hkv, d))
    out, lse = O.decode_attention(DK, DV, q, k, v)
    Qall = np.concatenate([concat(frames, 0), q])
    Kall = np.concatenate([concat(frames, 1), k])
    Vall = np.concatenate([concat(frames, 2), v])
    ref = sdpa_f64(Qall, Kall, Vall, is_causal=True)[-n_text:]
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    # lse against a direct log-sum-exp of the visible logits of head 0, row 0
    N = DK.shape[1]
    s0 = np.concatenate([DK[0], k[:1, 0]]) @ q[0, 0] / math.sqrt(d)
    np.testing.assert_allclose(lse[0, 0], np.log(np.exp(s0).sum()), rtol=1e-13)
    assert N == n_frames * T


def test_decode_attention_without_video_is_causal_attention():
    g = np.random.default_rng(23)
    n, Hq, Hkv, d = 4, 4, 2, 8
    q, k, v = g.standard_normal((n, Hq, d)), g.standard_normal((n, Hkv, d)), g.standard_normal((n, Hkv, d))
    out, _ = O.decode_attention(np.zeros((Hkv, 0, d)), np.zeros((Hkv, 0, d)), q, k, v)
    np.testing.assert_allclose(out, sdpa_f64(q, k, v, is_causal=True), rtol=0, atol=1e-12)


# ------------------------------------------ detailed state and positions ---
@pytest.mark.parametrize("select", [O.SELECT_GLOBAL, O.SELECT_PER_KV_HEAD])
def test_detailed_state_is_concatenation(select):
    wl = S.workload("tiny")
    frames = S.gen_frames(wl)
    st, res = O.run_stream(frames, B=wl.B, select_mode=select)
    K, V, pos = st.detailed()
    np.testing.assert_array_equal(K, concat(frames, 1).transpose(1, 0, 2))
    np.testing.assert_array_equal(V, concat(frames, 2).transpose(1, 0, 2))
    np.testing.assert_array_equal(pos, np.arange(wl.frames * wl.T))
    # C: capacity min(B, m+T), ascending positions, rows are the tokens' K/V
    m = 0
    for r in res:
        m = min(wl.B, m + wl.T)
        assert all(len(kk) == m for kk in r["kept"])
    for g in range(wl.Hkv):
        assert np.all(np.diff(st.pos_C[g]) > 0)
        np.testing.assert_array_equal(st.K_C[g], K[g][st.pos_C[g]])
        np.testing.assert_array_equal(st.V_C[g], V[g][st.pos_C[g]])


def test_sink_workload_prefers_planted_sinks():
    """Sanity (not a pin): on the planted-sink distribution the kept set holds
    clearly more planted sink tokens than a random B-subset would."""
    wl = S.workload("1b_layer", Hq=4, Hkv=2, d=32, T=32, B=64, frames=6, n_sinks=4)
    frames = S.gen_frames(wl)
    st, _ = O.run_stream(frames, B=wl.B)
    sinks = {int(n * wl.T + i) for n in range(wl.frames) for i in S.sink_indices(wl, 0, 0, n)}
    kept = set(int(p) for p in st.pos_C[0])
    chance = wl.B / (wl.frames * wl.T) * len(sinks)
    assert len(kept & sinks) >= 1.5 * chance


# ------------------------------------------------------- mutation checks ---
def _pins_fail(monkeypatch, patch):
    """Apply a planted mistake to the oracle; return True if some pin fails."""
    patch(monkeypatch)
    checks = [
        lambda: test_no_eviction_equals_causal_attention((5, 7, 6, 2, 8)),
        test_handworked_golden_cases,
        test_uniform_attention_closed_form,
        lambda: test_score_mass(O.SELECT_GLOBAL, O.MASK_FRAME_CAUSAL),
    ]
    for c in checks:
        try:
            c()
        except AssertionError:
            return True
    return False


def _wrong_mask(mp):
    orig = O.visible_mask

    def bad(T, m, mode):
        vis = orig(T, m, mode)
        if mode == O.MASK_FRAME_CAUSAL:
            i = np.arange(T)[:, None]
            t = np.arange(T)[None, :]
            vis[:, m:] = t < i + 2        # off by one
        return vis
    mp.setattr(O, "visible_mask", bad)


def _wrong_scale(mp):
    orig = O.attend_pool

    def bad(q_h, K_pool, V_pool, vis):
        return orig(q_h / math.sqrt(q_h.shape[1]), K_pool, V_pool, vis)   # 1/d
    mp.setattr(O, "attend_pool", bad)


def _wrong_tiebreak(mp):
    orig = O.select_top_b
    mp.setattr(O, "select_top_b", lambda score, pos, B: orig(score, -pos, B)[::-1])


def _transposed_mass(mp):
    orig = O.attend_pool

    def bad(q_h, K_pool, V_pool, vis):
        out, lse, P = orig(q_h, K_pool, V_pool, vis)
        P2 = P / np.maximum(P.sum(axis=0, keepdims=True), 1e-300) * P.sum(axis=1).mean()
        return out, lse, P2    # column-normalised instead of row-normalised
    mp.setattr(O, "attend_pool", bad)


def _dropped_frame_tokens(mp):
    orig = O.select_top_b

    def bad(score, pos, B):
        return orig(score[: max(len(score) - 1, 0)], pos[: max(len(pos) - 1, 0)], B)
    mp.setattr(O, "select_top_b", bad)


def _wrong_gqa(mp):
    mp.setattr(O, "kv_head_of", lambda h, Hq, Hkv: h % Hkv)   # interleaved groups


def test_planted_recency_mistake_is_caught(monkeypatch):
    """Keeping the oldest instead of the newest tokens fails the recency pin."""
    monkeypatch.setattr(O, "select_recent_b", lambda pos, B: np.arange(min(B, len(pos))))
    with pytest.raises(AssertionError):
        test_recency_keeps_the_last_b_tokens()


@pytest.mark.parametrize("patch", [_wrong_mask, _wrong_scale, _wrong_tiebreak,
                                   _transposed_mass, _dropped_frame_tokens,
                                   _wrong_gqa])
def test_planted_mistakes_are_caught(monkeypatch, patch):
    assert _pins_fail(monkeypatch, patch)


# ------------------------------------- sampled-row causal attention pins ---
def _rows_pin(Hq=7, Hkv=1, N=300, d=16, seed=11, rows=(0, 1, 2, 127, 128, 129, 255, 256, 298, 299)):
    """causal_attention_rows at rows that span the first row, 128-token tile
    boundaries and the last row, against torch SDPA (is_causal) in float64 for
    out, and for lse against a second SDPA call with one extra "probe" key
    (zero logit, visible to every row) whose value is a one-hot extra channel:
    that channel's output is p = 1 / (1 + sum_j exp(s_ij)), so
    lse_i = log((1 - p) / p).  Also the uniform case q = 0: lse_i = log(i + 1)."""
    g = np.random.default_rng(seed)
    q = g.standard_normal((N, Hq, d))
    k = g.standard_normal((N, Hkv, d))
    v = g.standard_normal((N, Hkv, d))
    rows = list(rows)
    out, lse = O.causal_attention_rows(q, k, v, rows)
    ref = sdpa_f64(q, k, v, is_causal=True)
    np.testing.assert_allclose(out, ref[rows], rtol=0, atol=1e-12)
    # probe-key identity for lse
    kp = np.concatenate([np.zeros((1, Hkv, d)), k], axis=0)
    vp = np.concatenate([np.zeros((1, Hkv, d + 1)), np.concatenate([v, np.zeros((N, Hkv, 1))], axis=2)], axis=0)
    vp[0, :, d] = 1.0
    mask = torch.ones((N, N + 1), dtype=torch.bool)
    mask[:, 1:] = torch.tril(torch.ones((N, N), dtype=torch.bool))
    probe = sdpa_f64(q, kp, vp, attn_mask=mask)[:, :, d]      # [N][Hq]
    want = np.log((1.0 - probe) / probe).T                    # [Hq][N]
    np.testing.assert_allclose(lse, want[:, rows], rtol=0, atol=1e-9)
    # uniform attention: every visible logit is 0
    _, lse0 = O.causal_attention_rows(np.zeros_like(q), k, v, rows)
    np.testing.assert_allclose(lse0, np.log(np.asarray(rows, dtype=np.float64) + 1)[None, :].repeat(Hq, 0),
                               rtol=0, atol=1e-12)


@pytest.mark.parametrize("Hq,Hkv", [(7, 1), (14, 2), (4, 4)])
def test_causal_attention_rows_pinned(Hq, Hkv):
    _rows_pin(Hq=Hq, Hkv=Hkv)


def test_causal_attention_rows_planted_mistakes(monkeypatch):
    """Plant an off-by-one in the visible prefix (keys 0..i-1 instead of 0..i)
    and an interleaved GQA map in the oracle; the pins above must fail."""
    import inspect
    import textwrap

    src = textwrap.dedent(inspect.getsource(O.causal_attention_rows))
    assert src.count("i + 1") == 3
    bad_src = src.replace("k[:i + 1", "k[:i").replace("v[:i + 1", "v[:i").replace("(1, i + 1)", "(1, i)")
    ns = dict(O.__dict__)
    exec(bad_src, ns)
    monkeypatch.setattr(O, "causal_attention_rows", ns["causal_attention_rows"])
    # row 0 would see no key at all under this mistake: sample rows >= 1
    with pytest.raises(AssertionError):
        _rows_pin(rows=(1, 2, 127, 128, 299))
    monkeypatch.undo()
    monkeypatch.setattr(O, "kv_head_of", lambda h, Hq, Hkv: h % Hkv)
    with pytest.raises(AssertionError):
        _rows_pin(Hq=14, Hkv=2)
