"""StateKV per-frame cache-builder step: plain float64 CPU oracle.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, constants or helpers with the CUDA library; the two meet only at the
seeded input generator (``kv_cache_selection_b200.synthetic``), which holds none
of the method's arithmetic.

Sources (web summaries of the paper "Linear Scaling Video VLMs for Long Video
Understanding"; cited by page and section):

  P1  "线性扩展视频视觉语言模型用于长视频理解 Linear Scaling Video VLMs for Long
      Video Understanding" (Chinese summary), sections 核心方法 and 方法步骤详情.
  P2  "Linear Scaling Video VLMs for Long Video Understanding" (section-by-section
      summary), sections 3.1-3.3 and Appendix A.
  P3  "Technische Samenvatting: Lineair Schalende Video VLMs voor Lange Video
      Begrip (StateKV)", section 2 "Architectuur en Mechanisme" / "Het Proces".

What one step computes (P1 §方法步骤详情; P2 §3.3; P3 §2 "Het Proces"), for one
layer and frame n with compressed state C_{n-1} (m entries per KV head):

  1. the frame's queries attend over [C_{n-1} ; frame n keys/values];
  2. the frame's K/V are appended to the detailed state D;
  3. every candidate j of the pool C_{n-1} u frame n gets the score
     sigma_j = sum over the frame's queries i (and query heads) of the
     normalised softmax weight P_ij;
  4. the top-B candidates by score become C_n.

Readings taken where the pages are silent:
  * softmax scale 1/sqrt(d);
  * mask: frame token t is visible to frame query i iff t <= i
    ("frame_causal"; the backbone LLM is causal, P1 §自注意力复杂度); all
    C entries are visible.  "frame_bidir" makes every frame token visible;
  * query head h uses KV head floor(h / G), G = Hq / Hkv;
  * scores use frame n's attention only (no accumulation across frames);
  * "global" selection sums sigma over all query heads and keeps one set for
    every KV head; "per_kv_head" sums over the G query heads of each KV head and
    selects per KV head (P2 §A "Protocol": sinks are kept per layer and KV head);
  * "recency" is the pages' comparison baseline (P2 Appendix A.3 "Supporting
    comparison: recency-based retention"; the sliding windows of ReKV in P2's
    related work): C_n holds the B candidates with the largest positions, i.e.
    the last B tokens seen, one set for every KV head; scores are computed and
    reported exactly as in "global" mode but do not decide what is kept;
  * ties are broken by lower original position; C_n is stored in ascending
    original position;
  * while m + T <= B nothing is evicted (top-B of fewer than B candidates);
  * inputs arrive with RoPE already applied at absolute ("virtual") positions
    (P2 §3.3); the oracle stores positions and never re-rotates.

Every function below is a direct transcription of that definition: no blocking,
no online softmax, no reordering.  Numpy matmul / exp / log / lexsort are the
only library primitives used.

Parity pins for this module live in ``tests/test_oracle_pins.py``: the
no-eviction identity against a library causal attention, closed-form scores for
uniform attention, hand-worked top-B sets with exact rational scores, the
score-mass identity and the detailed-state concatenation identity.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

MASK_FRAME_CAUSAL = "frame_causal"
MASK_FRAME_BIDIR = "frame_bidir"
SELECT_GLOBAL = "global"
SELECT_PER_KV_HEAD = "per_kv_head"
SELECT_RECENCY = "recency"


def to_f64(x) -> np.ndarray:
    """Exact upcast of f32 / bf16 (given as a torch tensor or array) to float64."""
    if hasattr(x, "detach"):  # torch tensor, possibly bf16
        x = x.detach().to("cpu")
        import torch  # local: the oracle itself needs only numpy

        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def kv_head_of(h: int, Hq: int, Hkv: int) -> int:
    """KV head read by query head h: floor(h / G) with G = Hq / Hkv."""
    return h // (Hq // Hkv)


def visible_mask(T: int, m: int, mask_mode: str) -> np.ndarray:
    """[T][m+T] bool: may frame query i look at pool entry j?

    Pool order: j < m are the compressed-state entries (always visible),
    j = m + t is frame token t (visible iff t <= i in frame-causal mode).
    """
    vis = np.ones((T, m + T), dtype=bool)
    if mask_mode == MASK_FRAME_CAUSAL:
        i = np.arange(T)[:, None]
        t = np.arange(T)[None, :]
        vis[:, m:] = t <= i
    elif mask_mode != MASK_FRAME_BIDIR:
        raise ValueError(f"unknown mask mode {mask_mode!r}")
    return vis


def attend_pool(q_h: np.ndarray, K_pool: np.ndarray, V_pool: np.ndarray,
                vis: np.ndarray):
    """Softmax attention of one query head over one pool.

    q_h [T][d], K_pool/V_pool [L][d], vis [T][L].  Returns out [T][d],
    lse [T] and the normalised weights P [T][L] (0 where masked).
    The definition: s_ij = <q_i, k_j> / sqrt(d); lse_i = log sum_visible exp s_ij;
    P_ij = exp(s_ij - lse_i); out_i = sum_j P_ij v_j  (P1 §方法步骤详情).
    """
    d = q_h.shape[1]
    S = (q_h @ K_pool.T) / math.sqrt(d)
    S = np.where(vis, S, -np.inf)
    row_max = S.max(axis=1, keepdims=True)
    lse = row_max[:, 0] + np.log(np.exp(S - row_max).sum(axis=1))
    P = np.where(vis, np.exp(S - lse[:, None]), 0.0)
    out = P @ V_pool
    return out, lse, P


def select_top_b(score: np.ndarray, pos: np.ndarray, B: int) -> np.ndarray:
    """Pool indices of the kept candidates, in ascending original position.

    Keep everything if the pool holds at most B candidates; otherwise order the
    pool by (score descending, position ascending), keep the first B, and
    return them sorted by position (P1 §方法步骤详情: top-B of the candidate pool;
    P2 §3.3).
    """
    L = score.shape[0]
    if L <= B:
        kept = np.arange(L)
    else:
        order = np.lexsort((pos, -score))  # primary key: -score, then pos
        kept = order[:B]
    return kept[np.argsort(pos[kept], kind="stable")]


def select_recent_b(pos: np.ndarray, B: int) -> np.ndarray:
    """Pool indices of the B candidates with the largest positions (the most
    recent tokens), in ascending position (P2 Appendix A.3: recency-based
    retention keeps the latest frames of the stream)."""
    L = pos.shape[0]
    if L <= B:
        kept = np.arange(L)
    else:
        kept = np.argsort(-pos, kind="stable")[:B]
    return kept[np.argsort(pos[kept], kind="stable")]


@dataclass
class LayerState:
    """Per-layer state: compressed C (per KV head) and detailed D."""

    Hkv: int
    d: int
    K_C: list = field(default_factory=list)      # per KV head: [m][d] f64
    V_C: list = field(default_factory=list)
    pos_C: list = field(default_factory=list)    # per KV head: [m] int64
    score_C: list = field(default_factory=list)  # per KV head: [m] f64
    D_K: list = field(default_factory=list)      # list of frames [T][Hkv][d]
    D_V: list = field(default_factory=list)
    D_pos: list = field(default_factory=list)

    @classmethod
    def empty(cls, Hkv: int, d: int) -> "LayerState":
        st = cls(Hkv=Hkv, d=d)
        st.K_C = [np.zeros((0, d)) for _ in range(Hkv)]
        st.V_C = [np.zeros((0, d)) for _ in range(Hkv)]
        st.pos_C = [np.zeros((0,), dtype=np.int64) for _ in range(Hkv)]
        st.score_C = [np.zeros((0,)) for _ in range(Hkv)]
        return st

    @classmethod
    def from_compressed(cls, K_C, V_C, pos_C, score_C=None) -> "LayerState":
        """Build a state from given C contents ([Hkv][m][d] arrays, [Hkv][m] pos)."""
        K_C = to_f64(K_C)
        V_C = to_f64(V_C)
        pos_C = np.asarray(pos_C, dtype=np.int64)
        Hkv, m, d = K_C.shape
        st = cls.empty(Hkv, d)
        st.K_C = [K_C[g].copy() for g in range(Hkv)]
        st.V_C = [V_C[g].copy() for g in range(Hkv)]
        st.pos_C = [pos_C[g].copy() for g in range(Hkv)]
        if score_C is None:
            st.score_C = [np.zeros((m,)) for _ in range(Hkv)]
        else:
            score_C = to_f64(score_C)
            st.score_C = [score_C[g].copy() for g in range(Hkv)]
        return st

    @property
    def m(self) -> int:
        return self.K_C[0].shape[0] if self.K_C else 0

    def detailed(self):
        """D as arrays: K/V [Hkv][n_tokens][d], pos [n_tokens]."""
        if not self.D_K:
            return (np.zeros((self.Hkv, 0, self.d)), np.zeros((self.Hkv, 0, self.d)),
                    np.zeros((0,), dtype=np.int64))
        K = np.concatenate(self.D_K, axis=0).transpose(1, 0, 2)
        V = np.concatenate(self.D_V, axis=0).transpose(1, 0, 2)
        return K, V, np.concatenate(self.D_pos)


def statekv_step(state: LayerState, q, k, v, pos, B: int,
                 mask_mode: str = MASK_FRAME_CAUSAL,
                 select_mode: str = SELECT_GLOBAL):
    """One StateKV cache-builder step for one layer and one frame.

    q [T][Hq][d], k/v [T][Hkv][d] (any float dtype; upcast exactly to f64),
    pos [T] absolute positions of the frame's tokens.

    Returns (new_state, result) where result holds
      out   [T][Hq][d]   attention output of the frame's queries,
      lse   [Hq][T]      per-row log-sum-exp,
      score [Hkv][m+T]   candidate scores over the pool (rows equal in global mode),
      kept  [Hkv][<=B]   kept pool indices (ascending position),
      pool_pos [Hkv][m+T].
    The input state is not modified.
    """
    q = to_f64(q)
    k = to_f64(k)
    v = to_f64(v)
    pos = np.asarray(pos, dtype=np.int64)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    m = state.m
    vis = visible_mask(T, m, mask_mode)

    out = np.zeros((T, Hq, d))
    lse = np.zeros((Hq, T))
    # col_mass[h][j] = sum_i P_hij  (the frame's queries of head h)
    col_mass = np.zeros((Hq, m + T))
    pool_K, pool_V, pool_pos = [], [], []
    for g in range(Hkv):
        pool_K.append(np.concatenate([state.K_C[g], k[:, g, :]], axis=0))
        pool_V.append(np.concatenate([state.V_C[g], v[:, g, :]], axis=0))
        pool_pos.append(np.concatenate([state.pos_C[g], pos]))
    for h in range(Hq):
        g = kv_head_of(h, Hq, Hkv)
        o_h, lse_h, P_h = attend_pool(q[:, h, :], pool_K[g], pool_V[g], vis)
        out[:, h, :] = o_h
        lse[h] = lse_h
        col_mass[h] = P_h.sum(axis=0)

    if select_mode == SELECT_GLOBAL:
        # one score vector for the layer: the pool positions agree across KV
        # heads because every KV head keeps the same set
        sigma = col_mass.sum(axis=0)
        score = np.tile(sigma, (Hkv, 1))
        kept_one = select_top_b(sigma, pool_pos[0], B)
        kept = [kept_one.copy() for _ in range(Hkv)]
    elif select_mode == SELECT_PER_KV_HEAD:
        score = np.stack([col_mass[[h for h in range(Hq) if kv_head_of(h, Hq, Hkv) == g]].sum(axis=0)
                          for g in range(Hkv)])
        kept = [select_top_b(score[g], pool_pos[g], B) for g in range(Hkv)]
    elif select_mode == SELECT_RECENCY:
        sigma = col_mass.sum(axis=0)
        score = np.tile(sigma, (Hkv, 1))
        kept_one = select_recent_b(pool_pos[0], B)
        kept = [kept_one.copy() for _ in range(Hkv)]
    else:
        raise ValueError(f"unknown select mode {select_mode!r}")

    new = LayerState.empty(Hkv, d)
    new.K_C = [pool_K[g][kept[g]] for g in range(Hkv)]
    new.V_C = [pool_V[g][kept[g]] for g in range(Hkv)]
    new.pos_C = [pool_pos[g][kept[g]] for g in range(Hkv)]
    new.score_C = [score[g][kept[g]] for g in range(Hkv)]
    # D <- D || (K_n, V_n): every frame token, unmodified (P1 §方法步骤详情; P3 §2)
    new.D_K = state.D_K + [k.copy()]
    new.D_V = state.D_V + [v.copy()]
    new.D_pos = state.D_pos + [pos.copy()]

    result = dict(out=out, lse=lse, score=score, kept=kept,
                  pool_pos=np.stack(pool_pos))
    return new, result


def run_stream(frames, B: int, mask_mode: str = MASK_FRAME_CAUSAL,
               select_mode: str = SELECT_GLOBAL):
    """Run StateKV over a list of frames (q, k, v, pos) from an empty state.

    Returns (final_state, [result per frame]).
    """
    frames = list(frames)
    if not frames:
        raise ValueError("no frames")
    Hkv, d = frames[0][1].shape[1], frames[0][1].shape[2]
    state = LayerState.empty(Hkv, d)
    results = []
    for (q, k, v, pos) in frames:
        state, res = statekv_step(state, q, k, v, pos, B, mask_mode, select_mode)
        results.append(res)
    return state, results


def causal_attention(q, k, v):
    """Full causal self-attention over N tokens (the quadratic comparator).

    q [N][Hq][d], k/v [N][Hkv][d]; token i sees tokens 0..i.  Query head h uses
    KV head floor(h / G).  Returns out [N][Hq][d], lse [Hq][N].
    """
    q = to_f64(q)
    k = to_f64(k)
    v = to_f64(v)
    N, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    vis = np.tril(np.ones((N, N), dtype=bool))
    out = np.zeros((N, Hq, d))
    lse = np.zeros((Hq, N))
    for h in range(Hq):
        g = kv_head_of(h, Hq, Hkv)
        o_h, lse_h, _ = attend_pool(q[:, h, :], k[:, g, :], v[:, g, :], vis)
        out[:, h, :] = o_h
        lse[h] = lse_h
    return out, lse


def decode_attention(D_K, D_V, q, k, v):
    """Attention of n text tokens that follow the video, over the detailed state.

    The detailed state D keeps every frame's K/V for the final generation
    (P1 §方法步骤详情: the frame's KV go to the detailed cache; P2 related work:
    the second cache preserves full per-frame visual detail for generation).
    Text token i sees every retained video token and text tokens 0..i.
    D_K, D_V [Hkv][N][d]; q [n][Hq][d]; k, v [n][Hkv][d].  Returns
    out [n][Hq][d], lse [Hq][n] (natural log).
    """
    D_K = to_f64(D_K)
    D_V = to_f64(D_V)
    q = to_f64(q)
    k = to_f64(k)
    v = to_f64(v)
    n, Hq, d = q.shape
    Hkv = k.shape[1]
    N = D_K.shape[1]
    vis = np.ones((n, N + n), dtype=bool)
    vis[:, N:] = np.tril(np.ones((n, n), dtype=bool))
    out = np.zeros((n, Hq, d))
    lse = np.zeros((Hq, n))
    for h in range(Hq):
        g = kv_head_of(h, Hq, Hkv)
        K_pool = np.concatenate([D_K[g], k[:, g]], axis=0)
        V_pool = np.concatenate([D_V[g], v[:, g]], axis=0)
        o_h, lse_h, _ = attend_pool(q[:, h], K_pool, V_pool, vis)
        out[:, h] = o_h
        lse[h] = lse_h
    return out, lse


def causal_attention_rows(q, k, v, rows):
    """Causal attention for selected query tokens only (for large N sampling).

    rows: iterable of token indices.  Returns out [len(rows)][Hq][d],
    lse [Hq][len(rows)].  Same definition as causal_attention.
    """
    k = to_f64(k)
    v = to_f64(v)
    rows = list(rows)
    Hq, d = q.shape[1], q.shape[2]
    Hkv = k.shape[1]
    G = Hq // Hkv
    out = np.zeros((len(rows), Hq, d))
    lse = np.zeros((Hq, len(rows)))
    for r, i in enumerate(rows):
        qi = to_f64(q[i])  # [Hq][d]
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            vis = np.ones((1, i + 1), dtype=bool)
            o, l, _ = attend_pool(qi[h:h + 1], k[:i + 1, g, :], v[:i + 1, g, :], vis)
            out[r, h] = o[0]
            lse[h, r] = l[0]
    return out, lse
