"""Seeded synthetic inputs for the StateKV per-frame step.

This module only draws inputs: it holds none of the method's arithmetic and is
shared by the CUDA path's callers (tests, bench) and by the CPU oracle.

Inputs stand in for the backbone's per-layer projections of 1 FPS video frames
(the pages evaluate on VideoMME / MLVU / OVOBench, which are not available here);
shapes follow the 1B- and 8B-class backbones.  Recipe, per layer and frame n:

  * q [T][Hq][d], k / v [T][Hkv][d]: i.i.d. N(0, 1) ("iid") or N(0, 1)/sqrt(d)
    ("sinks");
  * q and k are rotated by RoPE (base 10000, half-split layout) at the absolute
    token positions n*T + t: the step receives keys already rotated at their
    virtual positions and only stores positions;
  * "sinks": after rotation, a fixed per-layer unit vector u is added as
    k += 4u to a few sink tokens of every frame (all KV heads) and q += 1.5u to
    every query (all heads).  Sink indices are either drawn afresh each frame or
    drift by an integer step in {-2..2} per frame, reflected into [0, T);
  * bf16 workloads round the f32 draw to bf16 once; both sides of a parity
    check receive those same bf16 values.

Every frame is a pure function of (seed, layer, stream, frame index).
"""

from __future__ import annotations

from dataclasses import dataclass, field
from functools import lru_cache

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    Hq: int
    Hkv: int
    d: int
    T: int
    B: int
    frames: int
    dtype: str            # "f32" or "bf16"
    dist: str             # "iid" or "sinks"
    n_sinks: int = 0
    drift: int = 0        # 0: fresh sink indices per frame; k>0: drift by +-k
    seed: int = 0
    layers: int = 1
    streams: int = 1
    layer_seed_stride: int = 0   # per-layer seed = seed * layer_seed_stride + layer
    notes: str = ""

    def layer_seed(self, layer: int) -> int:
        if self.layer_seed_stride:
            return self.seed * self.layer_seed_stride + layer
        return self.seed + layer

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = {
    # tiny oracle case (fp32, i.i.d.), B=32 evicts, B=128 keeps every token
    "tiny": Workload("tiny", Hq=2, Hkv=1, d=64, T=16, B=32, frames=8,
                     dtype="f32", dist="iid", seed=0),
    "tiny_noevict": Workload("tiny_noevict", Hq=2, Hkv=1, d=64, T=16, B=128,
                             frames=8, dtype="f32", dist="iid", seed=0),
    # 1B-class layer: 8 fresh sinks per frame
    "1b_layer": Workload("1b_layer", Hq=14, Hkv=2, d=64, T=256, B=1024, frames=64,
                         dtype="bf16", dist="sinks", n_sinks=8, drift=0, seed=1),
    # 8B-class layer: 16 sinks drifting +-2 per frame
    "8b_layer": Workload("8b_layer", Hq=28, Hkv=4, d=128, T=256, B=4096,
                         frames=512, dtype="bf16", dist="sinks", n_sinks=16,
                         drift=2, seed=2),
    # 8B-class stack: 28 independent layers, seeds 3*1000 + layer
    "8b_stack": Workload("8b_stack", Hq=28, Hkv=4, d=128, T=256, B=4096,
                         frames=128, dtype="bf16", dist="sinks", n_sinks=16,
                         drift=2, seed=3, layers=28, layer_seed_stride=1000),
    # 8B-class sweep shape (frames / B vary per run), 4 streams per launch
    "8b_sweep": Workload("8b_sweep", Hq=28, Hkv=4, d=128, T=256, B=4096,
                         frames=512, dtype="bf16", dist="sinks", n_sinks=16,
                         drift=2, seed=4, streams=4),
}


def workload(name: str, **overrides) -> Workload:
    wl = WORKLOADS[name]
    if overrides:
        fields = dict(wl.__dict__)
        fields.update(overrides)
        wl = Workload(**fields)
    return wl


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(x) for x in key])))


def _rope(x: np.ndarray, positions: np.ndarray, base: float = 10000.0) -> np.ndarray:
    """Rotate x [T][H][d] at positions [T] (half-split pairs (j, j + d/2))."""
    d = x.shape[-1]
    half = d // 2
    inv_freq = base ** (-np.arange(half, dtype=np.float64) * 2.0 / d)
    ang = positions.astype(np.float64)[:, None] * inv_freq[None, :]   # [T][half]
    cos = np.cos(ang)[:, None, :]
    sin = np.sin(ang)[:, None, :]
    x1 = x[..., :half].astype(np.float64)
    x2 = x[..., half:].astype(np.float64)
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def sink_direction(wl: Workload, layer: int = 0) -> np.ndarray:
    u = _rng(wl.layer_seed(layer), 7).standard_normal(wl.d)
    return u / np.linalg.norm(u)


@lru_cache(maxsize=64)
def _drift_track(seed: int, T: int, n_sinks: int, drift: int, n_frames: int) -> np.ndarray:
    """Sink indices for frames 0..n_frames-1 when sinks drift by +-drift."""
    g = _rng(seed, 11)
    idx = g.choice(T, size=n_sinks, replace=False)
    track = np.zeros((n_frames, n_sinks), dtype=np.int64)
    for n in range(n_frames):
        if n > 0:
            step = g.integers(-drift, drift + 1, size=n_sinks)
            idx = idx + step
            idx = np.where(idx < 0, -idx, idx)                   # reflect at 0
            idx = np.where(idx > T - 1, 2 * (T - 1) - idx, idx)  # reflect at T-1
        track[n] = idx
    return track


def sink_indices(wl: Workload, layer: int, stream: int, n: int) -> np.ndarray:
    if wl.dist != "sinks" or wl.n_sinks == 0:
        return np.zeros((0,), dtype=np.int64)
    seed = wl.layer_seed(layer) * 100 + stream
    if wl.drift > 0:
        return _drift_track(seed, wl.T, wl.n_sinks, wl.drift, n + 1)[n]
    return _rng(seed, 13, n).choice(wl.T, size=wl.n_sinks, replace=False)


def frame_positions(wl: Workload, n: int) -> torch.Tensor:
    return torch.arange(n * wl.T, (n + 1) * wl.T, dtype=torch.int32)


def gen_frame(wl: Workload, n: int, layer: int = 0, stream: int = 0):
    """(q, k, v, pos) of frame n as CPU torch tensors in the workload dtype."""
    T, Hq, Hkv, d = wl.T, wl.Hq, wl.Hkv, wl.d
    g = _rng(wl.layer_seed(layer), stream, n, 3)
    q = g.standard_normal((T, Hq, d), dtype=np.float32)
    k = g.standard_normal((T, Hkv, d), dtype=np.float32)
    v = g.standard_normal((T, Hkv, d), dtype=np.float32)
    if wl.dist == "sinks":
        s = np.float32(1.0 / np.sqrt(d))
        q *= s
        k *= s
        v *= s
    pos = np.arange(n * T, (n + 1) * T)
    q = _rope(q, pos)
    k = _rope(k, pos)
    if wl.dist == "sinks":
        u = sink_direction(wl, layer)
        q = q + 1.5 * u[None, None, :]
        sinks = sink_indices(wl, layer, stream, n)
        k[sinks] = k[sinks] + 4.0 * u[None, None, :]
    dt = wl.torch_dtype
    q = torch.from_numpy(q.astype(np.float32)).to(dt)
    k = torch.from_numpy(k.astype(np.float32)).to(dt)
    v = torch.from_numpy(np.ascontiguousarray(v)).to(dt)
    return q, k, v, torch.from_numpy(pos.astype(np.int32))


def gen_frames(wl: Workload, n_frames: int | None = None, layer: int = 0,
               stream: int = 0, start: int = 0):
    n_frames = wl.frames if n_frames is None else n_frames
    return [gen_frame(wl, n, layer, stream) for n in range(start, start + n_frames)]


def gen_tokens(wl: Workload, n_tokens: int, layer: int = 0, stream: int = 0):
    """Concatenate frames into one sequence [N][H][d] (for the full causal comparator)."""
    n_frames = -(-n_tokens // wl.T)
    fr = gen_frames(wl, n_frames, layer, stream)
    q = torch.cat([f[0] for f in fr])[:n_tokens].contiguous()
    k = torch.cat([f[1] for f in fr])[:n_tokens].contiguous()
    v = torch.cat([f[2] for f in fr])[:n_tokens].contiguous()
    return q, k, v


def gen_frames_device(wl: Workload, n_frames: int, layer: int = 0, stream: int = 0,
                      device="cuda", start: int = 0):
    """The same recipe drawn with torch's device generator, for timing runs that
    need many frames (values differ from gen_frame's; parity checks use
    gen_frame).  Returns stacked q [n][T][Hq][d], k/v [n][T][Hkv][d] and
    pos [n][T] on `device`."""
    T, Hq, Hkv, d = wl.T, wl.Hq, wl.Hkv, wl.d
    g = torch.Generator(device=device)
    g.manual_seed(wl.layer_seed(layer) * 1_000_003 + stream * 10_007 + start)
    q = torch.randn((n_frames, T, Hq, d), generator=g, device=device, dtype=torch.float32)
    k = torch.randn((n_frames, T, Hkv, d), generator=g, device=device, dtype=torch.float32)
    v = torch.randn((n_frames, T, Hkv, d), generator=g, device=device, dtype=torch.float32)
    pos = (torch.arange(start * T, (start + n_frames) * T, device=device, dtype=torch.int64)
           .view(n_frames, T))
    if wl.dist == "sinks":
        s = 1.0 / float(np.sqrt(d))
        q *= s
        k *= s
        v *= s
    half = d // 2
    inv_freq = 10000.0 ** (-torch.arange(half, device=device, dtype=torch.float64) * 2.0 / d)
    ang = pos.to(torch.float64)[..., None] * inv_freq          # [n][T][half]
    cos = torch.cos(ang).to(torch.float32)[:, :, None, :]
    sin = torch.sin(ang).to(torch.float32)[:, :, None, :]

    def rope(x):
        x1, x2 = x[..., :half], x[..., half:]
        return torch.cat([x1 * cos - x2 * sin, x2 * cos + x1 * sin], dim=-1)

    q = rope(q)
    k = rope(k)
    if wl.dist == "sinks" and wl.n_sinks:
        u = torch.from_numpy(sink_direction(wl, layer)).to(device=device, dtype=torch.float32)
        q += 1.5 * u
        idx = torch.stack([torch.randperm(T, generator=g, device=device)[: wl.n_sinks] for _ in range(n_frames)])
        rows = torch.arange(n_frames, device=device)[:, None].expand_as(idx)
        k[rows, idx] += 4.0 * u
    dt = wl.torch_dtype
    return q.to(dt), k.to(dt), v.to(dt), pos.to(torch.int32)
