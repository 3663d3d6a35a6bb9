"""GPU parity of the StateKV step (C ABI through the Python binding) against
the float64 oracle, per step ("teacher forced"): at every checked frame the
oracle starts from the GPU's own compressed state C_{n-1}, runs one step on the
same inputs and is compared with the GPU's out, lse, pool scores and kept set.
D and the rows of C are checked bit-exact against the source tokens.
"""

import numpy as np
import pytest
import torch

from oracle import statekv_oracle as O
from kv_cache_selection_b200 import synthetic as Syn
from tests import parity as P

pytestmark = pytest.mark.gpu

cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def _skv():
    from kv_cache_selection_b200 import statekv
    return statekv


def _clone_C(C):
    return {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in C.items()}


def run_stream_parity(wl, n_frames, check, B=None, mask="frame_causal", select="global",
                      n_streams=1, layer=0, host=False):
    """Run n_frames on the GPU; teacher-forced oracle check at frames in `check`.
    host=True drives the step through statekv_prefill_frame_host (pinned host
    inputs and output, copies enqueued by the library)."""
    S = _skv()
    B = wl.B if B is None else B
    dev = torch.device("cuda")
    h = S.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, B, max_frames=n_frames, dtype=wl.dtype,
                  mask=mask, select=select, n_streams=n_streams)
    omask = O.MASK_FRAME_CAUSAL if mask == "frame_causal" else O.MASK_FRAME_BIDIR
    osel = {"global": O.SELECT_GLOBAL, "per_kv_head": O.SELECT_PER_KV_HEAD, "recency": O.SELECT_RECENCY}[select]
    per_head = select == "per_kv_head"
    G = wl.Hq // wl.Hkv
    mass = G * wl.T if per_head else wl.Hq * wl.T
    all_frames = [[Syn.gen_frame(wl, n, layer=layer, stream=s) for s in range(n_streams)]
                  for n in range(n_frames)]
    report = dict(near_boundary=0, checked=0, max_rel_l2=0.0, max_score_rel=0.0)
    for n in range(n_frames):
        fr = all_frames[n]
        stack = (lambda i: torch.stack([f[i] for f in fr]).to(dev)) if n_streams > 1 else \
                (lambda i: fr[0][i].to(dev))
        q, k, v, pos = stack(0), stack(1), stack(2), stack(3)
        do_check = n in check
        C_before = _clone_C(h.get_compressed(layer)) if (do_check and n > 0) else None
        if host:
            q, k, v, pos = (t.cpu().pin_memory() for t in (q, k, v, pos))
            out = torch.empty_like(q).pin_memory()
            h.prefill_frame_host(layer, q, k, v, pos, out)
            # the host buffers of this frame are released below: let the copies finish
            torch.cuda.synchronize()
        else:
            out = h.prefill_frame(layer, q, k, v, pos)
        if not do_check:
            continue
        torch.cuda.synchronize()
        stats = {k2: (v2.clone() if isinstance(v2, torch.Tensor) else v2) for k2, v2 in h.step_stats().items()}
        C_after = _clone_C(h.get_compressed(layer))
        for s in range(n_streams):
            st = P.oracle_state_from_gpu(C_before, s) if C_before is not None else \
                O.LayerState.empty(wl.Hkv, wl.d)
            qs, ks, vs, ps = fr[s]
            new, res = O.statekv_step(st, qs, ks, vs, ps.numpy(), B, omask, osel)
            o_s = out[s] if n_streams > 1 else out
            rel, _ = P.check_out(o_s, res["out"], wl.dtype, what=f"frame {n} stream {s} out")
            report["max_rel_l2"] = max(report["max_rel_l2"], rel)
            P.check_lse(stats["lse"][s], res["lse"], wl.dtype)
            L = stats["pool_len"]
            assert L == st.m + wl.T
            rows = slice(0, wl.Hkv) if per_head else slice(0, 1)
            sr = P.check_scores(stats["pool_score"][s, rows, :L], res["score"][rows], mass)
            report["max_score_rel"] = max(report["max_score_rel"], sr)
            assert C_after["len"] == min(B, st.m + wl.T)
            for g in range(wl.Hkv):
                got_pos = C_after["pos"][s, g, :C_after["len"]].cpu().numpy()
                if select == "recency":   # positions decide: exact
                    np.testing.assert_array_equal(got_pos, res["pool_pos"][g][res["kept"][g]])
                else:
                    report["near_boundary"] += P.check_selection(
                        got_pos, res["kept"][g], res["score"][g], res["pool_pos"][g], B)
                # kept rows are bit-exact copies of the source tokens
                pool_k = np.concatenate([st.K_C[g], O.to_f64(ks)[:, g]]) if st.m else O.to_f64(ks)[:, g]
                pool_v = np.concatenate([st.V_C[g], O.to_f64(vs)[:, g]]) if st.m else O.to_f64(vs)[:, g]
                where = {int(p): j for j, p in enumerate(res["pool_pos"][g])}
                sel = [where[int(p)] for p in got_pos]
                np.testing.assert_array_equal(O.to_f64(C_after["k"][s, g, :len(sel)]), pool_k[sel])
                np.testing.assert_array_equal(O.to_f64(C_after["v"][s, g, :len(sel)]), pool_v[sel])
                # stored scores are the pool scores of the kept candidates
                got_sc = C_after["score"][s, g, :len(sel)].cpu().numpy()
                np.testing.assert_array_equal(
                    got_sc, stats["pool_score"][s, g if per_head else 0, sel].cpu().numpy())
            report["checked"] += 1
    # D holds every frame token unmodified, in arrival order
    torch.cuda.synchronize()
    D = h.get_detailed(layer)
    assert D["len"] == n_frames * wl.T
    for s in range(n_streams):
        Kc = torch.cat([all_frames[n][s][1] for n in range(n_frames)]).transpose(0, 1)
        Vc = torch.cat([all_frames[n][s][2] for n in range(n_frames)]).transpose(0, 1)
        pc = torch.cat([all_frames[n][s][3] for n in range(n_frames)])
        assert torch.equal(D["k"][s, :, :D["len"]].cpu(), Kc)
        assert torch.equal(D["v"][s, :, :D["len"]].cpu(), Vc)
        assert torch.equal(D["pos"][s, :D["len"]].cpu(), pc)
    assert h.device_status() == 0
    h.close()
    return report


@cuda
def test_tiny_f32_every_frame():
    wl = Syn.workload("tiny")
    r = run_stream_parity(wl, wl.frames, check=range(wl.frames))
    assert r["checked"] == wl.frames


@cuda
def test_tiny_no_eviction_equals_full_causal():
    """B=128 >= 8*16 tokens: the streamed outputs equal causal attention over
    all 128 tokens (the oracle's quadratic comparator)."""
    S = _skv()
    wl = Syn.workload("tiny_noevict")
    frames = Syn.gen_frames(wl)
    h = S.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, wl.B, wl.frames, dtype="f32")
    outs = [h.prefill_frame(0, *(t.cuda() for t in f)).cpu() for f in frames]
    ref, _ = O.causal_attention(torch.cat([f[0] for f in frames]), torch.cat([f[1] for f in frames]),
                                torch.cat([f[2] for f in frames]))
    P.check_out(torch.cat(outs), ref, "f32")
    C = h.get_compressed(0)
    assert C["len"] == 128
    assert torch.equal(C["pos"][0, 0].cpu(), torch.arange(128, dtype=torch.int32))


@cuda
@pytest.mark.parametrize("mask,select", [("frame_causal", "per_kv_head"), ("frame_bidir", "global"),
                                         ("frame_bidir", "per_kv_head")])
def test_modes_small(mask, select):
    wl = Syn.workload("1b_layer", Hq=6, Hkv=2, d=64, T=24, B=40, frames=7, n_sinks=3)
    r = run_stream_parity(wl, wl.frames, check=range(wl.frames), mask=mask, select=select)
    assert r["checked"] == wl.frames


@cuda
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_recency_mode_small(dtype):
    """Recency retention: C after every frame is the last B tokens; the
    attention, scores and D are checked as in the score-based modes."""
    wl = Syn.workload("1b_layer", Hq=6, Hkv=2, d=64, T=24, B=40, frames=7, n_sinks=3, dtype=dtype)
    r = run_stream_parity(wl, wl.frames, check=range(wl.frames), select="recency")
    assert r["checked"] == wl.frames


@cuda
def test_recency_mode_1b_layer():
    """1B-class layer shape (B=1024, T=256): C fills at frame 4, then slides."""
    wl = Syn.workload("1b_layer", frames=8)
    r = run_stream_parity(wl, wl.frames, check={0, 3, 4, 7}, select="recency")
    assert r["checked"] == 4


@cuda
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
def test_ragged_shapes(dtype, d):
    """T and B not multiples of any tile; GQA group of 7."""
    wl = Syn.workload("1b_layer", Hq=7, Hkv=1, d=d, T=37, B=90, frames=6, n_sinks=4, dtype=dtype)
    run_stream_parity(wl, wl.frames, check=range(wl.frames))


@cuda
def test_zero_budget():
    wl = Syn.workload("1b_layer", Hq=4, Hkv=2, d=64, T=16, B=0, frames=3, n_sinks=2)
    r = run_stream_parity(wl, wl.frames, check=range(wl.frames), B=0)
    assert r["checked"] == 3


@cuda
def test_1b_layer_all_frames():
    wl = Syn.workload("1b_layer")
    r = run_stream_parity(wl, wl.frames, check=range(wl.frames))
    assert r["checked"] == wl.frames


@cuda
def test_8b_layer_full_size_sampled_frames():
    """The 8B-class layer at full size (512 frames, B=4096): per-step parity on
    sampled frames across the fill-up phase and the steady state."""
    wl = Syn.workload("8b_layer")
    r = run_stream_parity(wl, wl.frames, check={0, 1, 15, 16, 17, 100, 511})
    assert r["checked"] == 7


@cuda
def test_batched_streams_match_single():
    """Four streams in one handle give exactly what four single-stream handles
    give (the streams share no state)."""
    S = _skv()
    wl = Syn.workload("1b_layer", Hq=14, Hkv=2, d=64, T=64, B=192, frames=6)
    dev = torch.device("cuda")
    hb = S.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, wl.B, wl.frames, dtype="bf16", n_streams=4)
    singles = [S.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, wl.B, wl.frames, dtype="bf16") for _ in range(4)]
    for n in range(wl.frames):
        fr = [Syn.gen_frame(wl, n, stream=s) for s in range(4)]
        ob = hb.prefill_frame(0, *(torch.stack([f[i] for f in fr]).to(dev) for i in range(4)))
        for s in range(4):
            os_ = singles[s].prefill_frame(0, *(t.to(dev) for t in fr[s]))
            assert torch.equal(ob[s], os_)
    Cb = hb.get_compressed(0)
    for s in range(4):
        Cs = singles[s].get_compressed(0)
        assert torch.equal(Cb["pos"][s], Cs["pos"][0])
        assert torch.equal(Cb["k"][s], Cs["k"][0])


@cuda
def test_batched_streams_parity():
    wl = Syn.workload("1b_layer", Hq=14, Hkv=2, d=64, T=64, B=192, frames=5)
    run_stream_parity(wl, wl.frames, check=range(wl.frames), n_streams=3)


@cuda
def test_capacity_and_argument_errors():
    S = _skv()
    h = S.StateKV(2, 1, 64, 16, 32, max_frames=2, dtype="f32")
    wl = Syn.workload("tiny")
    for n in range(2):
        h.prefill_frame(0, *(t.cuda() for t in Syn.gen_frame(wl, n)))
    with pytest.raises(S.StateKVError) as e:
        h.prefill_frame(0, *(t.cuda() for t in Syn.gen_frame(wl, 2)))
    assert e.value.code == -3
    assert h.frames(0) == 2
    # a different layer is independent
    h.prefill_frame(3, *(t.cuda() for t in Syn.gen_frame(wl, 0)))
    assert h.frames(3) == 1 and h.frames(1) == 0
    with pytest.raises(S.StateKVError):
        h.get_compressed(1)  # never called (allocated by the resize, not ready)
    with pytest.raises(ValueError):
        h.prefill_frame(0, *(t.cuda() for t in Syn.gen_frame(Syn.workload("1b_layer"), 0)))


@cuda
@pytest.mark.parametrize("dtype,N,Hq,Hkv,d", [("f32", 100, 2, 1, 64), ("bf16", 333, 14, 2, 64),
                                             ("bf16", 300, 28, 4, 128), ("f32", 257, 4, 4, 128)])
def test_full_causal_prefill_small(dtype, N, Hq, Hkv, d):
    S = _skv()
    wl = Syn.workload("1b_layer", Hq=Hq, Hkv=Hkv, d=d, T=64, dtype=dtype)
    q, k, v = Syn.gen_tokens(wl, N)
    out, lse = S.full_causal_prefill(q.cuda(), k.cuda(), v.cuda())
    ref_out, ref_lse = O.causal_attention(q, k, v)
    P.check_out(out, ref_out, dtype)
    P.check_lse(lse, ref_lse, dtype)


@cuda
def test_full_causal_prefill_large_sampled_rows():
    """8B layer shape over 16 frames x 256 tokens; rows sampled across tiles."""
    S = _skv()
    wl = Syn.workload("8b_layer")
    N = 16 * 256
    q, k, v = Syn.gen_tokens(wl, N)
    out, lse = S.full_causal_prefill(q.cuda(), k.cuda(), v.cuda())
    rows = [0, 1, 127, 128, 129, 2047, 2048, 3000, N - 2, N - 1]
    ref_out, ref_lse = O.causal_attention_rows(q, k, v, rows)
    P.check_out(out[rows], ref_out, "bf16")
    P.check_lse(lse[:, rows], ref_lse, "bf16")


@cuda
def test_8b_stack_layers_interleaved():
    """28 independent 8B-class layers processed in order per frame (the
    full-stack workload): per-step parity on sampled (layer, frame) pairs across
    the fill phase and eviction; every layer's D holds its own frames."""
    S = _skv()
    wl = Syn.workload("8b_stack")
    n_frames = 18
    checks = {(0, 0), (13, 16), (27, 17), (5, 17)}
    dev = torch.device("cuda")
    h = S.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, wl.B, max_frames=n_frames, dtype="bf16")
    h.reserve_layers(wl.layers)
    for n in range(n_frames):
        for layer in range(wl.layers):
            q, k, v, pos = Syn.gen_frame(wl, n, layer=layer)
            check = (layer, n) in checks
            C_before = _clone_C(h.get_compressed(layer)) if (check and n > 0) else None
            out = h.prefill_frame(layer, q.to(dev), k.to(dev), v.to(dev), pos.to(dev))
            if not check:
                continue
            torch.cuda.synchronize()
            st = P.oracle_state_from_gpu(C_before) if C_before is not None else O.LayerState.empty(wl.Hkv, wl.d)
            _, res = O.statekv_step(st, q, k, v, pos.numpy(), wl.B)
            P.check_out(out, res["out"], "bf16", what=f"layer {layer} frame {n}")
            stats = h.step_stats()
            P.check_lse(stats["lse"][0], res["lse"], "bf16")
            P.check_scores(stats["pool_score"][0, :1, :stats["pool_len"]], res["score"][:1], wl.Hq * wl.T)
            C = h.get_compressed(layer)
            P.check_selection(C["pos"][0, 0, :C["len"]].cpu().numpy(), res["kept"][0], res["score"][0],
                              res["pool_pos"][0], wl.B)
    for layer in (0, 27):
        D = h.get_detailed(layer)
        assert D["len"] == n_frames * wl.T
        k_last = Syn.gen_frame(wl, n_frames - 1, layer=layer)[1]
        assert torch.equal(D["k"][0, :, (n_frames - 1) * wl.T:n_frames * wl.T].cpu(), k_last.transpose(0, 1))
    assert h.device_status() == 0
    h.close()


@cuda
@pytest.mark.parametrize("select", ["global", "per_kv_head"])
def test_8b_shape_score_query_split(select):
    """8B layer shape with B=2048 on one stream: the score pass splits each KV
    group's query-row chunks over several CTAs (8 at frame 0, where only the
    frame's two key tiles exist; 2 once C holds 2048 rows) and the selection
    adds their partial-sum rows.  Checked while C fills and after it evicts,
    in both selection modes."""
    wl = Syn.workload("8b_layer", B=2048, frames=10)
    r = run_stream_parity(wl, wl.frames, check={0, 1, 7, 8, 9}, select=select)
    assert r["checked"] == 5


@cuda
def test_8b_sweep_shape_four_streams():
    """The sweep workload's launch shape: 4 streams per call at the 8B layer
    shape, with B=1024 so eviction starts at frame 4."""
    wl = Syn.workload("8b_sweep", B=1024, frames=6)
    r = run_stream_parity(wl, wl.frames, check={0, 4, 5}, n_streams=4)
    assert r["checked"] == 3 * 4  # three frames, four streams


@cuda
def test_pool_above_48kb_of_selection_smem():
    """Pools whose selection needs 46 KB and 48 KB of dynamic shared memory (plus
    the kernel's static arrays, past the default 48 KB per block): B = 5888 at
    T = 256 gives pools of 5888 and 6144 candidates at frames 22 and 23."""
    wl = Syn.workload("1b_layer", B=5888, frames=24)
    r = run_stream_parity(wl, wl.frames, check={22, 23})
    assert r["checked"] == 2


@cuda
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_host_buffer_entry_parity(dtype):
    """statekv_prefill_frame_host (the end-to-end path: pinned host buffers,
    host-to-device copies, the step, the copy of out back) over frames that
    fill C and then evict, each checked against the oracle."""
    if dtype == "f32":
        wl = Syn.workload("tiny")
    else:
        wl = Syn.workload("1b_layer", Hq=14, Hkv=2, d=64, T=256, B=512, frames=5)
    r = run_stream_parity(wl, wl.frames, check=range(wl.frames), host=True)
    assert r["checked"] == wl.frames


@cuda
def test_host_and_device_entries_interleaved_without_synchronisation():
    """One layer's frames through both entry points in turn, with no host
    synchronisation between calls: the host-buffer steps run on the
    library's compute stream, so the library must order each step after the
    layer's previous one.  C, D and every frame's out equal those of a run
    through the device-buffer call alone (bit for bit: same kernels)."""
    S = _skv()
    wl = Syn.workload("1b_layer", Hq=14, Hkv=2, d=64, T=256, B=512, frames=8)
    dev = torch.device("cuda")
    frames = [Syn.gen_frame(wl, n) for n in range(wl.frames)]
    ref = S.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, wl.B, max_frames=wl.frames, dtype="bf16")
    ref_out = [ref.prefill_frame(0, *(t.to(dev) for t in fr)).clone() for fr in frames]
    torch.cuda.synchronize()
    h = S.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, wl.B, max_frames=wl.frames, dtype="bf16")
    outs, keep = [], []  # host buffers stay alive until the final synchronisation
    for n, fr in enumerate(frames):
        if n % 3 == 1 or n % 3 == 2:  # pattern: device, host, host, device, host, host, ...
            q, k, v, pos = (t.cpu().pin_memory() for t in fr)
            out = torch.empty_like(q).pin_memory()
            h.prefill_frame_host(0, q, k, v, pos, out)
            keep.append((q, k, v, pos))
            outs.append(out)
        else:
            dev_in = [t.to(dev) for t in fr]
            keep.append(dev_in)
            outs.append(h.prefill_frame(0, *dev_in))
    torch.cuda.synchronize()
    for n in range(wl.frames):
        assert torch.equal(outs[n].to(dev), ref_out[n]), f"out of frame {n}"
    Ca, Cb = h.get_compressed(0), ref.get_compressed(0)
    assert Ca["len"] == Cb["len"]
    for key in ("k", "v", "pos", "score"):
        assert torch.equal(Ca[key], Cb[key]), key
    Da, Db = h.get_detailed(0), ref.get_detailed(0)
    for key in ("k", "v", "pos"):
        assert torch.equal(Da[key], Db[key]), key
    h.close()
    ref.close()


@cuda
@pytest.mark.parametrize("dtype,Hq,Hkv,select", [("f32", 12, 12, "global"), ("bf16", 20, 10, "global"),
                                                ("bf16", 20, 10, "per_kv_head")])
def test_more_than_eight_kv_heads(dtype, Hq, Hkv, select):
    """Global selection sums the partial scores of every KV group, including
    groups past the eighth."""
    wl = Syn.workload("1b_layer", Hq=Hq, Hkv=Hkv, d=64, T=24, B=40, frames=5, n_sinks=3, dtype=dtype)
    r = run_stream_parity(wl, wl.frames, check=range(wl.frames), select=select)
    assert r["checked"] == wl.frames


@cuda
def test_full_causal_prefill_batched_8b_four_sequences():
    """full_causal_prefill_batched with four independent sequences of 2048
    tokens at the 8B layer shape (the launch shape of the crossover sweep), on
    rows sampled across tiles of every sequence."""
    S = _skv()
    wl = Syn.workload("8b_sweep")
    N = 2048
    seqs = [Syn.gen_tokens(wl, N, stream=s) for s in range(4)]
    q, k, v = (torch.stack([sq[i] for sq in seqs]).cuda() for i in range(3))
    out, lse = S.full_causal_prefill(q, k, v)
    torch.cuda.synchronize()
    rows = [0, 1, 127, 128, 255, 256, 1023, 1024, 2046, 2047]
    for s in range(4):
        ref_out, ref_lse = O.causal_attention_rows(*seqs[s], rows)
        P.check_out(out[s, rows], ref_out, "bf16", what=f"sequence {s}")
        P.check_lse(lse[s][:, rows], ref_lse, "bf16")


@cuda
def test_full_causal_prefill_long_sequence_sampled_rows():
    """One 65,536-token sequence (256 frames of the 8B layer shape, drawn on
    the device with the same recipe): sampled rows against the oracle."""
    S = _skv()
    wl = Syn.workload("8b_layer")
    n_frames = 256
    q, k, v, _ = Syn.gen_frames_device(wl, n_frames, device="cuda")
    N = n_frames * wl.T
    q = q.reshape(N, wl.Hq, wl.d).contiguous()
    k = k.reshape(N, wl.Hkv, wl.d).contiguous()
    v = v.reshape(N, wl.Hkv, wl.d).contiguous()
    out, lse = S.full_causal_prefill(q, k, v)
    torch.cuda.synchronize()
    rows = [0, 1, 4095, 4096, 32767, 32768, 50001, N - 2, N - 1]
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    ref_out, ref_lse = O.causal_attention_rows(qc, kc, vc, rows)
    P.check_out(out[rows], ref_out, "bf16")
    P.check_lse(lse[:, rows], ref_lse, "bf16")


@cuda
def test_diagnostics_library_fed_match_oracle_fed():
    """Appendix-A diagnostics computed from the library's no-eviction pool
    scores agree with the same diagnostics computed from the oracle's masses on
    the same frames (1B layer shape, 10 frames); the captured-mass comparison
    of A.3 uses the retained sets of a score-based and a recency handle."""
    import numpy as np
    from kv_cache_selection_b200 import diagnostics as Dg
    S = _skv()
    wl = Syn.workload("1b_layer", frames=10)
    n_tok = wl.frames * wl.T
    dev = torch.device("cuda")
    full = S.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, n_tok, max_frames=wl.frames, dtype=wl.dtype)
    Bsel = 512
    sel = {name: S.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, Bsel, max_frames=wl.frames, dtype=wl.dtype, select=mode)
           for name, mode in (("statekv", "global"), ("recency", "recency"))}
    st = O.LayerState.empty(wl.Hkv, wl.d)
    gpu_steps, ora_steps, kept = [], [], {name: [] for name in sel}
    for n in range(wl.frames):
        q, k, v, pos = Syn.gen_frame(wl, n)
        for name, h in sel.items():
            Cs = h.get_compressed(0) if n > 0 else None
            kept[name].append(Cs["pos"][0, 0, :Cs["len"]].cpu().numpy().copy() if Cs is not None else None)
            h.prefill_frame(0, q.to(dev), k.to(dev), v.to(dev), pos.to(dev))
        full.prefill_frame(0, q.to(dev), k.to(dev), v.to(dev), pos.to(dev))
        torch.cuda.synchronize()
        stats = full.step_stats()
        L = stats["pool_len"]
        gmass = stats["pool_score"][0, 0, :L].double().cpu().numpy()
        st, res = O.statekv_step(st, q, k, v, pos.numpy(), n_tok)
        assert L == (n + 1) * wl.T
        P.check_scores(gmass[None], res["score"][:1], wl.Hq * wl.T)
        fpos = pos.numpy().astype(np.int64)
        gpu_steps.append(dict(pos=np.arange(L, dtype=np.int64), mass=gmass, frame_pos=fpos))
        ora_steps.append(dict(pos=res["pool_pos"][0].astype(np.int64), mass=res["score"][0], frame_pos=fpos))
    budgets = [64, 256, 1024]
    rg = Dg.stream_report(gpu_steps, budgets, retained=kept)
    ro = Dg.stream_report(ora_steps, budgets, retained=kept)
    for B in budgets:
        # concentration is a sum of masses: close; the set-valued metrics may
        # differ by a swap at the B-th boundary (1/B each)
        assert abs(rg["concentration"][B] - ro["concentration"][B]) <= 1e-3
        for key in ("weighted_recall", "recall", "retention"):
            assert abs(rg[key][B] - ro[key][B]) <= 2.0 / B + 1e-3, (key, B, rg[key][B], ro[key][B])
    for name in sel:
        assert abs(rg["captured"][name] - ro["captured"][name]) <= 1e-3
    for h in list(sel.values()) + [full]:
        h.close()


def _decode_case(wl, n_frames, n_text, dtype, device_frames=False, n_streams=1):
    """Fill a handle's D with n_frames frames, then decode n_text text tokens
    over it; compare with the oracle's decode attention on the same D."""
    S = _skv()
    dev = torch.device("cuda")
    h = S.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, wl.B, max_frames=max(n_frames, 1), dtype=dtype,
                  n_streams=n_streams)
    h.reserve_layers(1)
    if device_frames:
        per = [Syn.gen_frames_device(wl, n_frames, stream=s, device=dev) for s in range(n_streams)]
        for n in range(n_frames):
            args = [torch.stack([p[i][n] for p in per]) if n_streams > 1 else per[0][i][n] for i in range(4)]
            h.prefill_frame(0, *args)
        del per
    else:
        for n in range(n_frames):
            fr = [Syn.gen_frame(wl, n, stream=s) for s in range(n_streams)]
            args = [(torch.stack([f[i] for f in fr]) if n_streams > 1 else fr[0][i]).to(dev) for i in range(4)]
            h.prefill_frame(0, *args)
    # text tokens: the recipe's next frame, first n_text tokens
    wl_txt = Syn.workload(wl.name, Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, dtype=dtype, T=n_text, dist="iid", n_sinks=0,
                          drift=0)
    txt = [Syn.gen_frame(wl_txt, n_frames, stream=s) for s in range(n_streams)]
    q = torch.stack([t[0] for t in txt]) if n_streams > 1 else txt[0][0]
    k = torch.stack([t[1] for t in txt]) if n_streams > 1 else txt[0][1]
    v = torch.stack([t[2] for t in txt]) if n_streams > 1 else txt[0][2]
    out, lse = h.decode(0, q.to(dev), k.to(dev), v.to(dev))
    torch.cuda.synchronize()
    D = h.get_detailed(0)
    N = D["len"]
    assert N == n_frames * wl.T
    for s in range(n_streams):
        DK = D["k"][s, :, :N].cpu()
        DV = D["v"][s, :, :N].cpu()
        ref_out, ref_lse = O.decode_attention(DK, DV, *(x[s] if n_streams > 1 else x for x in (q, k, v)))
        P.check_out(out[s] if n_streams > 1 else out, ref_out, dtype, what=f"decode stream {s}")
        P.check_lse(lse[s] if n_streams > 1 else lse, ref_lse, dtype)
    assert h.device_status() == 0
    h.close()


@cuda
@pytest.mark.parametrize("n_text", [1, 5, 16])
def test_decode_tiny_f32(n_text):
    _decode_case(Syn.workload("tiny"), 8, n_text, "f32")


@cuda
@pytest.mark.parametrize("n_text", [1, 7, 18, 19, 37, 130])
def test_decode_8b_shape(n_text):
    """8B layer shape after 16 frames (4096 D tokens): one stacked query tile
    (18 rows of 7 heads), a partly filled pair, two pairs, and text longer than
    one 128-token key tile."""
    _decode_case(Syn.workload("8b_layer"), 16, n_text, "bf16")


@cuda
@pytest.mark.parametrize("d,Hq,Hkv", [(64, 14, 2), (128, 8, 8)])
def test_decode_other_groups(d, Hq, Hkv):
    """Group sizes 7 and 1 and head dim 64; D that does not fill its last tile."""
    wl = Syn.workload("1b_layer", Hq=Hq, Hkv=Hkv, d=d, T=100, B=256)
    _decode_case(wl, 5, 9, "bf16")


@cuda
@pytest.mark.parametrize("n_text", [1, 12])
def test_decode_batched_streams(n_text):
    """Three streams; one text token takes the block-per-row merge of the
    split partials, twelve the row-parallel one."""
    wl = Syn.workload("1b_layer", Hq=14, Hkv=2, d=64, T=64, B=192)
    _decode_case(wl, 6, n_text, "bf16", n_streams=3)


@cuda
def test_decode_empty_detailed_state():
    """No frame yet: the text attends to itself only (causal attention)."""
    _decode_case(Syn.workload("8b_layer"), 0, 20, "bf16")


@cuda
def test_decode_8b_full_512_frames():
    """The full 8B-class stream: decode 16 text tokens over all 131,072 video
    tokens of D after 512 frames (the state the pages' generation reads)."""
    _decode_case(Syn.workload("8b_layer"), 512, 16, "bf16", device_frames=True)


@cuda
def test_pipeline_wait_timeout_is_reported_and_recovers():
    """Failure path of the tensor-core kernels, made to happen without a GPU
    fault: with a pipeline-wait limit of 1 ns the waits give up, record their
    code in the handle's device status word, drain their own copies and MMAs
    and exit.  The status reports it; with the default limit restored the next
    steps are correct again (checked against the oracle from the GPU's own
    compressed state) and report no error."""
    S = _skv()
    wl = Syn.workload("1b_layer", Hq=14, Hkv=2, d=64, T=128, B=256, frames=6)
    dev = torch.device("cuda")
    h = S.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, wl.B, max_frames=wl.frames, dtype="bf16")
    frames = [tuple(t.to(dev) for t in Syn.gen_frame(wl, n)) for n in range(wl.frames)]
    for n in range(2):
        h.prefill_frame(0, *frames[n])
    assert h.device_status() == 0
    h.set_wait_limit(1)
    codes = []
    for n in range(2, 4):
        h.prefill_frame(0, *frames[n])
        codes.append(h.device_status())
    assert any(c in (1, 2, 3, 4, 5) for c in codes), codes   # a pipeline wait gave up
    assert all(c in (0, 1, 2, 3, 4, 5) for c in codes), codes
    h.set_wait_limit(0)
    for n in range(4, 6):
        C_before = _clone_C(h.get_compressed(0))
        out = h.prefill_frame(0, *frames[n])
        torch.cuda.synchronize()
        st = P.oracle_state_from_gpu(C_before)
        q, k, v, pos = (t.cpu() for t in frames[n])
        _, res = O.statekv_step(st, q, k, v, pos.numpy(), wl.B)
        P.check_out(out, res["out"], "bf16", what=f"frame {n} after the timeout")
        stats = h.step_stats()
        P.check_lse(stats["lse"][0], res["lse"], "bf16")
        C = h.get_compressed(0)
        P.check_selection(C["pos"][0, 0, :C["len"]].cpu().numpy(), res["kept"][0], res["score"][0],
                          res["pool_pos"][0], wl.B)
    assert h.device_status() == 0
    h.close()


@cuda
def test_free_running_matches_until_a_boundary_tie():
    """Free-running comparison (the oracle keeps its own state, the GPU its
    own): the kept positions agree bit for bit frame after frame until the
    first frame whose oracle selection has a candidate within the 1e-4
    boundary band whose membership differs; that frame (if any) is reported.
    After a divergence the two states legitimately differ, so the comparison
    stops there."""
    S = _skv()
    wl = Syn.workload("1b_layer", frames=24)
    dev = torch.device("cuda")
    h = S.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, wl.B, max_frames=wl.frames, dtype="bf16")
    st = O.LayerState.empty(wl.Hkv, wl.d)
    first_tie = None
    for n in range(wl.frames):
        q, k, v, pos = Syn.gen_frame(wl, n)
        h.prefill_frame(0, q.to(dev), k.to(dev), v.to(dev), pos.to(dev))
        torch.cuda.synchronize()
        st, res = O.statekv_step(st, q, k, v, pos.numpy(), wl.B)
        C = h.get_compressed(0)
        got = C["pos"][0, 0, :C["len"]].cpu().numpy().astype(np.int64)
        want = np.asarray(st.pos_C[0], dtype=np.int64)
        if np.array_equal(got, want):
            continue
        # the sets differ: only candidates in the oracle's boundary band may
        score = res["score"][0]
        tau = np.sort(score)[::-1][wl.B - 1]
        near = set(int(p) for p, sc in zip(res["pool_pos"][0], score) if abs(sc - tau) <= P.BOUNDARY_RTOL * tau)
        diff = set(got.tolist()) ^ set(want.tolist())
        assert diff <= near, f"frame {n}: {sorted(diff - near)[:8]} differ outside the boundary band"
        first_tie = n
        break
    print(f"free-running: positions identical through frame {wl.frames - 1 if first_tie is None else first_tie - 1}"
          f"{'' if first_tie is None else f'; first boundary-tie frame {first_tie}'}")
    h.close()


@cuda
def test_layers_pipelined_on_two_streams_match_in_order():
    """Each layer owns its step scratch, so frame n+1 of layer l may run on one
    stream while frame n of layer l+1 runs on another (each layer's frames
    ordered by an event): the results equal the in-order run bit for bit."""
    S = _skv()
    wl = Syn.workload("1b_layer", Hq=14, Hkv=2, d=64, T=128, B=384, frames=6)
    n_layers = 3
    dev = torch.device("cuda")
    fr = [[tuple(t.to(dev) for t in Syn.gen_frame(wl, n, layer=l)) for l in range(n_layers)]
          for n in range(wl.frames)]
    ref = S.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, wl.B, max_frames=wl.frames, dtype="bf16")
    ref_out = {}
    for n in range(wl.frames):
        for l in range(n_layers):
            ref_out[n, l] = ref.prefill_frame(l, *fr[n][l]).clone()
    torch.cuda.synchronize()
    h = S.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, wl.B, max_frames=wl.frames, dtype="bf16")
    h.reserve_layers(n_layers)
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    done = [torch.cuda.Event() for _ in range(n_layers)]
    outs = {}
    for st in streams:
        st.wait_stream(torch.cuda.current_stream())
    for n in range(wl.frames):
        st = streams[n % 2]
        for l in range(n_layers):
            st.wait_event(done[l])
            with torch.cuda.stream(st):
                o = torch.empty_like(fr[n][l][0])
            outs[n, l] = h.prefill_frame(l, *fr[n][l], out=o, stream=st)
            done[l].record(st)
    torch.cuda.synchronize()
    for key, o in outs.items():
        assert torch.equal(o, ref_out[key]), key
    for l in range(n_layers):
        a, b = h.get_compressed(l), ref.get_compressed(l)
        assert a["len"] == b["len"]
        assert torch.equal(a["pos"], b["pos"]) and torch.equal(a["k"], b["k"]) and torch.equal(a["v"], b["v"])
    assert h.device_status() == 0
    h.close()
    ref.close()


@cuda
def test_profiling_modes_time_the_same_step():
    """Per-stage timing changes how the step is launched (mode 1: the split
    merge on its own, events around every kernel; mode 2: the attention and
    its merge under one event pair) but not what it computes: every mode
    gives bit-identical out, C and D, and records the expected stages."""
    S = _skv()
    wl = Syn.workload("1b_layer")
    dev = torch.device("cuda")
    n_frames = 7            # C fills after 4 frames (B = 1024, T = 256): 3 steady-state steps
    frames = [tuple(t.to(dev) for t in Syn.gen_frame(wl, n)) for n in range(n_frames)]
    results = {}
    for mode in (0, 1, 2):
        h = S.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, wl.B, max_frames=n_frames, dtype=wl.dtype)
        h.profile(mode)
        outs = [h.prefill_frame(0, *f).clone() for f in frames]
        torch.cuda.synchronize()
        rec = h.profile_read() if mode else {}
        C, D = h.get_compressed(0), h.get_detailed(0)
        results[mode] = (outs, {k: v.clone() for k, v in C.items() if isinstance(v, torch.Tensor)},
                         {k: v.clone() for k, v in D.items() if isinstance(v, torch.Tensor)})
        if mode == 1:
            for st in ("attention", "attention_combine", "score", "select", "gather"):
                assert rec[st][1] == n_frames, (st, rec[st])
            assert rec["attention_chained"][1] == 0
        if mode == 2:
            assert rec["attention_chained"][1] == n_frames
            assert rec["attention_combine"][1] == 0 and rec["attention"][1] == 0
            assert all(rec[st][1] == n_frames for st in ("score", "select", "gather"))
            assert rec["attention_chained"][0] > 0.0
        with pytest.raises(S.StateKVError):
            h.profile(3)
        assert h.device_status() == 0
        h.close()
    for mode in (1, 2):
        for a, b in zip(results[0][0], results[mode][0]):
            assert torch.equal(a, b)
        for part in (1, 2):
            for key, t in results[0][part].items():
                assert torch.equal(t, results[mode][part][key]), (mode, key)
