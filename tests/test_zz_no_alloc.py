"""statekv_step_noalloc: the step for callers that cannot allocate device memory
(for example a server whose memory pool already holds nearly all of the GPU,
or a latency-critical loop that cannot take cudaMalloc's device-wide
synchronisation).  It keeps its scratch in a fixed device array instead of
allocating; these tests call it through the C ABI on two calls in a row (the second one
evicts from the compressed state) and check each call against the float64
oracle with the parity tolerances of the other GPU tests, and against the
handle-based statekv_prefill_frame (bit for bit in float32, where both run
the same kernels; within tolerance in bf16, where the handle path uses the
tensor cores and this entry point the CUDA cores).

This file is collected last on purpose, so that a run that stops at the first
failure has already run every other test.
"""

import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


@needs_cuda
@pytest.mark.parametrize("dtype,select", [("bf16", "global"), ("f32", "per_kv_head")])
def test_noalloc_matches_handle_path_two_calls(dtype, select):
    import numpy as np

    from kv_cache_selection_b200 import statekv as S
    from kv_cache_selection_b200 import synthetic as Syn
    from oracle import statekv_oracle as O
    from tests import parity as P

    wl = Syn.workload("1b_layer", Hq=14, Hkv=2, d=64, T=256, B=384, frames=2, dtype=dtype)
    dev = torch.device("cuda")
    td = wl.torch_dtype
    frames_cpu = [Syn.gen_frame(wl, n) for n in range(2)]
    frames = [tuple(t.to(dev) for t in f) for f in frames_cpu]

    # existing entry point: a handle that owns C and D
    h = S.StateKV(wl.Hq, wl.Hkv, wl.d, wl.T, wl.B, max_frames=2, dtype=dtype, select=select)
    ref = []
    for f in frames:
        out = h.prefill_frame(0, *f).clone()
        C = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in h.get_compressed(0).items()}
        ref.append((out, C))
    torch.cuda.synchronize()
    D_ref = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in h.get_detailed(0).items()}
    h.close()

    # new entry point: the caller owns every buffer
    H, B, d, T = wl.Hkv, wl.B, wl.d, wl.T
    kc = [torch.zeros((H, B, d), dtype=td, device=dev) for _ in range(2)]
    vc = [torch.zeros((H, B, d), dtype=td, device=dev) for _ in range(2)]
    pc = [torch.zeros((H, B), dtype=torch.int32, device=dev) for _ in range(2)]
    sc = [torch.zeros((H, B), dtype=torch.float32, device=dev) for _ in range(2)]
    kd = torch.zeros((H, 2 * T, d), dtype=td, device=dev)
    vd = torch.zeros_like(kd)
    pd = torch.zeros((2 * T,), dtype=torch.int32, device=dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    osel = {"global": O.SELECT_GLOBAL, "per_kv_head": O.SELECT_PER_KV_HEAD}[select]
    per_head = select == "per_kv_head"
    m = 0
    cur = 0
    fn = S.lib.statekv_step_noalloc
    for n, (q, k, v, pos) in enumerate(frames):
        # the oracle starts from the caller's own C_{n-1} (teacher-forced step)
        if m:
            st = P.oracle_state_from_gpu(dict(k=kc[cur][None].clone(), v=vc[cur][None].clone(),
                                              pos=pc[cur][None].clone(), len=m))
        else:
            st = O.LayerState.empty(H, d)
        _, res = O.statekv_step(st, *frames_cpu[n][:3], frames_cpu[n][3].numpy(), B,
                                O.MASK_FRAME_CAUSAL, osel)
        out = torch.empty_like(q)
        nxt = cur ^ 1
        rc = fn(wl.Hq, wl.Hkv, d, T, B, S.BF16 if dtype == "bf16" else S.F32, S.MASKS["frame_causal"],
                S.SELECTS[select], _ptr(q), _ptr(k), _ptr(v), _ptr(pos), _ptr(kc[cur]), _ptr(vc[cur]),
                _ptr(pc[cur]), m, _ptr(out), _ptr(kc[nxt]), _ptr(vc[nxt]), _ptr(pc[nxt]), _ptr(sc[nxt]),
                _ptr(kd), _ptr(vd), _ptr(pd), n * T, 2 * T, stream)
        assert rc == 0, S.lib.statekv_last_error(None)
        torch.cuda.synchronize()
        m_new = min(B, m + T)
        # against the oracle, with the parity tolerances of every other GPU test
        P.check_out(out, res["out"], dtype, what=f"call {n + 1} out")
        for g in range(H):
            got_pos = pc[nxt][g, :m_new].cpu().numpy()
            P.check_selection(got_pos, res["kept"][g], res["score"][g], res["pool_pos"][g], B)
            where = {int(p): j for j, p in enumerate(res["pool_pos"][g])}
            sel = [where[int(p)] for p in got_pos]
            pool_k = np.concatenate([st.K_C[g], O.to_f64(frames_cpu[n][1])[:, g]])
            pool_v = np.concatenate([st.V_C[g], O.to_f64(frames_cpu[n][2])[:, g]])
            np.testing.assert_array_equal(O.to_f64(kc[nxt][g, :m_new]), pool_k[sel])
            np.testing.assert_array_equal(O.to_f64(vc[nxt][g, :m_new]), pool_v[sel])
            mass = (wl.Hq // H if per_head else wl.Hq) * T
            P.check_scores(sc[nxt][g:g + 1, :m_new], res["score"][g][sel][None], mass)
        r_out, r_C = ref[n]
        assert r_C["len"] == m_new
        if dtype == "f32":
            # same kernels as the handle path: identical results
            assert torch.equal(out, r_out)
            assert torch.equal(pc[nxt][:, :m_new], r_C["pos"][0, :, :m_new])
            assert torch.equal(kc[nxt][:, :m_new], r_C["k"][0, :, :m_new])
            assert torch.equal(sc[nxt][:, :m_new], r_C["score"][0, :, :m_new])
        else:
            # tensor-core handle path against the CUDA-core kernels here
            P.check_out(out, r_out.double().cpu().numpy(), dtype, what=f"call {n + 1} out vs handle")
        m = m_new
        cur = nxt
    assert torch.equal(kd, D_ref["k"][0])
    assert torch.equal(vd, D_ref["v"][0])
    assert torch.equal(pd, D_ref["pos"][0])


@needs_cuda
def test_noalloc_rejects_oversize_scratch():
    from kv_cache_selection_b200 import statekv as S

    bufs = [torch.zeros(16, dtype=torch.uint8, device="cuda") for _ in range(4)]
    p = _ptr(bufs[0])
    kc, vc, kc_new, vc_new = (_ptr(b) for b in bufs)
    # 8 KV heads x (30000 + 256) candidates needs ~2 MB of score scratch > 1 MiB;
    # the call is rejected before anything is enqueued
    rc = S.lib.statekv_step_noalloc(8, 8, 128, 256, 30000, S.BF16, 0, 0, p, p, p, p, kc, vc, p, 0, p,
                                    kc_new, vc_new, p, p, p, p, p, 0, 256, None)
    assert rc == -2
    assert b"scratch" in S.lib.statekv_last_error(None)
