"""The C-ABI library loads on a machine without a GPU and exports every
function that include/*.h declares; argument errors that the host catches
before touching the device return the documented status codes."""

import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DECL = re.compile(r"^\s*(?:int|const\s+char\s*\*|int64_t|long long)\s+\**(\w+)\s*\(", re.M)


def declared_functions():
    names = []
    for hdr in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(hdr).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += DECL.findall(text)
    return names


def test_header_declares_boundary():
    names = set(declared_functions())
    for required in ["statekv_create", "statekv_prefill_frame", "statekv_get_compressed",
                     "statekv_get_detailed", "statekv_destroy", "statekv_last_error",
                     "full_causal_prefill"]:
        assert required in names


def test_library_exports_every_declared_symbol():
    from kv_cache_selection_b200 import statekv as S
    missing = [n for n in declared_functions() if not hasattr(S.lib, n)]
    assert not missing, f"not exported: {missing}"


def test_host_side_argument_errors():
    from kv_cache_selection_b200 import statekv as S
    h = ctypes.c_void_p()
    # Hq not a multiple of Hkv
    assert S.lib.statekv_create(ctypes.byref(h), 3, 2, 64, 16, 32, 8, 0, 0, 0) == -1
    assert b"Hkv" in S.lib.statekv_last_error(None)
    # unsupported head dim
    assert S.lib.statekv_create(ctypes.byref(h), 2, 1, 96, 16, 32, 8, 0, 0, 0) == -2
    # bad enums
    assert S.lib.statekv_create(ctypes.byref(h), 2, 1, 64, 16, 32, 8, 7, 0, 0) == -1
    assert S.lib.statekv_create(ctypes.byref(h), 2, 1, 64, 16, 32, 8, 0, 5, 0) == -1
    assert S.lib.statekv_create(ctypes.byref(h), 2, 1, 64, 16, 32, 8, 0, 0, 9) == -1
    # negative budget, empty frames
    assert S.lib.statekv_create(ctypes.byref(h), 2, 1, 64, 16, -1, 8, 0, 0, 0) == -1
    assert S.lib.statekv_create(ctypes.byref(h), 2, 1, 64, 0, 32, 8, 0, 0, 0) == -1
    # null handle pointer and null handle
    assert S.lib.statekv_create(None, 2, 1, 64, 16, 32, 8, 0, 0, 0) == -1
    assert S.lib.statekv_prefill_frame(None, 0, None, None, None, None, None, None) == -1
    assert S.lib.statekv_destroy(None) == -1
    assert h.value is None
    # full_causal_prefill argument checks
    assert S.lib.full_causal_prefill(None, None, None, 4, 2, 1, 64, 0, None, None, None) == -1
    assert S.lib.statekv_frames(None, 0) == 0
    # select modes: 3 does not exist; 2 (recency retention) passes the host checks
    assert S.lib.statekv_create(ctypes.byref(h), 2, 1, 64, 16, 32, 8, 0, 0, 3) == -1
    assert b"select" in S.lib.statekv_last_error(None)
    h2 = ctypes.c_void_p()
    rc = S.lib.statekv_create(ctypes.byref(h2), 2, 1, 64, 16, 32, 8, 0, 0, 2)
    assert rc != -1, S.lib.statekv_last_error(None)
    if rc == 0:
        S.lib.statekv_destroy(h2)
    assert S.SELECTS == {"global": 0, "per_kv_head": 1, "recency": 2}


def test_binding_refuses_missing_library(tmp_path, monkeypatch):
    """No fallback: the binding raises if the library is absent."""
    import importlib
    import sys
    monkeypatch.setenv("STATEKV_LIB", str(tmp_path / "nope.so"))
    sys.modules.pop("kv_cache_selection_b200.statekv", None)
    with pytest.raises(ImportError):
        importlib.import_module("kv_cache_selection_b200.statekv")
    monkeypatch.delenv("STATEKV_LIB")
    sys.modules.pop("kv_cache_selection_b200.statekv", None)
    importlib.import_module("kv_cache_selection_b200.statekv")


def test_noalloc_host_side_errors():
    """statekv_step_noalloc validates its arguments before any device call, so
    these refusals need no GPU.  The pointers are never dereferenced."""
    from kv_cache_selection_b200 import statekv as S
    p = ctypes.c_void_p(4096)                  # aligned, never touched
    q = ctypes.c_void_p(4096 + 8)              # misaligned
    kc, vc = ctypes.c_void_p(8192), ctypes.c_void_p(12288)
    f = S.lib.statekv_step_noalloc

    def call(Hq=2, Hkv=1, d=64, T=16, B=32, dtype=S.BF16, mask=0, select=0, qp=p, kcp=kc, vcp=vc,
             kc_new=p, m=0, d_len=0, max_tok=64, posc=p, posc_new=p):
        return f(Hq, Hkv, d, T, B, dtype, mask, select, qp, p, p, p, kcp, vcp, posc, m, p,
                 kc_new, ctypes.c_void_p(16384), posc_new, p, p, p, p, d_len, max_tok, None)

    assert call(Hq=3, Hkv=2) == -1                       # Hq not a multiple of Hkv
    assert call(d=96) == -2                              # unsupported head dim
    assert call(select=3) == -1                          # no such select mode
    assert call(mask=5) == -1
    assert call(m=40) == -1                              # C longer than its capacity
    assert call(d_len=60) == -3                          # D full
    assert call(qp=q) == -1                              # misaligned tensor
    assert call(kc_new=kc) == -1                         # C_n over C_{n-1}
    assert call(posc=ctypes.c_void_p(4098)) == -1        # misaligned int32 positions
    assert b"4-byte" in S.lib.statekv_last_error(None)
    assert call(Hq=8, Hkv=8, d=128, T=256, B=30000, max_tok=512) == -2   # beyond the fixed scratch
    assert b"statekv_create" in S.lib.statekv_last_error(None)


def test_noalloc_rejects_overlapping_buffers():
    """Every output of statekv_step_noalloc must be disjoint from every input
    and from the other outputs (its kernels read C_{n-1} and the frame while
    they write C_n).  Checked on the host: the pointers are never touched."""
    from kv_cache_selection_b200 import statekv as S
    f = S.lib.statekv_step_noalloc
    Hq, Hkv, d, T, B, max_tok = 2, 1, 64, 16, 32, 64
    es = 2
    sizes = dict(q=T * Hq * d * es, k=T * Hkv * d * es, v=T * Hkv * d * es, pos=T * 4,
                 kc=Hkv * B * d * es, vc=Hkv * B * d * es, posc=Hkv * B * 4, out=T * Hq * d * es,
                 kc_new=Hkv * B * d * es, vc_new=Hkv * B * d * es, posc_new=Hkv * B * 4,
                 scorec_new=Hkv * B * 4, kd=Hkv * max_tok * d * es, vd=Hkv * max_tok * d * es,
                 posd=max_tok * 4)
    base, addr = 1 << 20, {}
    for name, n in sizes.items():          # disjoint, 256-byte aligned fake addresses
        addr[name] = base
        base += (n + 255) // 256 * 256

    def call(**over):
        a = dict(addr, **over)
        P = {k: ctypes.c_void_p(v) for k, v in a.items()}
        return f(Hq, Hkv, d, T, B, S.BF16, 0, 0, P["q"], P["k"], P["v"], P["pos"], P["kc"], P["vc"],
                 P["posc"], 0, P["out"], P["kc_new"], P["vc_new"], P["posc_new"], P["scorec_new"],
                 P["kd"], P["vd"], P["posd"], 0, max_tok, None)

    for out_name, in_name in (("posc_new", "posc"), ("scorec_new", "posc"), ("out", "q"),
                              ("kd", "k"), ("posd", "pos"), ("vc_new", "kc_new")):
        assert call(**{out_name: addr[in_name]}) == -1, (out_name, in_name)
        assert b"overlap" in S.lib.statekv_last_error(None)
    # a partial overlap (last bytes of an input) is refused too
    assert call(posc_new=addr["posc"] + sizes["posc"] - 16) == -1
