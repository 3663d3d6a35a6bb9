"""Python binding of libstatekv (argument marshalling only).

Every step of the path runs in the library's CUDA kernels; this module checks
tensor shapes, dtypes and devices, passes raw device pointers and the current
CUDA stream through the C ABI (include/statekv.h) and wraps borrowed device
buffers as torch tensors without copying.  There is no fallback: if the
library is missing, importing this module raises.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("STATEKV_LIB", os.path.join(_PKG, "lib", "libstatekv.so"))

BF16, F32 = 0, 1
MASKS = {"frame_causal": 0, "frame_bidir": 1}
SELECTS = {"global": 0, "per_kv_head": 1, "recency": 2}
N_STAGES = 8
STAGES = ["attention", "attention_combine", "score", "select", "gather", "decode", "decode_combine",
          "attention_chained"]
ERRORS = {0: "OK", -1: "INVALID_ARG", -2: "UNSUPPORTED", -3: "CAPACITY", -4: "OOM", -5: "CUDA"}

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libstatekv.so not found at {LIB_PATH}; build it with "
        "`python -m kv_cache_selection_b200.build`")

lib = ctypes.CDLL(LIB_PATH)

_vp = ctypes.c_void_p
_i = ctypes.c_int
_pp = ctypes.POINTER(ctypes.c_void_p)
_ip = ctypes.POINTER(ctypes.c_int)

_SIGS = {
    "statekv_create": (_i, [_pp, _i, _i, _i, _i, _i, _i, _i, _i, _i]),
    "statekv_create_batched": (_i, [_pp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i]),
    "statekv_reserve_layers": (_i, [_vp, _i]),
    "statekv_prefill_frame": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "statekv_prefill_frame_host": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "statekv_get_compressed": (_i, [_vp, _i, _pp, _pp, _pp, _pp, _ip]),
    "statekv_get_detailed": (_i, [_vp, _i, _pp, _pp, _pp, _ip]),
    "statekv_get_step_stats": (_i, [_vp, _pp, _pp, _ip]),
    "statekv_frames": (_i, [_vp, _i]),
    "statekv_profile_enable": (_i, [_vp, _i]),
    "statekv_profile_read": (_i, [_vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong)]),
    "statekv_kernel_launches": (ctypes.c_longlong, [_vp]),
    "statekv_device_status": (_i, [_vp, _ip]),
    "statekv_set_wait_limit": (_i, [_vp, ctypes.c_longlong]),
    "statekv_destroy": (_i, [_vp]),
    "statekv_last_error": (ctypes.c_char_p, [_vp]),
    "statekv_step_noalloc": (_i, [_i] * 8 + [_vp] * 7 + [_i] + [_vp] * 8 + [_i, _i, _vp]),
    "statekv_decode": (_i, [_vp, _i, _vp, _vp, _vp, _i, _vp, _vp, _vp]),
    "full_causal_prefill": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp]),
    "full_causal_prefill_batched": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class StateKVError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code


def _check(rc, handle=None):
    if rc != 0:
        msg = lib.statekv_last_error(handle)
        raise StateKVError(rc, msg.decode() if msg else "")


def _dtype_code(dtype) -> int:
    if dtype in ("bf16", torch.bfloat16, BF16):
        return BF16
    if dtype in ("f32", torch.float32, F32):
        return F32
    raise ValueError(f"unsupported dtype {dtype!r}")


def _torch_dtype(code: int):
    return torch.bfloat16 if code == BF16 else torch.float32


# the current stream's handle without building a torch.cuda.Stream object
_raw_current_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream_ptr(stream, device_index=None) -> int:
    if stream is None:
        if _raw_current_stream is not None and device_index is not None:
            return _raw_current_stream(device_index)
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


class _DevView:
    """Exposes a borrowed device buffer through __cuda_array_interface__."""

    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {
            "shape": tuple(int(s) for s in shape), "typestr": typestr,
            "data": (int(ptr), False), "version": 3, "strides": None,
        }


def borrow(ptr: int, shape, dtype: torch.dtype) -> torch.Tensor:
    """Zero-copy torch view of library-owned device memory."""
    if dtype == torch.bfloat16:
        t = torch.as_tensor(_DevView(ptr, shape, "<i2"), device="cuda")
        return t.view(torch.bfloat16)
    typestr = {torch.float32: "<f4", torch.int32: "<i4"}[dtype]
    return torch.as_tensor(_DevView(ptr, shape, typestr), device="cuda")


def _need(t: torch.Tensor, shape, dtype, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if t.shape != shape:
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


class StateKV:
    """One StateKV cache builder (one or n_streams video streams, any layers)."""

    def __init__(self, Hq, Hkv, d, T, B, max_frames, dtype="bf16", mask="frame_causal",
                 select="global", n_streams=1):
        self.Hq, self.Hkv, self.d, self.T, self.B = Hq, Hkv, d, T, B
        self.max_frames, self.S = max_frames, n_streams
        self.dtype_code = _dtype_code(dtype)
        self.dtype = _torch_dtype(self.dtype_code)
        self.mask, self.select = mask, select
        lead = () if n_streams == 1 else (n_streams,)
        self._step_shapes = (lead + (T, Hq, d), lead + (T, Hkv, d), lead + (T,))  # q/out, k/v, pos
        h = ctypes.c_void_p()
        rc = lib.statekv_create_batched(ctypes.byref(h), n_streams, Hq, Hkv, d, T, B, max_frames,
                                        self.dtype_code, MASKS[mask], SELECTS[select])
        _check(rc)
        self._h = h

    @property
    def handle(self):
        return self._h

    def _lead(self):
        return () if self.S == 1 else (self.S,)

    def reserve_layers(self, n_layers: int):
        _check(lib.statekv_reserve_layers(self._h, n_layers), self._h)

    def prefill_frame(self, layer, q, k, v, pos, out=None, stream=None):
        """One cache-builder step; returns out [.., T, Hq, d]."""
        sq, skv, sp = self._step_shapes
        _need(q, sq, self.dtype, "q")
        _need(k, skv, self.dtype, "k")
        _need(v, skv, self.dtype, "v")
        _need(pos, sp, torch.int32, "pos")
        if out is None:
            out = torch.empty_like(q)
        _need(out, sq, self.dtype, "out")
        rc = lib.statekv_prefill_frame(self._h, layer, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                       pos.data_ptr(), out.data_ptr(), _stream_ptr(stream, q.get_device()))
        _check(rc, self._h)
        return out

    def profile(self, on=True):
        """Per-stage device timing: False/0 off, True/1 one event pair per
        kernel, 2 the attention and its split merge under one event pair
        (stage "attention_chained")."""
        _check(lib.statekv_profile_enable(self._h, int(on)), self._h)

    def profile_read(self):
        """{stage: (total_ms, launches)} since the last read (synchronises)."""
        ms = (ctypes.c_double * N_STAGES)()
        cnt = (ctypes.c_longlong * N_STAGES)()
        _check(lib.statekv_profile_read(self._h, ms, cnt), self._h)
        return {name: (ms[i], cnt[i]) for i, name in enumerate(STAGES) if name}

    def device_status(self) -> int:
        """0, or the first error code a kernel recorded (synchronises)."""
        code = ctypes.c_int()
        _check(lib.statekv_device_status(self._h, ctypes.byref(code)), self._h)
        return code.value

    def set_wait_limit(self, ns: int):
        """Pipeline-wait limit of the tensor-core kernels (<= 0: the default)."""
        _check(lib.statekv_set_wait_limit(self._h, int(ns)), self._h)

    def kernel_launches(self) -> int:
        return lib.statekv_kernel_launches(self._h)

    def prefill_frame_host(self, layer, q, k, v, pos, out, stream=None):
        """Same step from host tensors (pinned for asynchronous copies); `out`
        (host) is filled once `stream` reaches the end of the call."""
        L = self._lead()
        for t, shape, dt, name in ((q, L + (self.T, self.Hq, self.d), self.dtype, "q"),
                                   (k, L + (self.T, self.Hkv, self.d), self.dtype, "k"),
                                   (v, L + (self.T, self.Hkv, self.d), self.dtype, "v"),
                                   (pos, L + (self.T,), torch.int32, "pos"),
                                   (out, L + (self.T, self.Hq, self.d), self.dtype, "out")):
            if t.device.type != "cpu" or tuple(t.shape) != shape or t.dtype != dt or not t.is_contiguous():
                raise ValueError(f"{name}: expected contiguous host tensor {shape} {dt}")
        rc = lib.statekv_prefill_frame_host(self._h, layer, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                            pos.data_ptr(), out.data_ptr(), _stream_ptr(stream))
        _check(rc, self._h)
        return out

    def decode(self, layer, q, k, v, out=None, lse=None, with_lse=True, stream=None):
        """Attention of n text tokens over the layer's detailed state D and
        causally over themselves: q [.., n, Hq, d], k/v [.., n, Hkv, d].
        Returns (out, lse [.., Hq, n] or None)."""
        L = self._lead()
        n = q.shape[-3]
        _need(q, L + (n, self.Hq, self.d), self.dtype, "q")
        _need(k, L + (n, self.Hkv, self.d), self.dtype, "k")
        _need(v, L + (n, self.Hkv, self.d), self.dtype, "v")
        if out is None:
            out = torch.empty_like(q)
        _need(out, L + (n, self.Hq, self.d), self.dtype, "out")
        if lse is None and with_lse:
            lse = torch.empty(L + (self.Hq, n), dtype=torch.float32, device=q.device)
        if lse is not None:
            _need(lse, L + (self.Hq, n), torch.float32, "lse")
        rc = lib.statekv_decode(self._h, layer, q.data_ptr(), k.data_ptr(), v.data_ptr(), n, out.data_ptr(),
                                lse.data_ptr() if lse is not None else None, _stream_ptr(stream))
        _check(rc, self._h)
        return out, lse

    def frames(self, layer) -> int:
        return lib.statekv_frames(self._h, layer)

    def get_compressed(self, layer):
        """Borrowed views of C: k, v [S][Hkv][B][d], pos, score [S][Hkv][B], len."""
        k, v, p, s = (ctypes.c_void_p() for _ in range(4))
        n = ctypes.c_int()
        _check(lib.statekv_get_compressed(self._h, layer, ctypes.byref(k), ctypes.byref(v),
                                          ctypes.byref(p), ctypes.byref(s), ctypes.byref(n)),
               self._h)
        S, H, B, d = self.S, self.Hkv, max(self.B, 0), self.d
        return dict(
            k=borrow(k.value, (S, H, B, d), self.dtype), v=borrow(v.value, (S, H, B, d), self.dtype),
            pos=borrow(p.value, (S, H, B), torch.int32), score=borrow(s.value, (S, H, B), torch.float32),
            len=n.value)

    def get_detailed(self, layer):
        """Borrowed views of D: k, v [S][Hkv][max_frames*T][d], pos [S][max_frames*T], len."""
        k, v, p = (ctypes.c_void_p() for _ in range(3))
        n = ctypes.c_int()
        _check(lib.statekv_get_detailed(self._h, layer, ctypes.byref(k), ctypes.byref(v),
                                        ctypes.byref(p), ctypes.byref(n)), self._h)
        S, H, N, d = self.S, self.Hkv, self.max_frames * self.T, self.d
        return dict(k=borrow(k.value, (S, H, N, d), self.dtype), v=borrow(v.value, (S, H, N, d), self.dtype),
                    pos=borrow(p.value, (S, N), torch.int32), len=n.value)

    def step_stats(self):
        """Borrowed views of the last step's lse [S][Hq][T] and pool scores [S][Hkv][B+T]."""
        l, s = ctypes.c_void_p(), ctypes.c_void_p()
        n = ctypes.c_int()
        _check(lib.statekv_get_step_stats(self._h, ctypes.byref(l), ctypes.byref(s), ctypes.byref(n)),
               self._h)
        return dict(lse=borrow(l.value, (self.S, self.Hq, self.T), torch.float32),
                    pool_score=borrow(s.value, (self.S, self.Hkv, self.B + self.T), torch.float32),
                    pool_len=n.value)

    def close(self):
        if getattr(self, "_h", None):
            lib.statekv_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def full_causal_prefill(q, k, v, out=None, lse=None, with_lse=True, stream=None):
    """Full causal attention over q [(S,) N, Hq, d], k/v [(S,) N, Hkv, d]."""
    batched = q.dim() == 4
    S = q.shape[0] if batched else 1
    N, Hq, d = q.shape[-3:]
    Hkv = k.shape[-2]
    code = _dtype_code(q.dtype)
    lead = (S,) if batched else ()
    _need(q, lead + (N, Hq, d), q.dtype, "q")
    _need(k, lead + (N, Hkv, d), q.dtype, "k")
    _need(v, lead + (N, Hkv, d), q.dtype, "v")
    if out is None:
        out = torch.empty_like(q)
    _need(out, lead + (N, Hq, d), q.dtype, "out")
    if lse is None and with_lse:
        lse = torch.empty(lead + (Hq, N), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, lead + (Hq, N), torch.float32, "lse")
    rc = lib.full_causal_prefill_batched(q.data_ptr(), k.data_ptr(), v.data_ptr(), S, N, Hq, Hkv, d,
                                         code, out.data_ptr(), lse.data_ptr() if lse is not None else None,
                                         _stream_ptr(stream))
    _check(rc)
    return out, lse
