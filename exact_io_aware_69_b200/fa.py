"""ctypes binding of libfa.so (include/fa.h): argument marshalling only.

Every step of the attention computation runs in the library's CUDA kernels; this
module turns torch tensors into device pointers and the current CUDA stream, and
turns status codes into exceptions. It never computes attention itself, and it
raises if the library is missing -- there is no fallback path.
"""

from __future__ import annotations

import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")

FA_OK = 0
FA_ERR_INVALID = -1
FA_ERR_UNSUPPORTED = -2
FA_ERR_CUDA = -3
FA_ERR_TIMEOUT = -4
FA_BF16 = 0
FA_FP16 = 1
FA_LAYOUT_BHND = 0
FA_LAYOUT_BNHD = 1
FA_STAGE_PREPROCESS = 1
FA_STAGE_DKDV = 2
FA_STAGE_DQ = 4
FA_STAGE_ALL = 7
LAYOUTS = {"bhnd": FA_LAYOUT_BHND, "bnhd": FA_LAYOUT_BNHD}
STAGES = {"preprocess": FA_STAGE_PREPROCESS, "dkdv": FA_STAGE_DKDV, "dq_convert": FA_STAGE_DQ}

# Every symbol include/fa.h declares, with its ctypes signature.
_vp, _int, _f32, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "fa_fwd": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _f32, _int,
                      _vp]),
    "fa_fwd_qk": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _int, _f32,
                         _int, _vp]),
    "fa_bwd_workspace_size": (_sz, [_int, _int, _int, _int]),
    "fa_bwd": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int,
                      _int, _f32, _int, _vp, _sz, _vp]),
    "fa_bwd_qk": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _int,
                         _int, _int, _int, _f32, _int, _vp, _sz, _vp]),
    "fa_bwd_preprocess": (_int, [_vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _vp, _sz,
                                 _vp]),
    "fa_bwd_dkdv": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _f32,
                           _int, _vp, _sz, _vp]),
    "fa_bwd_dq_convert": (_int, [_vp, _int, _int, _int, _int, _f32, _int, _vp, _sz, _vp]),
    "fa_bwd_noalloc": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _int,
                              _int, _int, _f32, _int, _vp]),
    "fa_fwd_ex": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _int, _int,
                         _int, _f32, _int, _vp]),
    "fa_bwd_ex_workspace_size": (_sz, [_int, _int, _int, _int, _int, _int]),
    "fa_bwd_ex": (_int, [_vp] * 10 + [_int] * 9 + [_f32, _int, _vp, _sz, _vp]),
    "fa_bwd_ex_stage": (_int, [_int] + [_vp] * 10 + [_int] * 9 + [_f32, _int, _vp, _sz, _vp]),
    "fa_tile_range": (_int, [_int] * 6 + [ctypes.POINTER(_int)] * 2),
    "fa_decode_workspace_size": (_sz, [_int] * 7),
    "fa_decode": (_int, [_vp] * 5 + [_int] * 8 + [_f32, _int, _vp, _sz, _vp]),
    "fa_get_device_status": (_int, [_vp]),
    "fa_selftest_wait_timeout": (_int, [ctypes.c_longlong, _vp]),
    "fa_selftest_exp2": (_int, [_vp, _vp, _int, _vp]),
    "fa_status_string": (ctypes.c_char_p, [_int]),
    "fa_version": (_int, []),
}

_lib = None


class FaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def load():
    """Load libfa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m exact_io_aware_69_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().fa_status_string(int(status)).decode()


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return FA_BF16
    if t.dtype == torch.float16:
        return FA_FP16
    raise FaError(FA_ERR_UNSUPPORTED, f"dtype {t.dtype}")


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(t, name, like=None):
    if not t.is_cuda:
        raise FaError(FA_ERR_INVALID, f"{name} is not a CUDA tensor")
    if not t.is_contiguous():
        raise FaError(FA_ERR_INVALID, f"{name} is not contiguous")
    if like is not None and (t.shape != like.shape or t.dtype != like.dtype):
        raise FaError(FA_ERR_INVALID, f"{name} shape/dtype differs from q")


def _ptr_or_none(t):
    return None if t is None else t.data_ptr()


def _dims(t, layout):
    """(B, H, N, d) of a tensor in `layout` ("bhnd": [B, H, N, d], "bnhd": [B, N, H, d])."""
    if t.dim() != 4:
        raise FaError(FA_ERR_INVALID, "expected a 4-D tensor")
    if layout == "bhnd":
        return tuple(t.shape)
    if layout == "bnhd":
        B, N, H, d = t.shape
        return B, H, N, d
    raise FaError(FA_ERR_INVALID, f"layout {layout!r}")


def _check_kv(q, k, v, layout="bhnd"):
    """k and v: like q except for the sequence length."""
    _check(k, "k")
    _check(v, "v", k)
    Bq, Hq, _, dq = _dims(q, layout)
    Bk, Hk, _, dk = _dims(k, layout)
    if (Bq, Hq, dq) != (Bk, Hk, dk) or k.dtype != q.dtype:
        raise FaError(FA_ERR_INVALID, "k/v batch, heads, head dim or dtype differ from q")


def _window(causal, window):
    """(left, right) key window; `window` overrides `causal` ((-1, 0) when set)."""
    if window is not None:
        return int(window[0]), int(window[1])
    return (-1, 0) if causal else (-1, -1)


def forward(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None,
            out_res=None, residual: bool = True, stream=None, window=None, layout="bhnd"):
    """(O, L, O_res) = attention(q, k, v) for bf16/fp16 CUDA tensors in `layout` ("bhnd":
    q [B, H, Nq, d], k and v [B, H, Nk, d]; "bnhd": [B, N, H, d]). Masks: `causal`, or
    a key window (left, right) around the bottom-right diagonal, negative = unbounded.

    O_res is the 16-bit rounding residual of O (None when residual=False); pass it to
    backward() so that D = rowsum(dO * O) is formed from O at near-fp32 precision."""
    import torch
    lib = load()
    _check(q, "q")
    _check_kv(q, k, v, layout)
    B, H, N, d = _dims(q, layout)
    Nk = _dims(k, layout)[2]
    wl, wr = _window(causal, window)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
    if out_res is None and residual:
        out_res = torch.empty_like(q)
    rc = lib.fa_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                       _ptr_or_none(out_res), lse.data_ptr(), B, H, N, Nk, d, LAYOUTS[layout],
                       wl, wr, float(scale), _dtype_code(q), _stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_ex")
    return out, lse, out_res


def workspace_size(B, H, N, d, Nk=None, deterministic=False) -> int:
    return int(load().fa_bwd_ex_workspace_size(B, H, N, N if Nk is None else Nk, d,
                                               int(bool(deterministic))))


def _bwd_call(stages, q, k, v, o, lse, do, dq, dk, dv, workspace, causal, scale, o_res,
              stream, window, layout, deterministic):
    lib = load()
    B, H, N, d = _dims(q, layout)
    Nk = _dims(k, layout)[2]
    wl, wr = _window(causal, window)

    def p(t):
        return None if t is None else t.data_ptr()
    rc = lib.fa_bwd_ex_stage(stages, p(q), p(k), p(v), p(o), p(o_res), p(do), p(lse), p(dq),
                             p(dk), p(dv), B, H, N, Nk, d, LAYOUTS[layout], wl, wr,
                             int(bool(deterministic)), float(scale), _dtype_code(q),
                             workspace.data_ptr(),
                             workspace.numel() * workspace.element_size(), _stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, f"fa_bwd_ex_stage({stages})")


def backward(q, k, v, o, lse, do, causal: bool = False, scale: float | None = None,
             o_res=None, workspace=None, dq=None, dk=None, dv=None, stream=None, window=None,
             layout="bhnd", deterministic=False):
    """dQ, dK, dV of attention, recomputing P from q, k, v and the forward's lse
    (o_res: the forward's rounding residual of O, or None). Masks and layouts as in
    forward()."""
    import torch
    for t, n in ((q, "q"), (o, "o"), (do, "do")):
        _check(t, n, q)
    _check_kv(q, k, v, layout)
    _check(lse, "lse")
    B, H, N, d = _dims(q, layout)
    Nk = _dims(k, layout)[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = workspace_size(B, H, N, d, Nk, deterministic)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=q.device, dtype=torch.uint8)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(k) if dv is None else dv
    _bwd_call(FA_STAGE_ALL, q, k, v, o, lse, do, dq, dk, dv, workspace, causal, scale, o_res,
              stream, window, layout, deterministic)
    return dq, dk, dv


def backward_stage(stage: str, q, k, v, o, lse, do, dq, dk, dv, workspace, causal: bool,
                   scale: float, o_res=None, stream=None, window=None, layout="bhnd",
                   deterministic=False) -> None:
    """Run one stage of the backward ("preprocess", "dkdv" or "dq_convert") on buffers
    the caller already holds; the three in that order equal backward()."""
    if stage not in STAGES:
        raise ValueError(stage)
    _bwd_call(STAGES[stage], q, k, v, o, lse, do, dq, dk, dv, workspace, causal, scale, o_res,
              stream, window, layout, deterministic)


def tile_range(query_side: bool, tile: int, Nq: int, Nk: int, window) -> tuple[int, int]:
    """(first, count) of the tiles a query tile (query_side) or key tile visits."""
    first, count = ctypes.c_int(), ctypes.c_int()
    rc = load().fa_tile_range(int(bool(query_side)), tile, Nq, Nk, int(window[0]),
                              int(window[1]), ctypes.byref(first), ctypes.byref(count))
    if rc != FA_OK:
        raise FaError(rc, "fa_tile_range")
    return first.value, count.value


def decode(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None,
           workspace=None, stream=None, window=None, layout="bhnd"):
    """(O, L) for a few query rows (1 <= Nq <= 16 per head) against a long key sequence:
    the split-KV decode path, forward only. Shapes, masks and layouts as in forward()."""
    import torch
    lib = load()
    _check(q, "q")
    _check_kv(q, k, v, layout)
    B, H, N, d = _dims(q, layout)
    Nk = _dims(k, layout)[2]
    wl, wr = _window(causal, window)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
    need = int(lib.fa_decode_workspace_size(B, H, N, Nk, d, wl, wr))
    if workspace is None and need > 0:
        workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
    ws = None if workspace is None else workspace.data_ptr()
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib.fa_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                       B, H, N, Nk, d, LAYOUTS[layout], wl, wr, float(scale), _dtype_code(q), ws,
                       wsb, _stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_decode")
    return out, lse


def device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error word."""
    return int(load().fa_get_device_status(_stream_handle(stream)))
