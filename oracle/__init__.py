"""fp64 CPU oracle for exact attention (forward and backward).

TEST INFRASTRUCTURE ONLY. Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg may import this package. The CUDA library never links
or calls it, and it imports nothing from the CUDA package.

The arithmetic lives in ``attn_oracle.c`` (plain C, OpenMP over rows, every sum and
product in double); this module compiles it with gcc when the shared object is
missing or older than the source, and marshals numpy arrays through ctypes.
``recurrence.py`` holds a second, independent restatement of the pages' per-row
online-softmax recurrence that the tests pin against this oracle.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

# Portable x86-64 baseline plus AVX2/FMA (present on every current server CPU);
# the library is built here and may run on another host.
CFLAGS = ["-O3", "-mavx2", "-mfma", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall"]


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into liboracle.so next to it (no-op when up to date)."""
    with _lock:
        if (not force and os.path.exists(_LIB)
                and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
            return _LIB
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
        return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
    L_ = ctypes.c_long
    dp = ctypes.c_void_p
    lib.oracle_attn_fwd.argtypes = [f64p, f64p, f64p, L_, L_, L_, ctypes.c_int, ctypes.c_double,
                                    dp, dp]
    lib.oracle_attn_bwd.argtypes = [f64p, f64p, f64p, f64p, L_, L_, L_, ctypes.c_int,
                                    ctypes.c_double, dp, dp, dp, dp, dp, dp]
    lib.oracle_attn_fwd_qk.argtypes = [f64p, f64p, f64p, L_, L_, L_, L_, ctypes.c_int,
                                       ctypes.c_double, dp, dp]
    lib.oracle_attn_bwd_qk.argtypes = [f64p, f64p, f64p, f64p, L_, L_, L_, L_, ctypes.c_int,
                                       ctypes.c_double, dp, dp, dp, dp, dp, dp]
    lib.oracle_attn_window.argtypes = [f64p, f64p, f64p, dp, L_, L_, L_, L_, L_, L_,
                                       ctypes.c_double, dp, dp, dp, dp, dp, dp]
    lib.oracle_attn_rows.argtypes = [f64p, f64p, f64p, dp, L_, L_, L_, ctypes.c_int,
                                     ctypes.c_double, L_, dp, dp, dp, dp, dp, dp]
    lib.oracle_attn_keys.argtypes = [f64p, f64p, f64p, f64p, L_, L_, L_, ctypes.c_int,
                                     ctypes.c_double, L_, dp, dp, dp, dp]
    for fn in ("oracle_attn_fwd", "oracle_attn_bwd", "oracle_attn_fwd_qk", "oracle_attn_bwd_qk",
               "oracle_attn_rows", "oracle_attn_keys", "oracle_attn_window"):
        getattr(lib, fn).restype = ctypes.c_int
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_set_threads.argtypes = [ctypes.c_int]
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(x):
    return np.ascontiguousarray(x, dtype=np.float64)


def _check(rc, name):
    if rc != 0:
        raise RuntimeError(f"{name} failed with code {rc}")


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def _shape(q):
    if q.ndim == 3:
        return q.shape
    if q.ndim == 4:
        return (q.shape[0] * q.shape[1], q.shape[2], q.shape[3])
    raise ValueError("expected [BH, N, d] or [B, H, N, d]")


def attn_fwd(q, k, v, causal: bool, scale: float):
    """Naive attention forward. Returns (O [.., N_q, d] float64, L [.., N_q] float64).

    k and v may have another sequence length N_k than q; causal masking is then
    bottom-right aligned (query i sees keys j <= i + N_k - N_q), and a query row that
    sees no key has O = 0 and L = -inf.
    """
    lib = _load()
    shp = q.shape
    BH, Nq, d = _shape(q)
    Nk = _shape(k)[1]
    q, k, v = _f64(q), _f64(k), _f64(v)
    o = np.empty((BH, Nq, d), np.float64)
    L = np.empty((BH, Nq), np.float64)
    _check(lib.oracle_attn_fwd_qk(q, k, v, BH, Nq, Nk, d, int(causal), float(scale), _ptr(o),
                                  _ptr(L)), "oracle_attn_fwd_qk")
    return o.reshape(shp), L.reshape(shp[:-1])


def attn_bwd(q, k, v, do, causal: bool, scale: float):
    """Naive attention forward and analytic backward.

    Returns a dict with float64 arrays o, L, dq, dk, dv and D (= sum_j P_ij dP_ij).
    k and v may be longer or shorter than q, as in attn_fwd; dk and dv then have k's
    shape.
    """
    lib = _load()
    shp, kshp = q.shape, k.shape
    BH, Nq, d = _shape(q)
    Nk = _shape(k)[1]
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    out = {name: np.empty((BH, Nq, d), np.float64) for name in ("o", "dq")}
    out.update({name: np.empty((BH, Nk, d), np.float64) for name in ("dk", "dv")})
    out["L"] = np.empty((BH, Nq), np.float64)
    out["D"] = np.empty((BH, Nq), np.float64)
    _check(lib.oracle_attn_bwd_qk(q, k, v, do, BH, Nq, Nk, d, int(causal), float(scale),
                                  _ptr(out["o"]), _ptr(out["L"]), _ptr(out["dq"]),
                                  _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["D"])),
           "oracle_attn_bwd_qk")
    for name in ("o", "dq"):
        out[name] = out[name].reshape(shp)
    for name in ("dk", "dv"):
        out[name] = out[name].reshape(kshp)
    out["L"] = out["L"].reshape(shp[:-1])
    out["D"] = out["D"].reshape(shp[:-1])
    return out


def attn_rows(q, k, v, do, causal: bool, scale: float, bh_idx, row_idx):
    """O, L (and dQ, D when ``do`` is given) for selected (head, query row) pairs only."""
    lib = _load()
    BH, N, d = _shape(q)
    q, k, v = _f64(q), _f64(k), _f64(v)
    do = None if do is None else _f64(do)
    bh_idx = np.ascontiguousarray(bh_idx, dtype=np.int64)
    row_idx = np.ascontiguousarray(row_idx, dtype=np.int64)
    n = bh_idx.size
    o = np.empty((n, d), np.float64)
    L = np.empty(n, np.float64)
    dq = np.empty((n, d), np.float64) if do is not None else None
    D = np.empty(n, np.float64) if do is not None else None
    _check(lib.oracle_attn_rows(q, k, v, _ptr(do), BH, N, d, int(causal), float(scale), n,
                                _ptr(bh_idx), _ptr(row_idx), _ptr(o), _ptr(L), _ptr(dq), _ptr(D)),
           "oracle_attn_rows")
    return {"o": o, "L": L, "dq": dq, "D": D}


def attn_keys(q, k, v, do, causal: bool, scale: float, bh_idx, key_idx):
    """dK and dV for selected (head, key) pairs only."""
    lib = _load()
    BH, N, d = _shape(q)
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    bh_idx = np.ascontiguousarray(bh_idx, dtype=np.int64)
    key_idx = np.ascontiguousarray(key_idx, dtype=np.int64)
    n = bh_idx.size
    dk = np.empty((n, d), np.float64)
    dv = np.empty((n, d), np.float64)
    _check(lib.oracle_attn_keys(q, k, v, do, BH, N, d, int(causal), float(scale), n,
                                _ptr(bh_idx), _ptr(key_idx), _ptr(dk), _ptr(dv)),
           "oracle_attn_keys")
    return {"dk": dk, "dv": dv}


def attn_window(q, k, v, do, window, scale: float):
    """Attention with a (left, right) key window (negative = unbounded on that side):
    query i sees keys j with i + Nk - Nq - left <= j <= i + Nk - Nq + right.
    (-1, -1) is unmasked attention, (-1, 0) the bottom-right causal mask. ``do`` may be
    None for the forward alone. Returns a dict like attn_bwd (gradients None without
    ``do``)."""
    lib = _load()
    shp, kshp = q.shape, k.shape
    BH, Nq, d = _shape(q)
    Nk = _shape(k)[1]
    wl, wr = (int(w) for w in window)
    q, k, v = _f64(q), _f64(k), _f64(v)
    do = None if do is None else _f64(do)
    out = {"o": np.empty((BH, Nq, d), np.float64), "L": np.empty((BH, Nq), np.float64)}
    if do is not None:
        out["dq"] = np.empty((BH, Nq, d), np.float64)
        out["dk"] = np.empty((BH, Nk, d), np.float64)
        out["dv"] = np.empty((BH, Nk, d), np.float64)
        out["D"] = np.empty((BH, Nq), np.float64)
    _check(lib.oracle_attn_window(q, k, v, _ptr(do), BH, Nq, Nk, d, wl, wr, float(scale),
                                  _ptr(out["o"]), _ptr(out["L"]), _ptr(out.get("dq")),
                                  _ptr(out.get("dk")), _ptr(out.get("dv")), _ptr(out.get("D"))),
           "oracle_attn_window")
    res = {"o": out["o"].reshape(shp), "L": out["L"].reshape(shp[:-1])}
    if do is not None:
        res.update(dq=out["dq"].reshape(shp), dk=out["dk"].reshape(kshp),
                   dv=out["dv"].reshape(kshp), D=out["D"].reshape(shp[:-1]))
    else:
        res.update(dq=None, dk=None, dv=None, D=None)
    return res
