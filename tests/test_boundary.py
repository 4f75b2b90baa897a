"""Host-side checks of the C ABI (no GPU needed, nothing is launched).

The library must load on a machine without a GPU, export every function that
include/fa.h declares, and reject bad arguments with the documented status code
before touching the device.
"""

import ctypes
import os
import re

import pytest

from exact_io_aware_69_b200 import build, fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


@pytest.fixture(scope="module")
def lib():
    build.build_library()
    return fa.load()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    assert names == sorted(["fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_get_device_status",
                            "fa_status_string", "fa_version", "fa_bwd_preprocess",
                            "fa_bwd_dkdv", "fa_bwd_dq_convert", "fa_bwd_noalloc",
                            "fa_selftest_wait_timeout", "fa_fwd_qk", "fa_bwd_qk"])


def test_every_declared_symbol_is_exported(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name
        assert name in fa.SIGNATURES, name


def test_version_and_status_strings(lib):
    assert lib.fa_version() == 1
    for code, text in [(0, "FA_OK"), (-1, "FA_ERR_INVALID"), (-2, "FA_ERR_UNSUPPORTED"),
                       (-3, "FA_ERR_CUDA"), (-4, "FA_ERR_TIMEOUT"), (7, "FA_ERR_UNKNOWN")]:
        assert fa.status_string(code) == text


def test_workspace_size(lib):
    assert lib.fa_bwd_workspace_size(2, 3, 256, 64) == 2 * 3 * 256 * (8 + 64 * 4)
    assert lib.fa_bwd_workspace_size(0, 3, 256, 64) == 0
    assert lib.fa_bwd_workspace_size(-1, 3, 256, 64) == ctypes.c_size_t(-1).value


# Fake, well-aligned device addresses: validation must reject before any use.
P = 0x7F0000000000


def _fwd(lib, **kw):
    a = dict(Q=P, K=P + 0x100000, V=P + 0x200000, O=P + 0x300000, R=P + 0xa00000,
             L=P + 0x400000, B=1, H=1, N=256, d=64, causal=0, scale=0.125, dtype=fa.FA_BF16,
             stream=None)
    a.update(kw)
    return lib.fa_fwd(a["Q"], a["K"], a["V"], a["O"], a["R"], a["L"], a["B"], a["H"], a["N"],
                      a["d"], a["causal"], a["scale"], a["dtype"], a["stream"])


def _bwd(lib, **kw):
    a = dict(Q=P, K=P + 0x100000, V=P + 0x200000, O=P + 0x300000, R=P + 0xa00000,
             dO=P + 0x400000,
             L=P + 0x500000, dQ=P + 0x600000, dK=P + 0x700000, dV=P + 0x800000, B=1, H=1, N=256,
             d=64, causal=0, scale=0.125, dtype=fa.FA_BF16, ws=P + 0x900000, ws_bytes=1 << 30,
             stream=None)
    a.update(kw)
    return lib.fa_bwd(a["Q"], a["K"], a["V"], a["O"], a["R"], a["dO"], a["L"], a["dQ"], a["dK"],
                      a["dV"],
                      a["B"], a["H"], a["N"], a["d"], a["causal"], a["scale"], a["dtype"], a["ws"],
                      a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(Q=None), fa.FA_ERR_INVALID),
    (dict(L=None), fa.FA_ERR_INVALID),
    (dict(B=-1), fa.FA_ERR_INVALID),
    (dict(N=-128), fa.FA_ERR_INVALID),
    (dict(K=P + 8), fa.FA_ERR_INVALID),
    (dict(R=P + 0xa00004), fa.FA_ERR_INVALID),
    (dict(scale=0.0), fa.FA_ERR_INVALID),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID),
    (dict(scale=float("inf")), fa.FA_ERR_INVALID),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(d=256), fa.FA_ERR_UNSUPPORTED),
    (dict(B=1 << 15, H=1 << 10, N=100), fa.FA_ERR_UNSUPPORTED),  # 2^32 padded rows
    (dict(dtype=2), fa.FA_ERR_UNSUPPORTED),
    (dict(B=0), fa.FA_OK),
    (dict(N=0, Q=None, K=None, V=None, O=None, L=None), fa.FA_OK),
])
def test_fwd_rejects_before_launch(lib, kw, code):
    assert _fwd(lib, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(dO=None), fa.FA_ERR_INVALID),
    (dict(ws=None), fa.FA_ERR_INVALID),
    (dict(ws=P + 0x900010), fa.FA_ERR_INVALID),  # workspace must be 256-byte aligned
    (dict(ws_bytes=1000), fa.FA_ERR_INVALID),
    (dict(dV=P + 0x800002), fa.FA_ERR_INVALID),
    (dict(R=P + 0xa00008), fa.FA_ERR_INVALID),
    (dict(H=-2), fa.FA_ERR_INVALID),
    (dict(d=32), fa.FA_ERR_UNSUPPORTED),
    (dict(B=1 << 20, H=16, N=130), fa.FA_ERR_UNSUPPORTED),  # 2^32 padded rows
    (dict(dtype=5), fa.FA_ERR_UNSUPPORTED),
    (dict(H=0), fa.FA_OK),
])
def test_bwd_rejects_before_launch(lib, kw, code):
    assert _bwd(lib, **kw) == code


def test_selftest_rejects_bad_limits(lib):
    assert lib.fa_selftest_wait_timeout(0, None) == fa.FA_ERR_INVALID
    assert lib.fa_selftest_wait_timeout(-5, None) == fa.FA_ERR_INVALID
    assert lib.fa_selftest_wait_timeout(10 ** 12, None) == fa.FA_ERR_INVALID


def test_binding_raises_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(fa, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(fa, "_lib", None)
    with pytest.raises(ImportError):
        fa.load()


@pytest.mark.parametrize("B,H,N,d", [(1, 2, 200, 64), (2, 3, 128, 128), (1, 1, 1, 128),
                                     (3, 1, 8193, 64)])
def test_workspace_size_pads_rows_per_head(lib, B, H, N, d):
    """D and Ls take N rounded up to 128 per head; the fp32 dQ accumulator that follows
    them starts on a 1024-byte boundary and holds exactly B*H*N*d values."""
    n_pad = -(-N // 128) * 128
    want = B * H * n_pad * 8 + B * H * N * d * 4
    assert lib.fa_bwd_workspace_size(B, H, N, d) == want
    assert (B * H * n_pad * 8) % 1024 == 0


def _fwd_qk(lib, Nq, Nk, **kw):
    a = dict(Q=P, K=P + 0x100000, V=P + 0x200000, O=P + 0x300000, R=None, L=P + 0x400000, B=1,
             H=1, d=64, causal=1, scale=0.125, dtype=fa.FA_BF16)
    a.update(kw)
    return lib.fa_fwd_qk(a["Q"], a["K"], a["V"], a["O"], a["R"], a["L"], a["B"], a["H"], Nq, Nk,
                         a["d"], a["causal"], a["scale"], a["dtype"], None)


def test_qk_shapes_rejected_before_launch(lib):
    """Nk = 0 with queries has no softmax; lengths are checked like N; Nq = 0 is empty."""
    assert _fwd_qk(lib, 128, 0) == fa.FA_ERR_INVALID
    assert _fwd_qk(lib, -1, 128) == fa.FA_ERR_INVALID
    assert _fwd_qk(lib, 128, -5) == fa.FA_ERR_INVALID
    assert _fwd_qk(lib, 128, 256, d=96) == fa.FA_ERR_UNSUPPORTED
    assert _fwd_qk(lib, 0, 256, Q=None, O=None, L=None) == fa.FA_OK
    assert _fwd_qk(lib, 100, 1 << 30, B=4) == fa.FA_ERR_UNSUPPORTED  # 2^32 padded key rows
    # no queries: the backward only zeroes dK and dV, which must then be valid
    assert lib.fa_bwd_qk(None, None, None, None, None, None, None, None, None, None, 1, 1, 0,
                         128, 64, 1, 0.125, fa.FA_BF16, None, 0, None) == fa.FA_ERR_INVALID


def test_noalloc_scratch_limit_at_its_edge(lib):
    """fa_bwd_noalloc's 32 MiB scratch: at d = 64 a row takes 8 + 256 bytes, so 992
    tiles of 128 rows (126,976 rows) fit and 993 tiles (127,104 rows) do not; the
    larger problem is refused before any pointer is used."""
    limit = 32 << 20
    assert lib.fa_bwd_workspace_size(1, 1, 126976, 64) <= limit
    assert lib.fa_bwd_workspace_size(1, 1, 127104, 64) > limit
    assert lib.fa_bwd_workspace_size(1, 1, 64512, 128) <= limit   # 504 tiles at d = 128
    assert lib.fa_bwd_workspace_size(1, 1, 64640, 128) > limit
    args = [P, P, P, P, None, P, P, P, P, P]
    for B, H, N, d in ((1, 1, 127104, 64), (3, 1, 42368, 64), (1, 1, 64640, 128)):
        assert lib.fa_bwd_noalloc(*args, B, H, N, d, 0, 0.125, fa.FA_BF16, None) == \
            fa.FA_ERR_UNSUPPORTED


def test_register_split_kernels_compiled_with_their_launch_budget():
    """fa_bwd_main_kernel's setmaxnreg split (2 x 128 + 200 + 56 per sub-partition)
    assumes exactly 128 registers per thread at launch; the build fails otherwise, and
    ptxas's report of this build must show it for every instantiation."""
    rep = build.resources()
    mains = {k: v for k, v in rep.items() if "fa_bwd_main_kernel" in k}
    assert len(mains) == 8  # d in {64, 128} x causal x dtype
    assert all(v["registers"] == 128 for v in mains.values()), mains
    with pytest.raises(RuntimeError):
        build.check_resources({"_ZN2fa18fa_bwd_main_kernelILi64E": {"registers": 120,
                                                                   "spill_stores": 0,
                                                                   "spill_loads": 0}})
