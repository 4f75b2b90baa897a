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
    return sorted(set(re.findall(r"\b(fa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    assert names == sorted(["fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_get_device_status",
                            "fa_status_string", "fa_version", "fa_bwd_preprocess",
                            "fa_bwd_dkdv", "fa_bwd_dq_convert", "fa_bwd_noalloc",
                            "fa_selftest_wait_timeout", "fa_selftest_exp2", "fa_fwd_qk", "fa_bwd_qk", "fa_fwd_ex",
                            "fa_bwd_ex", "fa_bwd_ex_stage", "fa_bwd_ex_workspace_size",
                            "fa_tile_range", "fa_decode", "fa_decode_workspace_size"])


def test_every_declared_symbol_is_exported(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name
        assert name in fa.SIGNATURES, name


def test_version_and_status_strings(lib):
    assert lib.fa_version() == 2
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
    (dict(d=192), fa.FA_ERR_UNSUPPORTED),
    (dict(d=512), fa.FA_ERR_UNSUPPORTED),
    (dict(d=256, B=0), fa.FA_OK),               # d = 256 passes the shape checks ...
    (dict(d=256, K=P + 8), fa.FA_ERR_INVALID),  # ... and reaches the pointer checks
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
    (dict(d=256), fa.FA_ERR_UNSUPPORTED),  # the backward has no d = 256 kernel
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
    assert len(mains) == 16  # d in {64, 128} x band x dtype x (with dQ, without)
    assert all(v["registers"] == 128 for v in mains.values()), mains
    with pytest.raises(RuntimeError):
        build.check_resources({"_ZN2fa18fa_bwd_main_kernelILi64E": {"registers": 120,
                                                                   "spill_stores": 0,
                                                                   "spill_loads": 0}})


def _visible(Nq, Nk, wl, wr):
    """Brute force: [Nq, Nk] boolean, query i sees key j under the (wl, wr) window."""
    import numpy as np
    i = np.arange(Nq)[:, None]
    j = np.arange(Nk)[None, :]
    off = Nk - Nq
    lo = np.full_like(i, -10 ** 9) if wl < 0 else i + off - wl
    hi = np.full_like(i, 10 ** 9) if wr < 0 else i + off + wr
    return (j >= lo) & (j <= hi)


WINDOWS = [(-1, -1), (-1, 0), (0, 0), (1, 1), (127, 0), (128, 0), (300, 5), (0, 300),
           (-1, 128), (5, -1), (1000, 1000)]


@pytest.mark.parametrize("Nq,Nk", [(128, 128), (300, 300), (1, 700), (700, 1), (333, 1000),
                                   (1000, 333), (256, 1024), (1100, 640)])
def test_tile_ranges_cover_exactly_the_window(lib, Nq, Nk):
    """fa_tile_range (the kernels' tile schedule) against brute force: every tile that
    holds a visible (query, key) pair is visited, and every visited range is tight --
    its first and last tiles hold a visible pair (a query tile's rows past Nq are
    padding and excluded)."""
    import numpy as np
    T = 128
    ntq, ntk = -(-Nq // T), -(-Nk // T)
    for wl, wr in WINDOWS:
        vis = _visible(Nq, Nk, wl, wr)
        pair = np.zeros((ntq, ntk), bool)
        for a in range(ntq):
            for b in range(ntk):
                pair[a, b] = vis[a * T:(a + 1) * T, b * T:(b + 1) * T].any()
        for a in range(ntq):
            first, count = fa.tile_range(True, a, Nq, Nk, (wl, wr))
            want = np.nonzero(pair[a])[0]
            if len(want) == 0:
                assert count == 0, (wl, wr, a)
            else:
                assert (first, count) == (want[0], want[-1] - want[0] + 1), (wl, wr, a)
        for b in range(ntk):
            first, count = fa.tile_range(False, b, Nq, Nk, (wl, wr))
            want = np.nonzero(pair[:, b])[0]
            if len(want) == 0:
                assert count == 0, (wl, wr, b)
            else:
                assert (first, count) == (want[0], want[-1] - want[0] + 1), (wl, wr, b)


def test_tile_range_rejects_bad_arguments(lib):
    first, count = ctypes.c_int(), ctypes.c_int()
    bad = [(1, 2, 256, 256), (0, 2, 256, 256), (1, -1, 256, 256), (1, 0, 0, 256),
           (1, 0, 256, 0), (1, 0, 1 << 29, 1)]
    for side, tile, Nq, Nk in bad:
        assert lib.fa_tile_range(side, tile, Nq, Nk, -1, 0, ctypes.byref(first),
                                 ctypes.byref(count)) == fa.FA_ERR_INVALID
    assert lib.fa_tile_range(1, 0, 256, 256, -1, 0, None, ctypes.byref(count)) == \
        fa.FA_ERR_INVALID


def _fwd_ex(lib, **kw):
    a = dict(Q=P, K=P + 0x100000, V=P + 0x200000, O=P + 0x300000, R=None, L=P + 0x400000, B=1,
             H=1, Nq=256, Nk=256, d=64, layout=0, wl=-1, wr=0, scale=0.125, dtype=fa.FA_BF16)
    a.update(kw)
    return lib.fa_fwd_ex(a["Q"], a["K"], a["V"], a["O"], a["R"], a["L"], a["B"], a["H"], a["Nq"],
                         a["Nk"], a["d"], a["layout"], a["wl"], a["wr"], a["scale"], a["dtype"],
                         None)


def _bwd_ex(lib, stages=7, **kw):
    a = dict(Q=P, K=P + 0x100000, V=P + 0x200000, O=P + 0x300000, R=None, dO=P + 0x400000,
             L=P + 0x500000, dQ=P + 0x600000, dK=P + 0x700000, dV=P + 0x800000, B=1, H=1,
             Nq=256, Nk=256, d=64, layout=0, wl=-1, wr=0, det=0, scale=0.125,
             dtype=fa.FA_BF16, ws=P + 0x900000, ws_bytes=1 << 30)
    a.update(kw)
    return lib.fa_bwd_ex_stage(stages, a["Q"], a["K"], a["V"], a["O"], a["R"], a["dO"], a["L"],
                               a["dQ"], a["dK"], a["dV"], a["B"], a["H"], a["Nq"], a["Nk"],
                               a["d"], a["layout"], a["wl"], a["wr"], a["det"], a["scale"],
                               a["dtype"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(layout=2), fa.FA_ERR_INVALID),
    (dict(layout=-1), fa.FA_ERR_INVALID),
    (dict(Nq=1 << 28, Nk=(1 << 28) + 1, B=1, H=1), fa.FA_ERR_UNSUPPORTED),  # Nq + Nk > 2^29
    (dict(Nk=0), fa.FA_ERR_INVALID),
    (dict(V=P + 0x200008), fa.FA_ERR_INVALID),
    (dict(Nq=0, Q=None, O=None, L=None), fa.FA_OK),
])
def test_fwd_ex_rejects_before_launch(lib, kw, code):
    assert _fwd_ex(lib, **kw) == code


@pytest.mark.parametrize("stages,kw,code", [
    (7, dict(layout=5), fa.FA_ERR_INVALID),
    (0, {}, fa.FA_ERR_INVALID),
    (8, {}, fa.FA_ERR_INVALID),
    (7, dict(ws=None), fa.FA_ERR_INVALID),
    (7, dict(ws_bytes=100), fa.FA_ERR_INVALID),
    (1, dict(O=None), fa.FA_ERR_INVALID),       # the preprocess reads O
    (2, dict(dK=None), fa.FA_ERR_INVALID),      # the dK/dV pass writes dK
    (4, dict(dQ=P + 0x600004), fa.FA_ERR_INVALID),
    (7, dict(d=256), fa.FA_ERR_UNSUPPORTED),
    (7, dict(Nq=0, dK=None), fa.FA_ERR_INVALID),   # no queries: dK = dV = 0 still owed
    (4, dict(Nq=0, dK=None, dV=None), fa.FA_OK),   # ... but only by the dK/dV stage
])
def test_bwd_ex_stage_rejects_before_launch(lib, stages, kw, code):
    assert _bwd_ex(lib, stages, **kw) == code


def test_ex_workspace_size_matches_the_basic_form(lib):
    for B, H, Nq, Nk, d in ((2, 3, 256, 256, 64), (1, 4, 200, 1000, 128), (3, 1, 1, 5, 64)):
        assert lib.fa_bwd_ex_workspace_size(B, H, Nq, Nk, d, 0) == \
            lib.fa_bwd_workspace_size(B, H, Nq, d)
    assert lib.fa_bwd_ex_workspace_size(1, 1, -1, 4, 64, 0) == ctypes.c_size_t(-1).value


def test_decode_workspace_size(lib):
    """One split (no workspace) for short key sequences; otherwise B*H*splits*Nq*(d+1)
    fp32 values, with the splits chosen from B*H and the visible key tiles only."""
    assert lib.fa_decode_workspace_size(1, 1, 1, 128, 128, -1, -1) == 0
    assert lib.fa_decode_workspace_size(4, 32, 16, 64, 128, -1, 0) == 0
    ws = lib.fa_decode_workspace_size(1, 8, 1, 65536, 128, -1, 0)
    assert ws > 0 and ws % (8 * 1 * 129 * 4) == 0
    splits = ws // (8 * 1 * 129 * 4)
    assert 1 < splits <= 512
    # a window that leaves 2 tiles visible needs at most 2 splits
    ws2 = lib.fa_decode_workspace_size(1, 8, 1, 65536, 128, 200, 0)
    assert ws2 <= 8 * 2 * 129 * 4
    assert lib.fa_decode_workspace_size(1, 1, 17, 4096, 64, -1, -1) == 0  # unsupported
    assert lib.fa_decode_workspace_size(-1, 1, 1, 4096, 64, -1, -1) == ctypes.c_size_t(-1).value


def test_decode_rejects_before_launch(lib):
    def call(Nq=1, Nk=4096, d=128, layout=0, ws=P + 0x900000, ws_bytes=1 << 30, O=P + 0x300000,
             dtype=fa.FA_BF16):
        return lib.fa_decode(P, P + 0x100000, P + 0x200000, O, P + 0x400000, 1, 2, Nq, Nk, d,
                             layout, -1, 0, 0.125, dtype, ws, ws_bytes, None)
    assert call(Nq=17) == fa.FA_ERR_UNSUPPORTED
    assert call(d=96) == fa.FA_ERR_UNSUPPORTED
    assert call(layout=3) == fa.FA_ERR_INVALID
    assert call(O=None) == fa.FA_ERR_INVALID
    assert call(Nk=0) == fa.FA_ERR_INVALID
    assert call(Nk=1 << 20, ws=None) == fa.FA_ERR_INVALID        # splits need a workspace
    assert call(Nk=1 << 20, ws_bytes=16) == fa.FA_ERR_INVALID
    assert call(Nk=1 << 20, ws=P + 0x900010) == fa.FA_ERR_INVALID  # 256-byte alignment
    assert call(Nq=0) == fa.FA_OK


# Threads per block of every kernel the library launches.
BLOCK_THREADS = {"fa_fwd_pp_kernel": 384, "fa_bwd_main_kernel": 512, "fa_bwd_dq_pass_kernel": 320,
                 "fa_fwd_d256_kernel": 352, "fa_decode_kernel": 160, "fa_decode_tc_kernel": 192, "fa_decode_merge_kernel": 256,
                 "fa_bwd_pre_kernel": 256, "fa_bwd_dq_kernel": 256,
                 "fa_selftest_wait_kernel": 32, "fa_selftest_exp2_kernel": 256}


def test_every_kernel_fits_the_register_file_at_its_block_size():
    """A block whose warps need more registers than a sub-partition holds (16,384: each
    of the SM's 4 sub-partitions runs every 4th warp) is refused at launch. Check each
    compiled kernel against the block size the library launches it with."""
    rep = build.resources()
    seen = set()
    for name, res in rep.items():
        fam = [k for k in BLOCK_THREADS if k in name]
        assert len(fam) == 1, name
        seen.add(fam[0])
        warps = -(-BLOCK_THREADS[fam[0]] // 32)
        per_sub = -(-warps // 4)
        regs = -(-res["registers"] // 8) * 8  # allocated in units of 8 per thread
        assert regs * 32 * per_sub <= 16384, (name, res["registers"], BLOCK_THREADS[fam[0]])
        assert res["spill_stores"] <= 8, (name, res)
    assert seen == set(BLOCK_THREADS)


def test_selftest_exp2_rejects_bad_arguments(lib):
    assert lib.fa_selftest_exp2(None, None, 0, None) == fa.FA_OK  # nothing to do, no launch
    assert lib.fa_selftest_exp2(None, None, -2, None) == fa.FA_ERR_INVALID
    assert lib.fa_selftest_exp2(None, None, 3, None) == fa.FA_ERR_INVALID
    assert lib.fa_selftest_exp2(None, None, 4, None) == fa.FA_ERR_INVALID
