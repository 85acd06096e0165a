"""Host-side tests of libsolattn (no GPU needed): the library loads, exports every
symbol include/solattn.h declares, sizes workspaces, and rejects bad arguments
before queueing any device work."""
import ctypes
import os
import re

import pytest
import torch

from block_sparse_online_b200 import solattn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "solattn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(solattn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("solattn_pool", "solattn_forward", "solattn_get_status", "solattn_workspace_size",
                 "solattn_strerror"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(solattn.library_path())
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) == set(solattn.EXPORTS)


def test_debug_library_exports_every_declared_symbol():
    """The bounds-checked build (-DSOLATTN_DEBUG) is the same boundary: it is built here if
    it is missing (nvcc cross-compiles without a GPU) and loaded without one."""
    if not os.path.exists(solattn.DEBUG_LIB_PATH):
        from block_sparse_online_b200 import build
        try:
            build.nvcc()
        except RuntimeError:
            pytest.skip("nvcc not available to build the debug library")
        build.build(debug=True)
    lib = ctypes.CDLL(solattn.DEBUG_LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.solattn_workspace_size(1, 12, 32760, 128, 128, 128) == \
        solattn.solattn_workspace_size(1, 12, 32760, 128, 128, 128)


def test_strerror():
    assert solattn.strerror(0) == "ok"
    assert "timed out" in solattn.strerror(solattn.SOLATTN_ETIMEOUT)
    assert "bounds check" in solattn.strerror(solattn.SOLATTN_EBOUNDS)
    assert solattn.strerror(12345) == "unknown status"


def test_workspace_sizes():
    ws = solattn.solattn_workspace_size
    assert ws(1, 12, 32760, 128, 128, 128) > 12 * 256 * 128 * 4 * 3
    assert ws(1, 1, 100, 96, 128, 128) == 0          # d unsupported
    assert ws(1, 1, 100, 128, 32, 128) == 0          # block size unsupported
    assert ws(1, 1, 0, 128, 128, 128) == 0           # empty
    assert ws(1, 1, 1024 * 128, 128, 128, 128) > 0   # at the key-block limit
    assert ws(1, 1, 1024 * 128 + 1, 128, 128, 128) == 0
    assert solattn.solattn_host_workspace_size(1, 2, 1000, 64, 64, 64) > 4 * 2 * 1000 * 64 * 2


def _call(**kw):
    """solattn_forward with placeholder pointers. Every case passed here carries an
    invalid argument, so the call must return before touching the device. The test
    only runs where no GPU is visible, so a missed check cannot reach a kernel."""
    a = dict(q=4096, k=4096, v=4096, out=4096, B=1, H=1, N=256, d=128, Bq=128, Bk=128, tau=2.0, mode=2,
             kept=4096, mask=None, ws=4096, ws_bytes=1 << 30)
    a.update(kw)
    st = solattn._Stats(a["kept"], a["mask"])
    return solattn._lib.solattn_forward(a["q"], a["k"], a["v"], a["out"], a["B"], a["H"], a["N"], a["d"], a["Bq"],
                                        a["Bk"], ctypes.c_float(a["tau"]), a["mode"], ctypes.byref(st), a["ws"],
                                        a["ws_bytes"], None)


@pytest.mark.skipif(torch.cuda.is_available(), reason="placeholder pointers are used only without a GPU")
@pytest.mark.parametrize("kw,want", [
    (dict(q=None), solattn.SOLATTN_EINVAL),
    (dict(out=None), solattn.SOLATTN_EINVAL),
    (dict(kept=None), solattn.SOLATTN_EINVAL),
    (dict(N=0), solattn.SOLATTN_EINVAL),
    (dict(B=0), solattn.SOLATTN_EINVAL),
    (dict(d=96), solattn.SOLATTN_EUNSUPPORTED),
    (dict(Bq=32), solattn.SOLATTN_EUNSUPPORTED),
    (dict(Bk=256), solattn.SOLATTN_EUNSUPPORTED),
    (dict(N=200000, Bk=128), solattn.SOLATTN_EUNSUPPORTED),
    (dict(mode=3), solattn.SOLATTN_EINVAL),
    (dict(mode=-1), solattn.SOLATTN_EINVAL),
    (dict(tau=-0.5), solattn.SOLATTN_EINVAL),
    (dict(tau=float("nan")), solattn.SOLATTN_EINVAL),
    (dict(q=4100), solattn.SOLATTN_EINVAL),          # not 16-byte aligned
    (dict(kept=4100), solattn.SOLATTN_EINVAL),       # not 8-byte aligned
    (dict(ws=None), solattn.SOLATTN_EWORKSPACE),
    (dict(ws=4096 + 64), solattn.SOLATTN_EWORKSPACE),  # not 256-byte aligned
    (dict(ws_bytes=100), solattn.SOLATTN_EWORKSPACE),
])
def test_forward_rejects_bad_arguments(kw, want):
    assert _call(**kw) == want


@pytest.mark.skipif(torch.cuda.is_available(), reason="placeholder pointers are used only without a GPU")
def test_forward_without_device_reports_cuda_error():
    # Valid arguments on a machine without a GPU: the device query fails cleanly.
    assert _call() in (solattn.SOLATTN_ECUDA, solattn.SOLATTN_EUNSUPPORTED)


def _call_gauss(beta=1.0, variant=0, mode=2, **kw):
    """solattn_forward_gaussian with placeholder pointers (invalid cases only, as _call)."""
    a = dict(q=4096, k=4096, v=4096, out=4096, B=1, H=1, N=256, d=128, Bq=128, Bk=128, kept=4096, mask=None,
             ws=4096, ws_bytes=1 << 30)
    a.update(kw)
    st = solattn._Stats(a["kept"], a["mask"])
    return solattn._lib.solattn_forward_gaussian(a["q"], a["k"], a["v"], a["out"], a["B"], a["H"], a["N"], a["d"],
                                                 a["Bq"], a["Bk"], ctypes.c_float(beta), variant, mode,
                                                 ctypes.byref(st), a["ws"], a["ws_bytes"], None)


@pytest.mark.skipif(torch.cuda.is_available(), reason="placeholder pointers are used only without a GPU")
@pytest.mark.parametrize("kw,want", [
    (dict(beta=float("nan")), solattn.SOLATTN_EINVAL),
    (dict(variant=2), solattn.SOLATTN_EINVAL),
    (dict(variant=-1), solattn.SOLATTN_EINVAL),
    (dict(mode=5), solattn.SOLATTN_EINVAL),
    (dict(q=None), solattn.SOLATTN_EINVAL),
    (dict(d=96), solattn.SOLATTN_EUNSUPPORTED),
    (dict(ws_bytes=100), solattn.SOLATTN_EWORKSPACE),
])
def test_forward_gaussian_rejects_bad_arguments(kw, want):
    assert _call_gauss(**kw) == want


@pytest.mark.skipif(torch.cuda.is_available(), reason="placeholder pointers are used only without a GPU")
def test_forward_gaussian_accepts_infinite_beta_and_negative_beta():
    # +-inf and negative beta are valid; without a GPU the call fails only at the device query.
    for beta in (float("inf"), float("-inf"), -1.5):
        assert _call_gauss(beta=beta) in (solattn.SOLATTN_ECUDA, solattn.SOLATTN_EUNSUPPORTED)


def _call_ex(rule=0, tau=1.0, beta=0.0, n_sink=0, route=True, correction=0, **kw):
    """solattn_forward_ex with placeholder pointers (invalid cases only, as _call)."""
    a = dict(q=4096, k=4096, v=4096, out=4096, B=1, H=1, N=256, d=128, Bq=128, Bk=128, mode=2, kept=4096,
             mask=None, ws=4096, ws_bytes=1 << 30)
    a.update(kw)
    st = solattn._Stats(a["kept"], a["mask"])
    r = solattn._Route(rule, tau, beta, n_sink, correction)
    return solattn._lib.solattn_forward_ex(a["q"], a["k"], a["v"], a["out"], a["B"], a["H"], a["N"], a["d"],
                                           a["Bq"], a["Bk"], ctypes.byref(r) if route else None, a["mode"],
                                           ctypes.byref(st), a["ws"], a["ws_bytes"], None)


@pytest.mark.skipif(torch.cuda.is_available(), reason="placeholder pointers are used only without a GPU")
@pytest.mark.parametrize("kw,want", [
    (dict(route=False), solattn.SOLATTN_EINVAL),
    (dict(rule=3), solattn.SOLATTN_EINVAL),
    (dict(rule=0, tau=-1.0), solattn.SOLATTN_EINVAL),
    (dict(rule=1, beta=float("nan")), solattn.SOLATTN_EINVAL),
    (dict(n_sink=-1), solattn.SOLATTN_EINVAL),
    (dict(n_sink=257), solattn.SOLATTN_EINVAL),   # more sinks than key tokens
    (dict(correction=2), solattn.SOLATTN_EINVAL),
    (dict(q=None), solattn.SOLATTN_EINVAL),
])
def test_forward_ex_rejects_bad_arguments(kw, want):
    assert _call_ex(**kw) == want


@pytest.mark.skipif(torch.cuda.is_available(), reason="placeholder pointers are used only without a GPU")
def test_forward_ex_accepts_valid_routes():
    # Valid options (a negative tau is valid under a Gaussian rule, n_sink = N is valid);
    # without a GPU the call fails only at the device query.
    for kw in (dict(rule=1, tau=-1.0, beta=1.0), dict(rule=2, n_sink=256), dict(rule=0, tau=float("inf")),
               dict(correction=1)):
        assert _call_ex(**kw) in (solattn.SOLATTN_ECUDA, solattn.SOLATTN_EUNSUPPORTED)


@pytest.mark.skipif(torch.cuda.is_available(), reason="placeholder pointers are used only without a GPU")
def test_pool_rejects_bad_arguments():
    f = solattn._lib.solattn_pool
    assert f(None, 4096, 1, 1, 128, 128, 128, None) == solattn.SOLATTN_EINVAL
    assert f(4096, 4096, 1, 1, 128, 96, 128, None) == solattn.SOLATTN_EUNSUPPORTED
    assert f(4104, 4096, 1, 1, 128, 128, 128, None) == solattn.SOLATTN_EINVAL


def test_binding_rejects_cpu_tensors():
    q = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        solattn.solattn_forward(q, q, q, 64, 64, 1.0, "keep_drop")


@pytest.mark.skipif(torch.cuda.is_available(), reason="placeholder pointers are used only without a GPU")
def test_routing_entry_points_reject_bad_arguments():
    L = solattn._lib
    f = ctypes.c_float
    args = (4096, 4096, 1, 2, 1000, 64, 64, 64)
    assert L.solattn_route_keep(None, 4096, *args[2:], f(1.0), 4096, None) == solattn.SOLATTN_EINVAL
    assert L.solattn_route_keep(*args, f(-1.0), 4096, None) == solattn.SOLATTN_EINVAL
    assert L.solattn_route_keep(*args, f(float("nan")), 4096, None) == solattn.SOLATTN_EINVAL
    assert L.solattn_route_keep(4096, 4096, 1, 2, 1000, 96, 64, 64, f(1.0), 4096, None) == solattn.SOLATTN_EUNSUPPORTED
    need = solattn._lib.solattn_proxy_map_bytes(1, 2, 1000, 64, 64)
    assert need == 2 * 16 * 16 * 4
    assert L.solattn_route_topk(*args, 0, 4096, need, 4096, None) == solattn.SOLATTN_EINVAL
    assert L.solattn_route_topk(*args, 3, 4096, need - 4, 4096, None) == solattn.SOLATTN_EWORKSPACE
    for p in (0.0, -0.5, 1.5, float("nan")):
        assert L.solattn_route_topp(*args, f(p), 4096, need, 4096, None) == solattn.SOLATTN_EINVAL
    assert L.solattn_route_topp(*args, f(0.9), None, need, 4096, None) == solattn.SOLATTN_EINVAL
