"""ctypes binding of libsolattn (the C ABI in include/solattn.h).

Argument marshalling only: every step of the operator runs in the library's
CUDA kernels. PyTorch supplies device memory and the current stream. Loading
fails loudly if ``libsolattn.so`` has not been built; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsolattn.so")
# The build with the kernels' device-side bounds checks (python -m block_sparse_online_b200.build
# --debug): same exports, failed checks reported as SOLATTN_EBOUNDS.
DEBUG_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsolattn_debug.so")

SOLATTN_DENSE = 0
SOLATTN_KEEP_DROP = 1
SOLATTN_KEEP_CORRECT = 2
MODES = {"dense": SOLATTN_DENSE, "keep_drop": SOLATTN_KEEP_DROP, "keep_correct": SOLATTN_KEEP_CORRECT}

SOLATTN_OK = 0
SOLATTN_EINVAL = -1
SOLATTN_EUNSUPPORTED = -2
SOLATTN_ECUDA = -3
SOLATTN_ETIMEOUT = -4
SOLATTN_EWORKSPACE = -5
SOLATTN_EBOUNDS = -6
MAX_KEY_BLOCKS = 1024

EXPORTS = ("solattn_workspace_size", "solattn_pool", "solattn_forward", "solattn_forward_events",
           "solattn_get_status",
           "solattn_host_workspace_size", "solattn_forward_host", "solattn_watchdog_selftest",
           "solattn_selftest_exp2", "solattn_forward_noalloc", "solattn_forward_gaussian", "solattn_forward_ex",
           "solattn_route_keep", "solattn_proxy_map_bytes", "solattn_route_topk", "solattn_route_topp",
           "solattn_strerror")
GAUSS_VARIANTS = {"exact": 0, "diag": 1}  # solattn_gauss_variant
RULES = {"running_max": 0, "gauss_exact": 1, "gauss_diag": 2}  # solattn_rule
CORRECTIONS = {"block": 0, "token": 1}  # solattn_correction


class SolAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {strerror(status)} ({status})")
        self.status = status


class _Stats(ctypes.Structure):
    _fields_ = [("kept_per_head", ctypes.c_void_p), ("keep_mask", ctypes.c_void_p)]


class _Route(ctypes.Structure):  # solattn_route
    _fields_ = [("rule", ctypes.c_int), ("tau", ctypes.c_float), ("beta", ctypes.c_float), ("n_sink", ctypes.c_int),
                ("correction", ctypes.c_int)]


def _load(path=_LIB_PATH):
    if not os.path.exists(path):
        raise ImportError(f"{os.path.basename(path)} is not built ({path}); run "
                          "`python -m block_sparse_online_b200.build`" + (" --debug" if path == DEBUG_LIB_PATH else ""))
    lib = ctypes.CDLL(path)
    i, sz, vp, f = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float
    lib.solattn_workspace_size.argtypes = [i, i, i, i, i, i]
    lib.solattn_workspace_size.restype = sz
    lib.solattn_host_workspace_size.argtypes = [i, i, i, i, i, i]
    lib.solattn_host_workspace_size.restype = sz
    lib.solattn_pool.argtypes = [vp, vp, i, i, i, i, i, vp]
    lib.solattn_pool.restype = i
    lib.solattn_forward.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, i, ctypes.POINTER(_Stats), vp, sz, vp]
    lib.solattn_forward.restype = i
    lib.solattn_forward_events.argtypes = lib.solattn_forward.argtypes + [vp, vp]
    lib.solattn_forward_gaussian.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, ctypes.POINTER(_Stats),
                                             vp, sz, vp]
    lib.solattn_forward_gaussian.restype = i
    lib.solattn_forward_ex.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, ctypes.POINTER(_Route), i,
                                       ctypes.POINTER(_Stats), vp, sz, vp]
    lib.solattn_forward_ex.restype = i
    lib.solattn_forward_events.restype = i
    lib.solattn_forward_host.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, vp, sz, vp]
    lib.solattn_forward_host.restype = i
    lib.solattn_get_status.argtypes = [vp, vp]
    lib.solattn_get_status.restype = i
    lib.solattn_watchdog_selftest.argtypes = [vp, sz, ctypes.c_uint64, vp]
    lib.solattn_watchdog_selftest.restype = i
    lib.solattn_forward_noalloc.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, i, ctypes.POINTER(_Stats), vp]
    lib.solattn_forward_noalloc.restype = i
    lib.solattn_selftest_exp2.argtypes = [vp, vp, i, vp]
    lib.solattn_selftest_exp2.restype = i
    lib.solattn_route_keep.argtypes = [vp, vp, i, i, i, i, i, i, f, vp, vp]
    lib.solattn_route_keep.restype = i
    lib.solattn_proxy_map_bytes.argtypes = [i, i, i, i, i]
    lib.solattn_proxy_map_bytes.restype = sz
    lib.solattn_route_topk.argtypes = [vp, vp, i, i, i, i, i, i, i, vp, sz, vp, vp]
    lib.solattn_route_topk.restype = i
    lib.solattn_route_topp.argtypes = [vp, vp, i, i, i, i, i, i, f, vp, sz, vp, vp]
    lib.solattn_route_topp.restype = i
    lib.solattn_strerror.argtypes = [i]
    lib.solattn_strerror.restype = ctypes.c_char_p
    return lib


_lib = _load()
_lib_path = _LIB_PATH


def library_path() -> str:
    return _lib_path


def load_library(path: str = _LIB_PATH) -> str:
    """Route every call of this module through the library at `path` (the release build by
    default, or DEBUG_LIB_PATH); returns the path that was active before."""
    global _lib, _lib_path
    lib = _load(path)
    prev = _lib_path
    _lib, _lib_path = lib, path
    return prev


def strerror(status: int) -> str:
    return _lib.solattn_strerror(int(status)).decode()


def _check(status: int, what: str):
    if status != SOLATTN_OK:
        raise SolAttnError(status, what)


def _stream(stream, device=None):
    """The CUDA stream handle to pass to the library: ``stream``, or the current stream
    of ``device`` (the tensors' device). A stream on another device is refused, since the
    library launches on the current device."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif device is not None and stream.device != torch.device(device):
        raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
    return ctypes.c_void_p(stream.cuda_stream)


def _check_buffer(t, name, dtypes, numel, device):
    """A caller-provided buffer the library writes or reads through a raw pointer: it must
    be contiguous, of an accepted dtype, hold at least ``numel`` elements and live on the
    inputs' device (the library checks none of this; a short or foreign buffer would be
    written out of bounds)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype not in dtypes:
        raise ValueError(f"{name} must have dtype {' or '.join(str(d) for d in dtypes)}, not {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements, {numel} needed")
    if t.device != torch.device(device):
        raise ValueError(f"{name} is on {t.device}, the inputs on {device}")


def _mode(mode) -> int:
    return MODES[mode] if isinstance(mode, str) else int(mode)


def _bhnd(x: torch.Tensor):
    if x.dim() != 4:
        raise ValueError("expected a [B, H, N, d] tensor")
    return tuple(int(s) for s in x.shape)


def solattn_workspace_size(B, H, N, d, Bq, Bk) -> int:
    return int(_lib.solattn_workspace_size(B, H, N, d, Bq, Bk))


def solattn_host_workspace_size(B, H, N, d, Bq, Bk) -> int:
    return int(_lib.solattn_host_workspace_size(B, H, N, d, Bq, Bk))


def alloc_workspace(B, H, N, d, Bq, Bk, device="cuda") -> torch.Tensor:
    n = solattn_workspace_size(B, H, N, d, Bq, Bk)
    if n == 0:
        raise SolAttnError(SOLATTN_EUNSUPPORTED, "solattn_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def solattn_pool(x: torch.Tensor, blk: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Block means of a bf16 [B, H, N, d] CUDA tensor -> fp32 [B, H, ceil(N/blk), d]."""
    B, H, N, d = _bhnd(x)
    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 CUDA tensor")
    nb = -(-N // blk)
    if out is None:
        out = torch.empty((B, H, nb, d), dtype=torch.float32, device=x.device)
    _check_buffer(out, "out", (torch.float32,), B * H * nb * d, x.device)
    with torch.cuda.device(x.device):
        rc = _lib.solattn_pool(x.data_ptr(), out.data_ptr(), B, H, N, d, blk, _stream(stream, x.device))
    _check(rc, "solattn_pool")
    return out


def _inputs(q, k, v):
    B, H, N, d = _bhnd(q)
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != (B, H, N, d):
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors of one shape")
        if t.device != q.device:
            raise ValueError("q, k, v must be on one device")
    return B, H, N, d


def _prepare(q, k, v, Bq, Bk, out, kept_per_head, keep_mask, workspace):
    """Checks the inputs and the buffers the caller passed, and allocates the others."""
    B, H, N, d = _inputs(q, k, v)
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    _check_buffer(out, "out", (torch.bfloat16,), B * H * N * d, dev)
    if kept_per_head is None:
        kept_per_head = torch.empty((B, H), dtype=torch.int64, device=dev)
    _check_buffer(kept_per_head, "kept_per_head", (torch.int64,), B * H, dev)
    mask = None
    nq, nk = -(-N // Bq), -(-N // Bk)
    if isinstance(keep_mask, torch.Tensor):
        mask = keep_mask
        _check_buffer(mask, "keep_mask", (torch.int32, torch.uint32), B * H * nq * (-(-nk // 32)), dev)
    elif keep_mask:
        mask = torch.empty((B, H, nq, -(-nk // 32)), dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = alloc_workspace(B, H, N, d, Bq, Bk, dev)
    _check_buffer(workspace, "workspace", (torch.uint8, torch.int8), 0, dev)
    stats = _Stats(kept_per_head.data_ptr(), mask.data_ptr() if mask is not None else None)
    return B, H, N, d, out, kept_per_head, mask, workspace, stats


def solattn_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, Bq: int, Bk: int, tau: float,
                    mode="keep_correct", out: torch.Tensor | None = None,
                    kept_per_head: torch.Tensor | None = None, keep_mask: bool | torch.Tensor = False,
                    workspace: torch.Tensor | None = None, stream=None, events=None):
    """Run the Sol-Attn forward operator on bf16 [B, H, N, d] CUDA tensors.

    ``events``: optional pair of ``torch.cuda.Event(enable_timing=True)`` recorded
    around the attention kernel (solattn_forward_events).

    Returns (out bf16 [B, H, N, d], kept_per_head int64 [B, H], keep_mask uint32
    [B, H, nQB, ceil(nKB/32)] or None). Asynchronous on ``stream``; device-side
    errors are reported by :func:`solattn_get_status` on the workspace.
    """
    B, H, N, d, out, kept_per_head, mask, workspace, stats = _prepare(q, k, v, Bq, Bk, out, kept_per_head,
                                                                      keep_mask, workspace)
    with torch.cuda.device(q.device):
        args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, H, N, d, Bq, Bk,
                ctypes.c_float(float(tau)), _mode(mode), ctypes.byref(stats), workspace.data_ptr(),
                workspace.numel(), _stream(stream, q.device))
        if events is None:
            rc = _lib.solattn_forward(*args)
        else:
            st = stream if stream is not None else torch.cuda.current_stream(q.device)
            for e in events:
                if e.cuda_event == 0:  # torch creates the CUDA event on its first record
                    e.record(st)
            rc = _lib.solattn_forward_events(*args, ctypes.c_void_p(events[0].cuda_event),
                                             ctypes.c_void_p(events[1].cuda_event))
    _check(rc, "solattn_forward")
    return out, kept_per_head, mask


def solattn_forward_gaussian(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, Bq: int, Bk: int, beta: float,
                             variant="exact", mode="keep_correct", out: torch.Tensor | None = None,
                             kept_per_head: torch.Tensor | None = None, keep_mask: bool | torch.Tensor = False,
                             workspace: torch.Tensor | None = None, stream=None):
    """The forward operator under the query-dependent Gaussian threshold
    (theta_i = mu_i + beta * sigma_i; ``variant`` "exact" or "diag"). Returns what
    :func:`solattn_forward` returns."""
    if variant not in GAUSS_VARIANTS:
        raise ValueError(f"unknown variant {variant!r}")
    B, H, N, d, out, kept_per_head, mask, workspace, stats = _prepare(q, k, v, Bq, Bk, out, kept_per_head,
                                                                      keep_mask, workspace)
    with torch.cuda.device(q.device):
        rc = _lib.solattn_forward_gaussian(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, H, N, d,
                                           Bq, Bk, ctypes.c_float(float(beta)), GAUSS_VARIANTS[variant],
                                           _mode(mode), ctypes.byref(stats), workspace.data_ptr(),
                                           workspace.numel(), _stream(stream, q.device))
    _check(rc, "solattn_forward_gaussian")
    return out, kept_per_head, mask


def solattn_forward_ex(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, Bq: int, Bk: int, mode="keep_correct",
                       rule="running_max", tau: float = 0.0, beta: float = 0.0, n_sink: int = 0,
                       correction="block", out: torch.Tensor | None = None,
                       kept_per_head: torch.Tensor | None = None,
                       keep_mask: bool | torch.Tensor = False, workspace: torch.Tensor | None = None, stream=None):
    """The forward operator with every routing option: ``rule`` "running_max" (tau),
    "gauss_exact" or "gauss_diag" (beta), ``n_sink`` leading key tokens kept as sinks, and
    the keep_correct ``correction``: "block" (block proxy) or "token" (token-to-block logit).
    Returns what :func:`solattn_forward` returns."""
    if rule not in RULES:
        raise ValueError(f"unknown rule {rule!r}")
    if correction not in CORRECTIONS:
        raise ValueError(f"unknown correction {correction!r}")
    B, H, N, d, out, kept_per_head, mask, workspace, stats = _prepare(q, k, v, Bq, Bk, out, kept_per_head,
                                                                      keep_mask, workspace)
    route = _Route(RULES[rule], float(tau), float(beta), int(n_sink), CORRECTIONS[correction])
    with torch.cuda.device(q.device):
        rc = _lib.solattn_forward_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, H, N, d, Bq, Bk,
                                     ctypes.byref(route), _mode(mode), ctypes.byref(stats), workspace.data_ptr(),
                                     workspace.numel(), _stream(stream, q.device))
    _check(rc, "solattn_forward_ex")
    return out, kept_per_head, mask


def solattn_get_status(workspace: torch.Tensor, stream=None) -> int:
    if not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA tensor")
    with torch.cuda.device(workspace.device):
        return int(_lib.solattn_get_status(workspace.data_ptr(), _stream(stream, workspace.device)))


def solattn_forward_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, Bq: int, Bk: int, tau: float,
                         mode="keep_correct", out: torch.Tensor | None = None,
                         kept_per_head: torch.Tensor | None = None, scratch: torch.Tensor | None = None,
                         stream=None):
    """End-to-end call on HOST (ideally pinned) bf16 tensors: host->device copies,
    the operator, and device->host copies of the output and per-head counts, all
    inside the library call, which returns after the stream is synchronised."""
    B, H, N, d = _bhnd(q)
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous() or tuple(t.shape) != (B, H, N, d):
            raise ValueError("q, k, v must be contiguous bf16 host tensors of one shape")
    if out is None:
        out = torch.empty_like(q, pin_memory=True)
    _check_buffer(out, "out", (torch.bfloat16,), B * H * N * d, "cpu")
    if kept_per_head is None:
        kept_per_head = torch.empty((B, H), dtype=torch.int64)
    _check_buffer(kept_per_head, "kept_per_head", (torch.int64,), B * H, "cpu")
    need = solattn_host_workspace_size(B, H, N, d, Bq, Bk)
    if scratch is None:
        scratch = torch.empty(need, dtype=torch.uint8, device="cuda")
    if not scratch.is_cuda:
        raise ValueError("scratch must be a CUDA tensor")
    _check_buffer(scratch, "scratch", (torch.uint8, torch.int8), 0, scratch.device)
    with torch.cuda.device(scratch.device):
        rc = _lib.solattn_forward_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, H, N, d, Bq,
                                       Bk, ctypes.c_float(float(tau)), _mode(mode), kept_per_head.data_ptr(),
                                       scratch.data_ptr(), scratch.numel(), _stream(stream, scratch.device))
    _check(rc, "solattn_forward_host")
    return out, kept_per_head


def solattn_watchdog_selftest(limit_ns: int = 2_000_000, stream=None) -> int:
    """Run the device watchdog self-test; returns the status the kernel stored
    (SOLATTN_ETIMEOUT when a wait that nobody completes is abandoned on time)."""
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with torch.cuda.device(ws.device):
        rc = _lib.solattn_watchdog_selftest(ws.data_ptr(), ws.numel(), int(limit_ns), _stream(stream, ws.device))
    _check(rc, "solattn_watchdog_selftest")
    return solattn_get_status(ws, stream)


NOALLOC_SCRATCH_BYTES = 64 << 20


def solattn_forward_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, Bq: int, Bk: int, tau: float,
                            mode="keep_correct", out: torch.Tensor | None = None,
                            kept_per_head: torch.Tensor | None = None, stream=None):
    """solattn_forward without a workspace: the library uses its static device scratch
    (for callers that cannot allocate device memory). Output and count tensors are
    allocated here only when not given; the library call itself allocates nothing.
    Calls that overlap on the GPU race on the shared scratch."""
    B, H, N, d = _inputs(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    _check_buffer(out, "out", (torch.bfloat16,), B * H * N * d, q.device)
    if kept_per_head is None:
        kept_per_head = torch.empty((B, H), dtype=torch.int64, device=q.device)
    _check_buffer(kept_per_head, "kept_per_head", (torch.int64,), B * H, q.device)
    stats = _Stats(kept_per_head.data_ptr(), None)
    with torch.cuda.device(q.device):
        rc = _lib.solattn_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, H, N, d, Bq,
                                          Bk, ctypes.c_float(float(tau)), _mode(mode), ctypes.byref(stats),
                                          _stream(stream, q.device))
    _check(rc, "solattn_forward_noalloc")
    return out, kept_per_head


def _route_args(qbar: torch.Tensor, kbar: torch.Tensor, N: int, Bq: int, Bk: int, keep_mask):
    if qbar.dim() != 4 or kbar.dim() != 4:
        raise ValueError("qbar and kbar must be [B, H, nB, d]")
    B, H, nQB, d = (int(x) for x in qbar.shape)
    nKB = -(-N // Bk)
    if nQB != -(-N // Bq) or tuple(kbar.shape) != (B, H, nKB, d):
        raise ValueError("qbar / kbar do not match N, Bq, Bk")
    for name, t in (("qbar", qbar), ("kbar", kbar)):
        _check_buffer(t, name, (torch.float32,), t.numel(), qbar.device)
    if keep_mask is None:
        keep_mask = torch.empty((B, H, nQB, -(-nKB // 32)), dtype=torch.int32, device=qbar.device)
    _check_buffer(keep_mask, "keep_mask", (torch.int32, torch.uint32), B * H * nQB * (-(-nKB // 32)), qbar.device)
    return B, H, d, keep_mask


def solattn_route_keep(qbar: torch.Tensor, kbar: torch.Tensor, N: int, Bq: int, Bk: int, tau: float,
                       keep_mask: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The running-maximum routing rule alone on pooled blocks (fp32 [B, H, nB, d]); returns the
    keep bits [B, H, nQB, ceil(nKB/32)] (int32 storage of u32 words)."""
    B, H, d, keep_mask = _route_args(qbar, kbar, N, Bq, Bk, keep_mask)
    with torch.cuda.device(qbar.device):
        rc = _lib.solattn_route_keep(qbar.data_ptr(), kbar.data_ptr(), B, H, N, d, Bq, Bk, ctypes.c_float(float(tau)),
                                     keep_mask.data_ptr(), _stream(stream, qbar.device))
    _check(rc, "solattn_route_keep")
    return keep_mask


def solattn_proxy_map_bytes(B, H, N, Bq, Bk) -> int:
    """Bytes of the fp32 proxy map the top-k and top-p routers write (0 if the shape is invalid)."""
    return int(_lib.solattn_proxy_map_bytes(B, H, N, Bq, Bk))


def _proxy_map(B, H, N, Bq, Bk, proxy_map, device):
    n = solattn_proxy_map_bytes(B, H, N, Bq, Bk)
    if proxy_map is None:
        proxy_map = torch.empty(n // 4, dtype=torch.float32, device=device)
    _check_buffer(proxy_map, "proxy_map", (torch.float32,), n // 4, device)
    return proxy_map


def solattn_route_topk(qbar: torch.Tensor, kbar: torch.Tensor, N: int, Bq: int, Bk: int, k: int,
                       keep_mask: torch.Tensor | None = None, proxy_map: torch.Tensor | None = None, stream=None):
    """Top-k routing (materialised proxy map, the k largest proxies per query block).
    Returns (keep bits, proxy map)."""
    B, H, d, keep_mask = _route_args(qbar, kbar, N, Bq, Bk, keep_mask)
    proxy_map = _proxy_map(B, H, N, Bq, Bk, proxy_map, qbar.device)
    with torch.cuda.device(qbar.device):
        rc = _lib.solattn_route_topk(qbar.data_ptr(), kbar.data_ptr(), B, H, N, d, Bq, Bk, int(k),
                                     proxy_map.data_ptr(), proxy_map.numel() * 4, keep_mask.data_ptr(),
                                     _stream(stream, qbar.device))
    _check(rc, "solattn_route_topk")
    return keep_mask, proxy_map


def solattn_route_topp(qbar: torch.Tensor, kbar: torch.Tensor, N: int, Bq: int, Bk: int, p: float,
                       keep_mask: torch.Tensor | None = None, proxy_map: torch.Tensor | None = None, stream=None):
    """Top-p routing (materialised proxy map; the heaviest blocks until their share of the
    row's mass reaches p). Returns (keep bits, proxy map)."""
    B, H, d, keep_mask = _route_args(qbar, kbar, N, Bq, Bk, keep_mask)
    proxy_map = _proxy_map(B, H, N, Bq, Bk, proxy_map, qbar.device)
    with torch.cuda.device(qbar.device):
        rc = _lib.solattn_route_topp(qbar.data_ptr(), kbar.data_ptr(), B, H, N, d, Bq, Bk, ctypes.c_float(float(p)),
                                     proxy_map.data_ptr(), proxy_map.numel() * 4, keep_mask.data_ptr(),
                                     _stream(stream, qbar.device))
    _check(rc, "solattn_route_topp")
    return keep_mask, proxy_map


def solattn_selftest_exp2(x: torch.Tensor, stream=None) -> torch.Tensor:
    """2^x by the software exp2 of the softmax, for a contiguous fp32 CUDA tensor."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous fp32 CUDA tensor")
    y = torch.empty_like(x)
    with torch.cuda.device(x.device):
        rc = _lib.solattn_selftest_exp2(x.data_ptr(), y.data_ptr(), x.numel(), _stream(stream, x.device))
    _check(rc, "solattn_selftest_exp2")
    return y


__all__ = [n for n in globals() if n.startswith("solattn_")] + ["SolAttnError", "MODES"]
