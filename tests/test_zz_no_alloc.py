"""GPU test of solattn_forward_noalloc, the entry point for callers that cannot
allocate device memory (plugin interfaces that only hand over input/output buffers
and a stream, code running while the host framework's allocator is locked, processes
with a fixed device-memory budget). It uses the library's static device scratch
instead of a caller workspace.

Two calls in a row must reproduce the workspace entry point's output (same tolerance
as the parity tests: max-abs 1e-2 beyond the bf16 half-ulp, mean relative 2e-3; in
practice the results are identical), and a shape whose scratch exceeds the static
size must be rejected before any device work. Collected last so that a run stopping
at its first failure has already run every other test; it also passes alone in a
fresh process."""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

from block_sparse_online_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _close(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    err = np.abs(a - b)
    half_ulp = 0.5 * np.exp2(np.floor(np.log2(np.maximum(np.abs(b), 2.0 ** -126))) - 7)
    assert (err - half_ulp).max() <= 1e-2
    assert err.sum() <= 2e-3 * np.abs(b).sum()


CASES = [
    ("tiny", None, 64, 64, 2.0, "keep_correct"),
    ("video480", 2, 128, 128, 6.0, "keep_correct"),
    ("video480", 2, 128, 128, 3.0, "keep_drop"),
    ("image", None, 64, 64, 0.0, "dense"),
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}-{c[5]}" for c in CASES])
def test_noalloc_matches_workspace_entry_point_twice(case):
    from block_sparse_online_b200 import solattn
    name, heads, Bq, Bk, tau, mode = case
    cfg = synth.CONFIGS[name]
    if heads:
        cfg = dataclasses.replace(cfg, H=heads)
    if name == "image":
        cfg = dataclasses.replace(cfg, B=1, H=4)
    assert solattn.solattn_workspace_size(*cfg.shape(), Bq, Bk) <= solattn.NOALLOC_SCRATCH_BYTES
    q, k, v = (t.cuda() for t in synth.make_inputs(cfg))
    ref_out, ref_kept, _ = solattn.solattn_forward(q, k, v, Bq, Bk, tau, mode)
    torch.cuda.synchronize()
    for _ in range(2):
        out, kept = solattn.solattn_forward_noalloc(q, k, v, Bq, Bk, tau, mode)
        torch.cuda.synchronize()
        assert torch.equal(kept, ref_kept)
        _close(out, ref_out)


def test_noalloc_rejects_shapes_beyond_the_static_scratch():
    from block_sparse_online_b200 import solattn
    B, H, N, d = 1, 12, 32760, 128  # the 480p shape needs ~105 MB of scratch
    assert solattn.solattn_workspace_size(B, H, N, d, 128, 128) > solattn.NOALLOC_SCRATCH_BYTES
    buf = torch.zeros(1 << 12, dtype=torch.uint8, device="cuda")  # never read: rejected first
    kept = torch.zeros(B * H, dtype=torch.int64, device="cuda")
    st = solattn._Stats(kept.data_ptr(), None)
    p = buf.data_ptr()
    rc = solattn._lib.solattn_forward_noalloc(p, p, p, p, B, H, N, d, 128, 128, ctypes.c_float(2.0), 2,
                                              ctypes.byref(st), None)
    assert rc == solattn.SOLATTN_EWORKSPACE
