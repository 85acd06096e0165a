"""The bounds-checked build (libsolattn_debug.so, -DSOLATTN_DEBUG) on the GPU: on valid
inputs of every path (modes, ragged shapes, two query blocks per tile, the token-to-block
correction, the Gaussian threshold, sink tokens, routing alone) no check fires (status 0),
and the checks change no arithmetic: outputs, counts and keep masks equal the release
build's bit for bit."""
import os

import pytest
import torch

from block_sparse_online_b200 import solattn, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _debug_lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if not os.path.exists(solattn.DEBUG_LIB_PATH):
        from block_sparse_online_b200 import build
        build.build(debug=True)
    yield
    solattn.load_library()  # back to the release build


def _run(q, k, v, Bq, Bk, call):
    ws = solattn.alloc_workspace(*q.shape, Bq, Bk)
    out, kept, mask = call(ws)
    st = solattn.solattn_get_status(ws)
    torch.cuda.synchronize()
    return st, out.cpu(), kept.cpu(), mask.cpu()


CASES = [
    # (B, H, N, d, Bq, Bk)
    (1, 2, 1000, 64, 64, 64),
    (1, 2, 777, 128, 128, 64),
    (2, 1, 777, 128, 64, 128),
    (1, 3, 640, 128, 128, 128),
    (1, 2, 32760, 128, 128, 128),
]


@pytest.mark.parametrize("shape", CASES, ids=[str(c) for c in CASES])
def test_debug_build_matches_release(shape):
    B, H, N, d, Bq, Bk = shape
    q, k, v = (t.cuda() for t in synth.make_random(B, H, N, d, seed=5 + N))
    calls = {
        "dense": lambda ws: solattn.solattn_forward(q, k, v, Bq, Bk, 0.0, "dense", keep_mask=True, workspace=ws),
        "keep_drop": lambda ws: solattn.solattn_forward(q, k, v, Bq, Bk, 3.0, "keep_drop", keep_mask=True,
                                                        workspace=ws),
        "keep_correct": lambda ws: solattn.solattn_forward(q, k, v, Bq, Bk, 2.0, "keep_correct", keep_mask=True,
                                                           workspace=ws),
        "token": lambda ws: solattn.solattn_forward_ex(q, k, v, Bq, Bk, "keep_correct", tau=3.0, correction="token",
                                                       keep_mask=True, workspace=ws),
        "sinks": lambda ws: solattn.solattn_forward_ex(q, k, v, Bq, Bk, "keep_drop", tau=2.0, n_sink=200,
                                                       keep_mask=True, workspace=ws),
        "gauss": lambda ws: solattn.solattn_forward_gaussian(q, k, v, Bq, Bk, 1.0, "exact", "keep_correct",
                                                             keep_mask=True, workspace=ws),
    }
    for name, call in calls.items():
        solattn.load_library()
        want = _run(q, k, v, Bq, Bk, call)
        solattn.load_library(solattn.DEBUG_LIB_PATH)
        got = _run(q, k, v, Bq, Bk, call)
        solattn.load_library()
        assert want[0] == 0 and got[0] == 0, (name, want[0], got[0])
        for a, b in zip(want[1:], got[1:]):
            assert torch.equal(a, b), name
    # routing alone (the routing pass without its fold and schedule; no status word)
    qb, kb = solattn.solattn_pool(q, Bq), solattn.solattn_pool(k, Bk)
    masks = []
    for path in (solattn.DEBUG_LIB_PATH, None):
        solattn.load_library(path) if path else solattn.load_library()
        masks.append(solattn.solattn_route_keep(qb, kb, N, Bq, Bk, 3.0).cpu())
    assert torch.equal(masks[0], masks[1])
