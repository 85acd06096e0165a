"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Kept-block sets must match bit for bit except where the oracle's proxy lies
within 1e-3 of the threshold; outputs must stay within max-abs 1e-2 (where the
oracle value is below 2 in magnitude; above it, 1e-2 beyond the half-ulp of the
bf16 result) and L1-relative 2e-3 (bf16 inputs, fp32 accumulation), computed on
the GPU's own keep set. Small cases are checked on every row; the full-size
configurations on a seeded sample of query blocks per head (block 0, the middle
one, the ragged last one and each head's most- and least-kept blocks always
included). Keep sets are compared on every query block.
"""
import math

import numpy as np
import pytest
import torch

import oracle.solattn_ref as ref
from block_sparse_online_b200 import synth
from tests.parity_util import check_case, half_ulp_bf16, run_gpu, sampled_blocks, unpack_mask

pytestmark = pytest.mark.gpu
INF = math.inf
MODES = ("dense", "keep_drop", "keep_correct")


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


# ------------------------------------------------------------ small shapes, all rows

@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("tau", [2.0, 4.0, INF])
def test_tiny_config(mode, tau):
    q, k, v = synth.make_inputs("tiny")
    check_case(q, k, v, 64, 64, tau, mode, label=f"tiny {mode} {tau}")


SHAPES = [
    # (B, H, N, d, Bq, Bk): ragged tails, Bq != Bk, single partial tile, odd tile counts
    (1, 1, 1000, 64, 64, 64),
    (1, 2, 777, 128, 128, 64),
    (2, 1, 777, 128, 64, 128),
    (1, 1, 50, 64, 64, 64),
    (1, 1, 129, 128, 128, 128),
    (1, 3, 640, 128, 128, 128),
    (2, 2, 1300, 64, 128, 128),
    (1, 1, 2000, 128, 64, 64),
]


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
@pytest.mark.parametrize("mode", MODES)
def test_shapes(shape, mode):
    B, H, N, d, Bq, Bk = shape
    cfg = synth.Config("adhoc", B=B, H=H, d=d, grid=(1, 1, N), Bq=Bq, Bk=Bk, taus=(), seed=11 + N)
    q, k, v = synth.make_inputs(cfg)
    for tau in (0.0, 1.5, 3.0):
        check_case(q, k, v, Bq, Bk, tau, mode, label=f"{shape} {mode} {tau}")


def test_random_inputs_extreme_logits():
    # Large logits (std ~ 8) stress the lazy rescaling of the running max.
    q, k, v = synth.make_random(1, 2, 900, 128, seed=3, scale=2.2)
    for mode in MODES:
        check_case(q, k, v, 128, 128, 2.0, mode, label=f"extreme {mode}")


def test_constant_blocks_correction_exact_on_gpu():
    """Constant Q rows per query block and K rows per key block: keep_correct equals dense."""
    g = torch.Generator().manual_seed(5)
    N, d, blk = 1000, 128, 128
    nb = -(-N // blk)
    qb = torch.randn(nb, d, generator=g) * 0.6
    kb = torch.randn(nb, d, generator=g) * 0.6
    q = qb.repeat_interleave(blk, 0)[:N].to(torch.bfloat16)[None, None].contiguous()
    k = kb.repeat_interleave(blk, 0)[:N].to(torch.bfloat16)[None, None].contiguous()
    v = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    dense, _, _ = run_gpu(q, k, v, blk, blk, 0.0, "dense")
    for tau in (0.0, 1.0):
        out, kept, mask = run_gpu(q, k, v, blk, blk, tau, "keep_correct")
        assert unpack_mask(mask, nb).mean() < 1.0
        err = (out.double() - dense.double()).abs()
        tol = 2e-3 + 2 * torch.from_numpy(half_ulp_bf16(dense.double().numpy()))
        assert (err <= tol).all(), err.max().item()


def test_tau_inf_equals_dense_bitwise():
    q, k, v = synth.make_inputs("tiny")
    d_out, d_kept, _ = run_gpu(q, k, v, 64, 64, 0.0, "dense")
    for mode in ("keep_drop", "keep_correct"):
        out, kept, _ = run_gpu(q, k, v, 64, 64, INF, mode)
        assert torch.equal(out, d_out)
        assert torch.equal(kept, d_kept)


def test_deterministic():
    cfg = synth.small_config(N=3000, d=128, Bq=128, Bk=128, H=3)
    q, k, v = synth.make_inputs(cfg)
    a = run_gpu(q, k, v, 128, 128, 3.0, "keep_correct")
    b = run_gpu(q, k, v, 128, 128, 3.0, "keep_correct")
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and torch.equal(a[2].cpu(), b[2].cpu())


def test_pool_matches_oracle():
    from block_sparse_online_b200 import solattn
    q, _, _ = synth.make_random(2, 3, 1111, 128, seed=9)
    for blk in (64, 128):
        got = solattn.solattn_pool(q.cuda(), blk).cpu().double().numpy()
        want = ref.pool(q, blk)
        np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-6)


def test_watchdog_reports_timeout():
    from block_sparse_online_b200 import solattn
    assert solattn.solattn_watchdog_selftest(limit_ns=2_000_000) == solattn.SOLATTN_ETIMEOUT


def test_host_entry_point_matches_device_call():
    from block_sparse_online_b200 import solattn
    q, k, v = synth.make_inputs("tiny")
    dev_out, dev_kept, _ = run_gpu(q, k, v, 64, 64, 2.0, "keep_correct")
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    out, kept = solattn.solattn_forward_host(qh, kh, vh, 64, 64, 2.0, "keep_correct")
    assert torch.equal(out, dev_out)
    assert torch.equal(kept, dev_kept)


HOST_SHAPES = [
    # (B, H, N, d, Bq, Bk, pinned): one head; 17 heads in 9 chunks with a one-head last
    # chunk; 2 x 9 heads in 9 even chunks; 40 heads in 14 chunks; pageable host memory
    (1, 1, 777, 128, 128, 128, True),
    (1, 17, 1000, 128, 128, 64, True),
    (2, 9, 700, 64, 64, 64, True),
    (1, 40, 300, 128, 128, 128, True),
    (1, 5, 900, 128, 128, 128, False),
]


@pytest.mark.parametrize("shape", HOST_SHAPES, ids=[str(s) for s in HOST_SHAPES])
@pytest.mark.parametrize("mode", MODES)
def test_pipelined_host_call_equals_one_device_call(shape, mode):
    """The host entry point runs chunks of heads as a copy/compute pipeline; every
    output element and kept count equals the one device call over all heads."""
    from block_sparse_online_b200 import solattn
    B, H, N, d, Bq, Bk, pinned = shape
    q, k, v = synth.make_random(B, H, N, d, seed=100 + H)
    dev_out, dev_kept, _ = run_gpu(q, k, v, Bq, Bk, 3.0, mode)
    if pinned:
        q, k, v = (t.pin_memory() for t in (q, k, v))
    for _ in range(2):  # the second call reuses the device's copy streams and events
        out, kept = solattn.solattn_forward_host(q, k, v, Bq, Bk, 3.0, mode)
        assert torch.equal(out, dev_out)
        assert torch.equal(kept, dev_kept)


# ------------------------------------------------------------ full-size configurations

def _full(name, taus, modes, per_head):
    cfg = synth.CONFIGS[name]
    q, k, v = synth.make_inputs(cfg)
    blocks = sampled_blocks(cfg.B, cfg.H, cfg.N, cfg.Bq, cfg.Bk, per_head, seed=cfg.seed)
    stats = {}
    for mode in modes:
        for tau in (taus if mode != "dense" else (0.0,)):
            stats[(mode, tau)] = check_case(q, k, v, cfg.Bq, cfg.Bk, tau, mode, qblocks=blocks,
                                            label=f"{name} {mode} {tau}")
    return stats


def test_image_config():
    _full("image", (2.0, 4.0, 6.0, INF), MODES, per_head=4)


def test_video480_config():
    _full("video480", (2.0, 3.0, 4.0, 6.0, INF), MODES, per_head=32)


def test_single_block_items_repeatable():
    """Items that keep one key block leave the second softmax warpgroup without work, and
    the routing-free attention kernel runs them back to back: the largest Gaussian
    threshold (every query block keeps its top block only) and tau = 0 on the 480p shape.
    Repeated calls give identical outputs, and sampled rows match the oracle."""
    import dataclasses
    cfg = dataclasses.replace(synth.CONFIGS["video480"], H=4)
    q, k, v = synth.make_inputs(cfg)
    blocks = sampled_blocks(cfg.B, cfg.H, cfg.N, cfg.Bq, cfg.Bk, 16, seed=cfg.seed + 7)
    cases = [dict(tau=0.0, mode="keep_drop"), dict(tau=0.0, mode="keep_correct"),
             dict(tau=0.0, mode="keep_drop", gauss=(INF, "exact"))]
    for c in cases:
        first = None
        for _ in range(3):
            out, kept, _ = run_gpu(q, k, v, cfg.Bq, cfg.Bk, c["tau"], c["mode"], gauss=c.get("gauss"))
            if first is None:
                first = (out, kept)
            else:
                assert torch.equal(out, first[0]) and torch.equal(kept, first[1]), c
        check_case(q, k, v, cfg.Bq, cfg.Bk, c["tau"], c["mode"], qblocks=blocks, gauss=c.get("gauss"),
                   label=f"single-block items {c}")


@pytest.mark.slow
def test_video720_config():
    _full("video720", (3.0, 4.0, 6.0), MODES, per_head=32)


@pytest.mark.slow
def test_long_config():
    _full("long", (3.0, 4.0, 6.0, INF), MODES, per_head=6)


@pytest.mark.slow
def test_video720_gaussian_and_sinks():
    """The pages' Gaussian threshold (both variants) and sink tokens on the 720p shape, whose
    per-head logit scale varies (so do the per-head thresholds and keep ratios)."""
    cfg = synth.CONFIGS["video720"]
    q, k, v = synth.make_inputs(cfg)
    blocks = sampled_blocks(cfg.B, cfg.H, cfg.N, cfg.Bq, cfg.Bk, 8, seed=cfg.seed + 1)
    for variant in ("exact", "diag"):
        for beta in (0.5, 1.5):
            check_case(q, k, v, cfg.Bq, cfg.Bk, 0.0, "keep_correct", qblocks=blocks, gauss=(beta, variant),
                       label=f"video720 gauss {variant} keep_correct {beta}")
    for mode in ("keep_drop", "keep_correct"):
        check_case(q, k, v, cfg.Bq, cfg.Bk, 4.0, mode, qblocks=blocks, n_sink=256,
                   label=f"video720 sinks 256 {mode} 4.0")


def test_software_exp2_within_bound():
    """The FMA-pipe exp2 of the softmax against fp64 2^x: relative error <= 7.5e-5 + fp32
    rounding on the softmax's input range, and exact powers of two stay exact."""
    from block_sparse_online_b200 import solattn
    x = torch.cat([torch.linspace(-125.0, 8.0, 2_000_001), torch.arange(-125.0, 9.0),
                   torch.rand(1_000_000) * 20 - 16]).contiguous()
    y = solattn.solattn_selftest_exp2(x.cuda()).cpu().double().numpy()
    want = np.exp2(x.double().numpy())
    rel = np.abs(y - want) / want
    assert rel.max() <= 7.6e-5, rel.max()
    ints = torch.arange(-125.0, 9.0).double().numpy()
    yi = solattn.solattn_selftest_exp2(torch.arange(-125.0, 9.0).cuda()).cpu().double().numpy()
    np.testing.assert_allclose(yi, np.exp2(ints), rtol=7.6e-5)
    # far below the clamp the result is a tiny positive number (zero once packed to fp16)
    tiny = solattn.solattn_selftest_exp2(torch.tensor([-200.0, -1e30], device="cuda")).cpu()
    assert (tiny >= 0).all() and (tiny < 1e-37).all()


# ------------------------------------------------------------ query-dependent Gaussian threshold

GAUSS_SHAPES = [
    (1, 2, 1000, 64, 64, 64),
    (1, 2, 777, 128, 128, 64),
    (2, 1, 1300, 128, 64, 128),
    (1, 3, 640, 128, 128, 128),
]


@pytest.mark.parametrize("variant", ("exact", "diag"))
@pytest.mark.parametrize("mode", MODES)
def test_gaussian_tiny(variant, mode):
    q, k, v = synth.make_inputs("tiny")
    for beta in (-INF, 0.0, 0.8, 1.5):
        check_case(q, k, v, 64, 64, 0.0, mode, gauss=(beta, variant), label=f"tiny gauss {variant} {mode} {beta}")


@pytest.mark.parametrize("shape", GAUSS_SHAPES, ids=[str(s) for s in GAUSS_SHAPES])
@pytest.mark.parametrize("variant", ("exact", "diag"))
def test_gaussian_shapes(shape, variant):
    B, H, N, d, Bq, Bk = shape
    cfg = synth.Config("adhoc", B=B, H=H, d=d, grid=(1, 1, N), Bq=Bq, Bk=Bk, taus=(), seed=31 + N)
    q, k, v = synth.make_inputs(cfg)
    for mode in ("keep_drop", "keep_correct"):
        for beta in (0.5, 1.0, 2.5):
            check_case(q, k, v, Bq, Bk, 0.0, mode, gauss=(beta, variant), label=f"{shape} gauss {variant} {mode} {beta}")


def test_gaussian_top_block_only():
    # beta = +inf: every query block keeps exactly its top block.
    q, k, v = synth.make_inputs("tiny")
    stats = check_case(q, k, v, 64, 64, 0.0, "keep_correct", gauss=(INF, "exact"), label="gauss +inf")
    assert stats["flips"] == 0
    out, kept, mask = run_gpu(q, k, v, 64, 64, 0.0, "keep_drop", gauss=(INF, "diag"))
    assert (unpack_mask(mask, 16).sum(axis=-1) == 1).all()


def test_gaussian_video480_config():
    cfg = synth.CONFIGS["video480"]
    q, k, v = synth.make_inputs(cfg)
    blocks = sampled_blocks(cfg.B, cfg.H, cfg.N, cfg.Bq, cfg.Bk, 4, seed=cfg.seed)
    for variant in ("exact", "diag"):
        for mode, beta in (("keep_correct", 1.0), ("keep_drop", 1.5)):
            check_case(q, k, v, cfg.Bq, cfg.Bk, 0.0, mode, qblocks=blocks, gauss=(beta, variant),
                       label=f"video480 gauss {variant} {mode} {beta}")


# ------------------------------------------------------------ sink tokens (solattn_forward_ex)

@pytest.mark.parametrize("rule", ("running_max", "gauss_exact", "gauss_diag"))
def test_sinks(rule):
    gauss = None if rule == "running_max" else (1.5, rule.split("_")[1])
    for shape in ((1, 2, 1000, 64, 64, 64), (1, 2, 777, 128, 128, 64)):
        B, H, N, d, Bq, Bk = shape
        cfg = synth.Config("adhoc", B=B, H=H, d=d, grid=(1, 1, N), Bq=Bq, Bk=Bk, taus=(), seed=41 + N)
        q, k, v = synth.make_inputs(cfg)
        for n_sink in (1, 64, 100, N):
            for mode in ("keep_drop", "keep_correct"):
                stats = check_case(q, k, v, Bq, Bk, 1.0, mode, gauss=gauss, n_sink=n_sink,
                                   label=f"{shape} sinks {rule} {n_sink} {mode}")
                if n_sink == N:
                    assert stats["keep_ratio"] == 1.0


def test_forward_ex_without_sinks_matches_the_other_entry_points():
    from block_sparse_online_b200 import solattn
    q, k, v = (t.cuda() for t in synth.make_inputs("tiny"))
    a = solattn.solattn_forward(q, k, v, 64, 64, 2.0, "keep_correct")
    b = solattn.solattn_forward_ex(q, k, v, 64, 64, "keep_correct", "running_max", tau=2.0)
    c = solattn.solattn_forward_gaussian(q, k, v, 64, 64, 1.0, "diag", "keep_drop")
    e = solattn.solattn_forward_ex(q, k, v, 64, 64, "keep_drop", "gauss_diag", beta=1.0)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert torch.equal(c[0], e[0]) and torch.equal(c[1], e[1])


# ------------------------------------------------------------ token-to-block correction

TOKEN_SHAPES = [
    (1, 2, 1000, 64, 64, 64),
    (1, 2, 777, 128, 128, 64),
    (2, 1, 1300, 128, 64, 128),
    (1, 1, 50, 64, 64, 64),
]


@pytest.mark.parametrize("shape", TOKEN_SHAPES, ids=[str(s) for s in TOKEN_SHAPES])
def test_token_correction_shapes(shape):
    B, H, N, d, Bq, Bk = shape
    cfg = synth.Config("adhoc", B=B, H=H, d=d, grid=(1, 1, N), Bq=Bq, Bk=Bk, taus=(), seed=51 + N)
    q, k, v = synth.make_inputs(cfg)
    for tau in (0.0, 1.5, 3.0):
        check_case(q, k, v, Bq, Bk, tau, "keep_correct", correction="token", label=f"{shape} token {tau}")
    check_case(q, k, v, Bq, Bk, 0.0, "keep_correct", gauss=(1.0, "exact"), n_sink=min(70, N), correction="token",
               label=f"{shape} token gauss sinks")


def test_token_correction_exact_for_block_constant_keys():
    """K constant inside each key block: the token-to-block correction reproduces dense attention."""
    g = torch.Generator().manual_seed(6)
    N, d, blk = 1000, 128, 128
    nb = -(-N // blk)
    kb = torch.randn(nb, d, generator=g) * 0.6
    k = kb.repeat_interleave(blk, 0)[:N].to(torch.bfloat16)[None, None].contiguous()
    q = (torch.randn(1, 1, N, d, generator=g) * 0.8).to(torch.bfloat16)
    v = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    dense, _, _ = run_gpu(q, k, v, blk, blk, 0.0, "dense")
    for tau in (0.0, 0.02):  # the proxies here span about 0.14: these taus drop blocks
        out, kept, mask = run_gpu(q, k, v, blk, blk, tau, "keep_correct", correction="token")
        assert unpack_mask(mask, nb).mean() < 1.0
        err = (out.double() - dense.double()).abs()
        tol = 2e-3 + 2 * torch.from_numpy(half_ulp_bf16(dense.double().numpy()))
        assert (err <= tol).all(), err.max().item()


def test_token_correction_video480_config():
    cfg = synth.CONFIGS["video480"]
    q, k, v = synth.make_inputs(cfg)
    blocks = sampled_blocks(cfg.B, cfg.H, cfg.N, cfg.Bq, cfg.Bk, 4, seed=cfg.seed)
    for tau in (3.0, 6.0):
        check_case(q, k, v, cfg.Bq, cfg.Bk, tau, "keep_correct", qblocks=blocks, correction="token",
                   label=f"video480 token {tau}")
