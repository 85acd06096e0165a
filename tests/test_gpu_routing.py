"""GPU parity of the routing stage on its own (the routing-overhead measurement): Sol-Attn's
running-max rule, and the top-k and top-p routers that materialise the proxy map, each
against the fp64 oracle on pooled blocks of the same bf16 inputs. Keep sets must be equal
except where the decision is within rounding of a tie (the oracle's proxy within 1e-3 of
the running-max threshold; for top-k, the k-th and (k+1)-th ranked proxies within 1e-4;
for top-p, the mass ranked before the boundary within 1e-4 of p times the total)."""
import math

import numpy as np
import pytest
import torch

import oracle.solattn_ref as ref
from block_sparse_online_b200 import synth
from tests.parity_util import unpack_mask

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _pooled(cfg):
    from block_sparse_online_b200 import solattn
    q, k, _ = synth.make_inputs(cfg)
    qd, kd = q.cuda(), k.cuda()
    return q, k, solattn.solattn_pool(qd, cfg.Bq), solattn.solattn_pool(kd, cfg.Bk)


CASES = [
    synth.Config("adhoc", B=1, H=2, d=64, grid=(1, 1, 1000), Bq=64, Bk=64, taus=(), seed=61),
    synth.Config("adhoc", B=2, H=1, d=128, grid=(1, 1, 777), Bq=128, Bk=64, taus=(), seed=62),
    synth.Config("adhoc", B=1, H=3, d=128, grid=(1, 1, 3000), Bq=64, Bk=128, taus=(), seed=63),
]


def _ids(cfgs):
    return [f"{c.B}x{c.H}x{c.N}x{c.d}-{c.Bq}-{c.Bk}" for c in cfgs]


@pytest.mark.parametrize("cfg", CASES + [synth.CONFIGS["tiny"]], ids=_ids(CASES + [synth.CONFIGS["tiny"]]))
def test_route_keep_matches_oracle(cfg):
    from block_sparse_online_b200 import solattn
    q, k, qb, kb = _pooled(cfg)
    for tau in (0.0, 1.0, 3.0):
        mask = solattn.solattn_route_keep(qb, kb, cfg.N, cfg.Bq, cfg.Bk, tau)
        torch.cuda.synchronize()
        got = unpack_mask(mask, cfg.nKB)
        want, margin, _ = ref.keep_sets(q, k, cfg.Bq, cfg.Bk, tau, "keep_drop")
        diff = got != want
        assert not diff.any() or np.abs(margin[diff]).max() < 1e-3, (cfg, tau)


def _topk_ties(sbar, k):
    """Rows where the k-th and (k+1)-th ranked proxies are within 1e-4 (rounding may swap them)."""
    srt = -np.sort(-sbar, axis=-1)
    if k >= sbar.shape[-1]:
        return np.zeros(sbar.shape[:-1], dtype=bool)
    return (srt[..., k - 1] - srt[..., k]) < 1e-4


def _topp_near(sbar, counts, p):
    """Rows where some block's preceding mass lies within 1e-4 (relative) of p * total."""
    out = np.zeros(sbar.shape[:-1], dtype=bool)
    flat = sbar.reshape(-1, sbar.shape[-1])
    o = out.reshape(-1)
    lg = np.log(counts)
    for r in range(flat.shape[0]):
        key = flat[r] + lg
        w = np.exp(np.sort(key)[::-1] - key.max())
        before = np.concatenate([[0.0], np.cumsum(w)[:-1]])
        o[r] = (np.abs(before - p * w.sum()) < 1e-4 * w.sum()).any()
    return out


@pytest.mark.parametrize("cfg", CASES + [synth.CONFIGS["tiny"]], ids=_ids(CASES + [synth.CONFIGS["tiny"]]))
def test_topk_and_topp_match_oracle(cfg):
    from block_sparse_online_b200 import solattn
    q, k, qb, kb = _pooled(cfg)
    sbar = ref.proxy(ref.pool(q, cfg.Bq), ref.pool(k, cfg.Bk))
    counts = ref.valid_counts(cfg.N, cfg.Bk).astype(np.float64)
    for kk in (1, 3, cfg.nKB // 2, cfg.nKB):
        mask, smap = solattn.solattn_route_topk(qb, kb, cfg.N, cfg.Bq, cfg.Bk, kk)
        torch.cuda.synchronize()
        got = unpack_mask(mask, cfg.nKB)
        assert (got.sum(-1) == min(kk, cfg.nKB)).all()
        want = ref.topk_keep(sbar, kk)
        bad = (got != want).any(-1)
        assert not (bad & ~_topk_ties(sbar, kk)).any(), (cfg, kk)
        np.testing.assert_allclose(smap.view(sbar.shape).cpu().double().numpy(), sbar, rtol=1e-5, atol=1e-5)
    for pm in (0.5, 0.9, 0.99, 1.0):
        mask, _ = solattn.solattn_route_topp(qb, kb, cfg.N, cfg.Bq, cfg.Bk, pm)
        torch.cuda.synchronize()
        got = unpack_mask(mask, cfg.nKB)
        want = ref.topp_keep(sbar, counts, pm)
        bad = (got != want).any(-1)
        assert not (bad & ~_topp_near(sbar, counts, pm)).any(), (cfg, pm)
        if pm == 1.0:
            assert got.all()


def test_route_keep_equals_the_forward_kernels_keep_sets():
    """The stand-alone router takes the same decisions as the attention kernel's router."""
    from block_sparse_online_b200 import solattn
    cfg = synth.CONFIGS["video480"]
    q, k, v = (t.cuda() for t in synth.make_inputs(synth.Config("v", B=1, H=2, d=128, grid=(21, 30, 52), Bq=128,
                                                                 Bk=128, taus=(), seed=1002)))
    qb, kb = solattn.solattn_pool(q, 128), solattn.solattn_pool(k, 128)
    for tau in (3.0, 6.0):
        mask = solattn.solattn_route_keep(qb, kb, q.shape[2], 128, 128, tau)
        _, _, fmask = solattn.solattn_forward(q, k, v, 128, 128, tau, "keep_drop", keep_mask=True)
        torch.cuda.synchronize()
        assert torch.equal(mask.cpu(), fmask.cpu())
