"""Pins of the fp64 oracle to things other than itself.

Each pin checks the oracle against a closed form, a library routine, a
hand-worked case or a brute-force loop, so that a plausible mistake anywhere in
the oracle (a dropped term, a wrong scale, sign, index or order) fails at least
one of them. ``test_planted_mistakes_are_caught`` plants such mistakes in the
oracle (on the CPU) and checks that the pins catch every one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle.solattn_ref as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "handworked_d4.json")


def _rand(B, H, N, d, seed, scale=1.0):
    """Q/K with a component shared by runs of 16 tokens (so block means spread and some
    blocks fall below the threshold) plus per-token noise; V standard normal."""
    rng = np.random.default_rng(seed)

    def qk():
        runs = rng.standard_normal((B, H, -(-N // 16), d)) * scale
        return np.repeat(runs, 16, axis=2)[:, :, :N] + 0.5 * rng.standard_normal((B, H, N, d))

    q, k = qk(), qk()
    v = rng.standard_normal((B, H, N, d))
    return q, k, v


def _sdpa(q, k, v, mask=None):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))
    out = torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=None if mask is None else t(mask))
    return out.numpy()


def _token_mask(keep, N, Bq, Bk):
    """[.., N, N] bool: query token r may see key token c iff its blocks are kept."""
    rb = np.arange(N) // Bq
    cb = np.arange(N) // Bk
    return keep[..., rb, :][..., :, cb]


# ------------------------------------------------------------------ pins

def pin_handworked():
    g = json.load(open(GOLDEN))
    env = {"ln4": math.log(4.0), "ln2": math.log(2.0), "sqrt2": math.sqrt(2.0)}
    ev = lambda x: float(eval(str(x), {"__builtins__": {}}, env))  # closed forms only
    q = np.array([[ev(x) for x in r] for r in g["q"]])[None, None]
    k = np.array([[ev(x) for x in r] for r in g["k"]])[None, None]
    v = np.array([[ev(x) for x in r] for r in g["v"]])[None, None]
    for case in g["cases"]:
        out, keep = ref.forward(q, k, v, g["Bq"], g["Bk"], case["tau"], case["mode"],
                                order=case["order"])
        if case["mode"] != "dense":
            assert np.array_equal(keep[0, 0].astype(int), np.array(case["keep"])), case
        for row, vals in case["rows"].items():
            np.testing.assert_allclose(out[0, 0, int(row)], [ev(x) for x in vals],
                                       rtol=1e-13, atol=1e-13, err_msg=str(case))


def pin_pool_is_block_mean():
    x = np.random.default_rng(1).standard_normal((2, 3, 203, 8))
    for blk in (16, 64):
        p = ref.pool(x, blk)
        assert p.shape == (2, 3, -(-203 // blk), 8)
        for j in range(p.shape[2]):
            np.testing.assert_allclose(p[:, :, j], np.mean(x[:, :, j * blk:(j + 1) * blk], axis=2),
                                       rtol=1e-14, atol=1e-14)


def pin_dense_is_softmax_attention():
    q, k, v = _rand(1, 2, 200, 16, seed=2, scale=1.5)
    want = _sdpa(q, k, v)
    for mode, tau in (("dense", 0.5), ("keep_drop", math.inf), ("keep_correct", math.inf)):
        out, _ = ref.forward(q, k, v, 32, 48, tau, mode)
        np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-12, err_msg=mode)


def pin_keep_drop_is_masked_attention():
    q, k, v = _rand(1, 2, 190, 16, seed=3, scale=1.5)
    for Bq, Bk, tau in ((32, 32, 1.0), (32, 64, 2.0), (64, 32, 0.5)):
        out, keep = ref.forward(q, k, v, Bq, Bk, tau, "keep_drop")
        assert not keep.all()
        mask = _token_mask(keep, 190, Bq, Bk)
        np.testing.assert_allclose(out, _sdpa(q, k, v, mask), rtol=1e-12, atol=1e-12)


def pin_keep_correct_is_augmented_attention():
    """keep_correct == softmax attention over the kept keys plus one pseudo-key per
    dropped block (zero key vector, additive bias s_ij + ln n_j, value = block mean of V)."""
    N, d = 170, 16
    q, k, v = _rand(1, 1, N, d, seed=4, scale=1.5)
    for Bq, Bk, tau in ((32, 32, 1.0), (64, 32, 0.3)):
        out, keep = ref.forward(q, k, v, Bq, Bk, tau, "keep_correct")
        assert not keep.all()
        nQB, nKB = keep.shape[-2:]
        qb = np.mean  # pooled means via numpy directly (library routine)
        qbar = np.stack([qb(q[0, 0, i * Bq:(i + 1) * Bq], axis=0) for i in range(nQB)])
        kbar = np.stack([qb(k[0, 0, j * Bk:(j + 1) * Bk], axis=0) for j in range(nKB)])
        vbar = np.stack([qb(v[0, 0, j * Bk:(j + 1) * Bk], axis=0) for j in range(nKB)])
        counts = np.array([min(N, (j + 1) * Bk) - j * Bk for j in range(nKB)])
        sbar = np.einsum("id,jd->ij", qbar, kbar) / math.sqrt(d)
        keys = np.concatenate([k[0, 0], np.zeros((nKB, d))])
        vals = np.concatenate([v[0, 0], vbar])
        bias = np.full((N, N + nKB), -np.inf)
        rb, cb = np.arange(N) // Bq, np.arange(N) // Bk
        kp = keep[0, 0]
        bias[:, :N] = np.where(kp[rb][:, cb], 0.0, -np.inf)
        bias[:, N:] = np.where(kp[rb], -np.inf, sbar[rb] + np.log(counts)[None, :])
        want = _sdpa(q[0, 0][None], keys[None], vals[None], bias[None])[0]
        np.testing.assert_allclose(out[0, 0], want, rtol=1e-12, atol=1e-12)


def pin_constant_blocks_correction_exact():
    """Zero centred score spread (constant Q rows per query block, constant K rows per
    key block) makes the zeroth-order correction exact: keep_correct == dense for every tau
    (paperlayer summary, App. B: the error vanishes with the score spread)."""
    rng = np.random.default_rng(5)
    N, d = 150, 8
    for Bq, Bk in ((32, 32), (32, 64), (64, 32)):
        nQB, nKB = -(-N // Bq), -(-N // Bk)
        q = np.repeat(rng.standard_normal((nQB, d)) * 2.0, Bq, axis=0)[:N][None, None]
        k = np.repeat(rng.standard_normal((nKB, d)) * 2.0, Bk, axis=0)[:N][None, None]
        v = rng.standard_normal((1, 1, N, d))
        dense, _ = ref.forward(q, k, v, Bq, Bk, 0.0, "dense")
        for tau in (0.0, 0.5, 2.0, math.inf):
            out, keep = ref.forward(q, k, v, Bq, Bk, tau, "keep_correct")
            np.testing.assert_allclose(out, dense, rtol=1e-12, atol=1e-12)
        assert not ref.keep_sets(q, k, Bq, Bk, 0.5)[0].all()


def pin_constant_v_is_reproduced():
    q, k, _ = _rand(1, 2, 130, 8, seed=6, scale=2.0)
    v = np.broadcast_to(np.array([1.5, -2.0, 0.25, 3.0, 0.0, 1.0, -1.0, 7.0]), q.shape).copy()
    for mode in ("dense", "keep_drop", "keep_correct"):
        out, _ = ref.forward(q, k, v, 32, 32, 0.5, mode)
        np.testing.assert_allclose(out, v, rtol=1e-13, atol=1e-13)


def pin_tau_zero_keeps_records():
    """tau = 0 keeps exactly the record positions of the visit sequence: position t is
    kept iff its proxy is >= every earlier proxy (ties included; brute force pairwise)."""
    rng = np.random.default_rng(7)
    N, d, Bq, Bk = 320, 8, 32, 32
    q = rng.standard_normal((1, 1, N, d))
    palette = rng.integers(-2, 3, size=(3, d)).astype(float)  # 3 distinct pooled keys
    k = np.repeat(palette[rng.integers(0, 3, size=N // Bk)], Bk, axis=0)[None, None]
    keep, _, sbar = ref.keep_sets(q, k, Bq, Bk, 0.0)
    nQB, nKB = keep.shape[-2:]
    for i in range(nQB):
        j0 = min(i * Bq // Bk, nKB - 1)
        seq = [(j0 + t) % nKB for t in range(nKB)]
        for t, j in enumerate(seq):
            record = all(sbar[0, 0, i, j] >= sbar[0, 0, i, jp] for jp in seq[:t])
            assert keep[0, 0, i, j] == record, (i, t)
    # exact ties occur in this input (repeated pooled keys), and some are kept
    assert all(len(set(sbar[0, 0, i].tolist())) <= 3 for i in range(nQB))
    assert keep.sum() > nQB


def pin_keep_set_structure():
    q, k, _ = _rand(2, 2, 260, 16, seed=8, scale=2.0)
    prev = None
    for tau in (0.0, 0.5, 1.0, 2.0, 4.0, math.inf):
        keep, margin, _ = ref.keep_sets(q, k, 32, 64, tau)
        nQB, nKB = keep.shape[-2:]
        for i in range(nQB):
            assert keep[:, :, i, min(i * 32 // 64, nKB - 1)].all()  # first visit kept
        if prev is not None:
            assert (keep | ~prev).all()  # monotone: kept at smaller tau => kept
        if tau == math.inf:
            assert keep.all()
        else:
            assert np.array_equal(keep, margin >= 0)
        prev = keep


def pin_visit_order():
    for N, Bq, Bk in ((1000, 64, 64), (1000, 128, 64), (1000, 64, 128), (130, 64, 128)):
        nQB, nKB = -(-N // Bq), -(-N // Bk)
        for i in range(nQB):
            vo = ref.visit_order(i, nKB, Bq, Bk)
            assert sorted(vo.tolist()) == list(range(nKB))
            first_tok = i * Bq
            assert vo[0] == min(first_tok // Bk, nKB - 1)  # block holding the first token
            assert all((vo[t + 1] - vo[t]) % nKB == 1 for t in range(nKB - 1))


def _brute_force(q, k, v, Bq, Bk, tau, mode):
    """Pure-Python scalar loops over one head: the definition written out."""
    N, d = len(q), len(q[0])
    nQB, nKB = -(-N // Bq), -(-N // Bk)

    def mean(rows):
        return [sum(r[c] for r in rows) / len(rows) for c in range(d)]

    qb = [mean(q[i * Bq:(i + 1) * Bq]) for i in range(nQB)]
    kb = [mean(k[j * Bk:(j + 1) * Bk]) for j in range(nKB)]
    vb = [mean(v[j * Bk:(j + 1) * Bk]) for j in range(nKB)]
    out = []
    for r in range(N):
        i = r // Bq
        keep = [True] * nKB
        if mode != "dense":
            j0 = min(i * Bq // Bk, nKB - 1)
            best = -math.inf
            for t in range(nKB):
                j = (j0 + t) % nKB
                s = sum(qb[i][c] * kb[j][c] for c in range(d)) / math.sqrt(d)
                best = max(best, s)
                keep[j] = s >= best - tau
        num = [0.0] * d
        den = 0.0
        for j in range(nKB):
            if keep[j]:
                for col in range(j * Bk, min(N, (j + 1) * Bk)):
                    w = math.exp(sum(q[r][c] * k[col][c] for c in range(d)) / math.sqrt(d))
                    den += w
                    num = [num[c] + w * v[col][c] for c in range(d)]
            elif mode == "keep_correct":
                nj = min(N, (j + 1) * Bk) - j * Bk
                s = sum(qb[i][c] * kb[j][c] for c in range(d)) / math.sqrt(d)
                w = nj * math.exp(s)
                den += w
                num = [num[c] + w * vb[j][c] for c in range(d)]
        out.append([x / den for x in num])
    return out


def pin_brute_force_tiny():
    q, k, v = _rand(1, 1, 75, 4, seed=9, scale=1.2)
    for Bq, Bk, tau in ((16, 16, 0.4), (16, 32, 0.2), (32, 16, 1.0)):
        for mode in ("dense", "keep_drop", "keep_correct"):
            out, _ = ref.forward(q, k, v, Bq, Bk, tau, mode)
            want = _brute_force(q[0, 0].tolist(), k[0, 0].tolist(), v[0, 0].tolist(),
                                Bq, Bk, tau, mode)
            np.testing.assert_allclose(out[0, 0], np.array(want), rtol=1e-11, atol=1e-12,
                                       err_msg=f"{mode} {Bq} {Bk} {tau}")


PINS = [pin_handworked, pin_pool_is_block_mean, pin_dense_is_softmax_attention,
        pin_keep_drop_is_masked_attention, pin_keep_correct_is_augmented_attention,
        pin_constant_blocks_correction_exact, pin_constant_v_is_reproduced,
        pin_tau_zero_keeps_records, pin_keep_set_structure, pin_visit_order,
        pin_brute_force_tiny]


# ------------------------------------------------- query-dependent Gaussian threshold

def _block_constant_keys(kbar_rows, blk):
    """K whose blocks of blk tokens are constant rows (so the pooled keys are those rows)."""
    return np.repeat(kbar_rows, blk, axis=-2)


def pin_gaussian_matches_row_statistics():
    # The exact variant's mu_i and sigma_i are the mean and (1/nKB) standard deviation of
    # query block i's proxy row, whatever the keys: computed here from the row directly.
    q, k, _ = _rand(1, 2, 1000, 32, seed=21, scale=1.3)
    sbar = ref.proxy(ref.pool(q, 64), ref.pool(k, 64))
    for beta in (-0.7, 0.0, 1.0, 2.5):
        theta = ref.gaussian_threshold(ref.pool(q, 64), ref.pool(k, 64), beta, "exact")
        want = sbar.mean(axis=-1) + beta * sbar.std(axis=-1)
        np.testing.assert_allclose(theta, want, rtol=1e-11, atol=1e-11)


def pin_gaussian_diagonal_design():
    # Pooled keys k_j = a * h_j with h_j the rows of columns 1..d of a 2d x 2d Sylvester
    # Hadamard matrix: the columns are orthogonal and zero-mean, so the mean is 0 and
    # Cov[K] = diag(a^2) exactly. Then sigma_i^2 = sum_e q_ie^2 a_e^2 / d for both variants.
    d, blk = 16, 4
    H = np.array([[1.0]])
    while H.shape[0] < 2 * d:
        H = np.block([[H, H], [H, -H]])
    rng = np.random.default_rng(5)
    a = rng.uniform(0.5, 2.0, d)
    krows = H[:, 1:d + 1] * a  # [2d, d]
    k = _block_constant_keys(krows, blk)[None, None]
    q = rng.standard_normal((1, 1, k.shape[2], d))
    qbar = ref.pool(q, blk)
    want = np.sqrt((qbar ** 2 * a ** 2).sum(axis=-1) / d)
    for variant in ("exact", "diag"):
        theta = ref.gaussian_threshold(qbar, ref.pool(k, blk), 1.0, variant)
        np.testing.assert_allclose(theta, want, rtol=1e-12, atol=1e-12)


def pin_gaussian_keep_fraction():
    # i.i.d. Gaussian pooled keys: each proxy row is (close to) normal with the row's own
    # mean and std, so the kept fraction approaches 1 - Phi(beta).
    d, blk, nkb = 32, 2, 2048
    rng = np.random.default_rng(8)
    k = _block_constant_keys(rng.standard_normal((nkb, d)), blk)[None, None]
    q = rng.standard_normal((1, 1, 64 * blk, d)) + 0.3
    for beta, frac in ((0.0, 0.5), (1.0, 0.158655), (2.0, 0.022750)):
        keep, _, _ = ref.keep_sets_gaussian(q, k, blk, blk, beta, "exact")
        assert abs(keep.mean() - frac) < 0.02 + 0.1 * frac, (beta, keep.mean())


def pin_gaussian_limits_and_monotone():
    q, k, _ = _rand(1, 2, 777, 16, seed=4)
    sbar = ref.proxy(ref.pool(q, 64), ref.pool(k, 64))
    keep, _, _ = ref.keep_sets_gaussian(q, k, 64, 64, -math.inf, "exact")
    assert keep.all()
    keep, _, _ = ref.keep_sets_gaussian(q, k, 64, 64, 1e9, "diag")
    assert (keep.sum(axis=-1) == 1).all()
    assert (np.argmax(keep, axis=-1) == np.argmax(sbar, axis=-1)).all()
    prev = None
    for beta in (-1.0, 0.0, 0.5, 1.0, 2.0):
        cur, _, _ = ref.keep_sets_gaussian(q, k, 64, 64, beta, "exact")
        assert (cur.sum(axis=-1) >= 1).all()
        if prev is not None:
            assert not (cur & ~prev).any()  # a larger beta keeps a subset
        prev = cur
    # correlated keys: the diagonal estimator differs from the exact one
    kc = k.copy()
    kc[..., 1] = kc[..., 0] * 0.9 + 0.1 * kc[..., 1]
    t_ex = ref.gaussian_threshold(ref.pool(q, 64), ref.pool(kc, 64), 1.0, "exact")
    t_dg = ref.gaussian_threshold(ref.pool(q, 64), ref.pool(kc, 64), 1.0, "diag")
    assert np.abs(t_ex - t_dg).max() > 1e-3


def pin_sinks():
    # Sinks add exactly the leading ceil(n_sink / Bk) key blocks to every keep set and
    # change nothing else (their proxies already entered the running max).
    q, k, v = _rand(1, 2, 777, 16, seed=12)
    base, _, sbar = ref.keep_sets(q, k, 64, 64, 1.0, "keep_drop")
    for n_sink, nb in ((1, 1), (64, 1), (65, 2), (200, 4)):
        got, margin, _ = ref.keep_sets(q, k, 64, 64, 1.0, "keep_drop", n_sink=n_sink)
        assert got[..., :nb].all() and np.isinf(margin[..., :nb]).all()
        np.testing.assert_array_equal(got[..., nb:], base[..., nb:])
        g2, _, _ = ref.keep_sets_gaussian(q, k, 64, 64, 3.0, "exact", n_sink=n_sink)
        assert g2[..., :nb].all()
    # every key token a sink: keep_drop is dense attention, by SDPA
    out, _ = ref.forward(q, k, v, 64, 64, 1.0, "keep_drop", n_sink=777)
    np.testing.assert_allclose(out, _sdpa(q, k, v), rtol=1e-9, atol=1e-9)
    # a Gaussian row with sinks but nothing over its threshold keeps only the sinks
    g3, _, _ = ref.keep_sets_gaussian(q, k, 64, 64, 1e9, "diag", n_sink=10)
    assert (g3.sum(axis=-1) == 1).all() and g3[..., 0].all()


def pin_token_correction():
    N, d, blk = 700, 16, 64
    rng = np.random.default_rng(17)
    nb = -(-N // blk)
    # (1) K constant inside each key block: the token-to-block pseudo-key reproduces every
    # dropped block exactly, so keep_correct equals dense attention for any tau.
    kb = rng.standard_normal((1, 2, nb, d)) * 0.8
    k = np.repeat(kb, blk, axis=2)[:, :, :N]
    q = rng.standard_normal((1, 2, N, d))
    v = rng.standard_normal((1, 2, N, d))
    dense = _sdpa(q, k, v)
    for tau in (0.0, 0.05, 0.15):  # the proxies here span about 0.4: these taus drop blocks
        out, keep = ref.forward(q, k, v, blk, blk, tau, "keep_correct", correction="token")
        assert (~keep).any()
        np.testing.assert_allclose(out, dense, rtol=1e-9, atol=1e-10)
    # (2) Q constant inside each query block: token and block corrections coincide.
    qb = rng.standard_normal((1, 2, nb, d))
    qc = np.repeat(qb, blk, axis=2)[:, :, :N]
    kr = rng.standard_normal((1, 2, N, d))
    a, _ = ref.forward(qc, kr, v, blk, blk, 1.0, "keep_correct", correction="token")
    b, _ = ref.forward(qc, kr, v, blk, blk, 1.0, "keep_correct", correction="block")
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)
    # (3) SDPA over the kept keys plus the dropped blocks' pooled keys, biased by log n_j.
    q, k, v = _rand(1, 1, 300, 8, seed=23)
    out, keep = ref.forward(q, k, v, 64, 64, 1.0, "keep_correct", correction="token")
    kbar, vbar = ref.pool(k, 64), ref.pool(v, 64)
    counts = ref.valid_counts(300, 64)
    for i in range(keep.shape[2]):
        rows = slice(i * 64, min(300, i * 64 + 64))
        cols = keep[0, 0, i][np.arange(300) // 64]
        drop = np.nonzero(~keep[0, 0, i])[0]
        kk = np.concatenate([k[0, 0, cols], kbar[0, 0, drop]])
        vv = np.concatenate([v[0, 0, cols], vbar[0, 0, drop]])
        bias = np.concatenate([np.zeros(cols.sum()), np.log(counts[drop])])
        want = _sdpa(q[:, :, rows], kk[None, None], vv[None, None], np.broadcast_to(bias, (1, 1, rows.stop - rows.start, kk.shape[0])).copy())
        np.testing.assert_allclose(out[:, :, rows], want, rtol=1e-9, atol=1e-10)


def pin_kept_per_head():
    """Per-head kept-block counts (the statistic the operator returns): the hand-worked case
    keeps blocks {0} for query block 0 and {0, 1} for query block 1 at tau = 1, i.e. 3 for its
    only head; on a ragged multi-head case the count equals a scalar loop over the keep
    decisions taken one (b, h, i, j) at a time from the proxies and the visit order."""
    g = json.load(open(GOLDEN))
    env = {"ln4": math.log(4.0), "ln2": math.log(2.0), "sqrt2": math.sqrt(2.0)}
    ev = lambda x: float(eval(str(x), {"__builtins__": {}}, env))  # closed forms only
    q = np.array([[ev(x) for x in r] for r in g["q"]])[None, None]
    k = np.array([[ev(x) for x in r] for r in g["k"]])[None, None]
    keep, _, _ = ref.keep_sets(q, k, g["Bq"], g["Bk"], 1.0, "keep_drop")
    counts = ref.kept_per_head(keep)
    assert counts.shape == (1, 1) and counts.dtype == np.int64 and int(counts[0, 0]) == 3
    B, H, N, d, Bq, Bk, tau = 2, 3, 205, 8, 32, 16, 0.7
    q, k, _ = _rand(B, H, N, d, seed=21)
    keep, _, sbar = ref.keep_sets(q, k, Bq, Bk, tau, "keep_correct")
    nQB, nKB = -(-N // Bq), -(-N // Bk)
    want = np.zeros((B, H), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            for i in range(nQB):
                j0 = min(i * Bq // Bk, nKB - 1)
                m = -math.inf
                for t in range(nKB):
                    j = (j0 + t) % nKB
                    m = max(m, sbar[b, h, i, j])
                    want[b, h] += int(sbar[b, h, i, j] >= m - tau)
    got = ref.kept_per_head(keep)
    assert got.shape == (B, H) and np.array_equal(got, want), (got, want)
    # dense mode keeps every pair
    dense, _, _ = ref.keep_sets(q, k, Bq, Bk, tau, "dense")
    assert np.array_equal(ref.kept_per_head(dense), np.full((B, H), nQB * nKB))


def pin_topk():
    """Top-k: a hand-worked row with a tie (lower index wins), and on random rows exactly
    min(k, nKB) blocks kept, none of them below a dropped one."""
    s = np.array([[3.0, 1.0, 3.0, 2.0]])
    assert ref.topk_keep(s, 2).tolist() == [[True, False, True, False]]
    assert ref.topk_keep(s, 1).tolist() == [[True, False, False, False]]
    assert ref.topk_keep(s, 3).tolist() == [[True, False, True, True]]
    assert ref.topk_keep(s, 9).all()
    rng = np.random.default_rng(23)
    s = rng.standard_normal((3, 7, 29))
    for k in (1, 5, 29):
        keep = ref.topk_keep(s, k)
        assert (keep.sum(-1) == k).all()
        lo = np.where(keep, s, np.inf).min(-1)
        hi = np.where(keep, -np.inf, s).max(-1)
        assert (lo >= hi).all()


def pin_topp():
    """Top-p: a hand-worked row (block sizes 2, 2, 2, 1; proxies ln 4, 0, ln 2, ln 8; masses
    n_j e^s = 8, 2, 4, 8 of 22; rank 0, 3, 2, 1) and, on random rows, kept mass >= p of the
    total while the kept set without its lightest block stays below."""
    s = np.array([[math.log(4.0), 0.0, math.log(2.0), math.log(8.0)]])
    n = np.array([2.0, 2.0, 2.0, 1.0])
    assert ref.topp_keep(s, n, 0.5).tolist() == [[True, False, False, True]]     # 0 + 8 < 11 <= 16
    assert ref.topp_keep(s, n, 0.75).tolist() == [[True, False, True, True]]     # 16 < 16.5
    assert ref.topp_keep(s, n, 16.0 / 22.0).tolist() == [[True, False, False, True]]  # exactly 16: not below
    assert ref.topp_keep(s, n, 1.0).all()
    assert ref.topp_keep(s, n, 1e-9).tolist() == [[True, False, False, False]]   # the heaviest (tie: lower index)
    rng = np.random.default_rng(29)
    s = rng.standard_normal((2, 5, 33)) * 2.0
    n = np.full(33, 64.0)
    n[-1] = 17.0
    for p in (0.3, 0.8, 0.95):
        keep = ref.topp_keep(s, n, p)
        w = n * np.exp(s)
        kept = np.where(keep, w, 0.0).sum(-1)
        assert (kept >= p * w.sum(-1) - 1e-12).all()
        lightest = np.where(keep, w, np.inf).min(-1)
        assert (kept - lightest < p * w.sum(-1)).all()
        hi_drop = np.where(keep, -np.inf, w).max(-1)
        assert (lightest >= hi_drop).all()


PINS += [pin_gaussian_matches_row_statistics, pin_gaussian_diagonal_design, pin_gaussian_keep_fraction,
         pin_gaussian_limits_and_monotone, pin_sinks, pin_token_correction, pin_kept_per_head, pin_topk, pin_topp]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


# -------------------------------------------------------- planted mistakes

def _mut_pool_by_blk(x, blk):
    x = ref.as_f64(x)
    N = x.shape[-2]
    out = np.empty(x.shape[:-2] + (ref.n_blocks(N, blk), x.shape[-1]))
    for j in range(out.shape[-2]):
        out[..., j, :] = x[..., j * blk:(j + 1) * blk, :].sum(axis=-2) / blk
    return out


def _mut_proxy_unscaled(qbar, kbar):
    return np.matmul(qbar, np.swapaxes(kbar, -1, -2))


def _mut_visit_natural(i, nKB, Bq, Bk, order="rotated"):
    return np.arange(nKB, dtype=np.int64)


def _mut_diag_index(i, Bq, Bk, nKB):
    return min(i, nKB - 1)


def _mut_keep_strict(s, m, tau):
    return s > m - tau


def _mut_corr_no_multiplicity(sbar_row, dropped, counts, vbar):
    idx = np.nonzero(dropped)[0]
    return sbar_row[idx], np.ones(idx.size), vbar[idx]


def _mut_corr_summed_value(sbar_row, dropped, counts, vbar):
    idx = np.nonzero(dropped)[0]
    return sbar_row[idx], counts[idx].astype(float), vbar[idx] * counts[idx][:, None]


def _mut_attend_no_pseudo_den(q_rows, k, v, kept_cols, pseudo):
    d = q_rows.shape[-1]
    s = (q_rows @ k[kept_cols].T) / math.sqrt(d)
    m = s.max(axis=1)
    e = np.exp(s - m[:, None])
    num, den = e @ v[kept_cols], e.sum(axis=1)
    if pseudo is not None and pseudo[0].size:
        logits, mult, vals = pseudo
        w = mult[None, :] * np.exp(logits[None, :] - m[:, None])
        num = num + w @ vals
    return num / den[:, None]


def _mut_attend_scale_d(q_rows, k, v, kept_cols, pseudo):
    return ref.__dict__["_orig_attend"](q_rows * (1.0 / math.sqrt(q_rows.shape[-1])), k, v,
                                        kept_cols, pseudo)


def _mut_moments_sample(kbar):
    m = kbar.mean(axis=-2)
    c = kbar - m[..., None, :]
    return m, np.swapaxes(c, -1, -2) @ c / (kbar.shape[-2] - 1)


def _mut_variance_no_d(qbar, cov, variant):
    return np.einsum("...id,...de,...ie->...i", qbar, cov, qbar) if variant == "exact" else \
        np.einsum("...id,...d->...i", qbar * qbar, np.diagonal(cov, axis1=-2, axis2=-1))


def _mut_variance_diag_everywhere(qbar, cov, variant):
    return np.einsum("...id,...d->...i", qbar * qbar, np.diagonal(cov, axis1=-2, axis2=-1)) / qbar.shape[-1]


def _mut_threshold_variance_not_std(qbar, kbar, beta, variant="exact"):
    d = qbar.shape[-1]
    m, cov = ref.key_moments(kbar)
    return np.einsum("...id,...d->...i", qbar, m) / math.sqrt(d) + beta * ref.threshold_variance(qbar, cov, variant)


def _mut_gaussian_keep_no_top(sbar, theta, n_sink_blocks=0):
    keep = sbar >= theta[..., None]
    keep[..., :n_sink_blocks] = True
    return keep


def _mut_sink_blocks_floor(n_sink, Bk):
    return int(n_sink) // Bk


def _mut_token_uses_block_logit(q_rows, kbar, dropped, counts, vbar):
    idx = np.nonzero(dropped)[0]
    d = q_rows.shape[-1]
    qbar = q_rows.mean(axis=0)
    return np.broadcast_to((kbar[idx] @ qbar) / math.sqrt(d), (q_rows.shape[0], idx.size)), \
        counts[idx].astype(np.float64), vbar[idx]


def _mut_token_no_multiplicity(q_rows, kbar, dropped, counts, vbar):
    idx = np.nonzero(dropped)[0]
    d = q_rows.shape[-1]
    return (q_rows @ kbar[idx].T) / math.sqrt(d), np.ones(idx.size), vbar[idx]


def _mut_kept_counts_dropped(keep):
    return (~keep).sum(axis=(-1, -2)).astype(np.int64)


def _mut_kept_one_block_axis(keep):
    return keep.sum(axis=-1)[..., 0].astype(np.int64)


def _mut_topk_one_more(sbar, k):
    return ref.__dict__["_orig_topk"](sbar, k + 1)


def _mut_topp_not_strict(sbar, counts, p):
    keep = np.zeros(sbar.shape, dtype=bool)
    flat_s, flat_k = sbar.reshape(-1, sbar.shape[-1]), keep.reshape(-1, sbar.shape[-1])
    log_n = np.log(counts)
    for r in range(flat_s.shape[0]):
        order = ref.rank_desc(flat_s[r] + log_n)
        w = np.exp(flat_s[r][order] + log_n[order] - (flat_s[r] + log_n).max())
        before = np.concatenate([[0.0], np.cumsum(w)[:-1]])
        flat_k[r, order[before <= p * w.sum()]] = True
    return keep


def _mut_topp_no_counts(sbar, counts, p):
    return ref.__dict__["_orig_topp"](sbar, np.ones_like(counts), p)


MUTANTS = {
    "pool divides by block size": ("pool", _mut_pool_by_blk),
    "proxy without 1/sqrt(d)": ("proxy", _mut_proxy_unscaled),
    "natural visit order": ("visit_order", _mut_visit_natural),
    "diagonal block by index": ("diagonal_block", _mut_diag_index),
    "strict threshold": ("keep_test", _mut_keep_strict),
    "correction without n_j": ("correction_terms", _mut_corr_no_multiplicity),
    "correction with summed value": ("correction_terms", _mut_corr_summed_value),
    "pseudo-keys missing from denominator": ("attend_block", _mut_attend_no_pseudo_den),
    "exact logits scaled by 1/d": ("attend_block", _mut_attend_scale_d),
    "key covariance normalised by nKB - 1": ("key_moments", _mut_moments_sample),
    "threshold variance without 1/d": ("threshold_variance", _mut_variance_no_d),
    "exact threshold from the diagonal only": ("threshold_variance", _mut_variance_diag_everywhere),
    "threshold uses the variance, not sigma": ("gaussian_threshold", _mut_threshold_variance_not_std),
    "top block not forced": ("gaussian_keep", _mut_gaussian_keep_no_top),
    "sink blocks rounded down": ("sink_blocks", _mut_sink_blocks_floor),
    "token correction with the block logit": ("correction_terms_token", _mut_token_uses_block_logit),
    "token correction without n_j": ("correction_terms_token", _mut_token_no_multiplicity),
    "kept count of the dropped blocks": ("kept_per_head", _mut_kept_counts_dropped),
    "kept count of one query block only": ("kept_per_head", _mut_kept_one_block_axis),
    "top-k keeps one block too many": ("topk_keep", _mut_topk_one_more),
    "top-p keeps the block that reaches p exactly": ("topp_keep", _mut_topp_not_strict),
    "top-p without block sizes": ("topp_keep", _mut_topp_no_counts),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_planted_mistakes_are_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setitem(ref.__dict__, "_orig_attend", ref.attend_block)
    monkeypatch.setitem(ref.__dict__, "_orig_topk", ref.topk_keep)
    monkeypatch.setitem(ref.__dict__, "_orig_topp", ref.topp_keep)
    monkeypatch.setattr(ref, attr, fn)
    failed = []
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"planted mistake '{name}' passed every pin"
