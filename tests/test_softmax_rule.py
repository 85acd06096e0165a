"""The attention kernel's per-row softmax rule, replayed on the CPU (no GPU needed).

Each row sees its key tiles one at a time. From its second tile on, a tile is exponentiated
against the row's current reference max m (log2 units) without the tile's maximum; if some
row sum of the tile exceeds 2^15 the tile is redone the way a first tile is: the reference
moves to the tile maximum when that exceeds m by more than 8, and O and l are rescaled. P is
stored in fp16, O and l accumulate in fp32. The checks: no P value ever overflows fp16, the
normalised output matches an fp64 softmax within the kernel's tolerance, and a row sum above
2^15 always comes with a maximum more than 8 above the reference (so a redo moves it).
"""
import numpy as np
import pytest

SLACK = 8.0
LIMIT = 2.0 ** 15
FP16_MAX = 65504.0


def replay(s_log2, v, bk):
    """s_log2: [n_tiles * bk] logits in log2 units of one row; v: [n_tiles * bk, d]."""
    m = -np.inf
    o = np.zeros(v.shape[1], dtype=np.float32)
    l = np.float32(0.0)
    redo = 0
    for t in range(len(s_log2) // bk):
        x = s_log2[t * bk:(t + 1) * bk].astype(np.float32)
        vt = v[t * bk:(t + 1) * bk].astype(np.float32)
        done = False
        if m != -np.inf:
            p = np.exp2(x - np.float32(m))
            lsum = p.astype(np.float32).sum(dtype=np.float32)
            done = bool(lsum <= LIMIT)
            if not done:
                redo += 1
                assert x.max() > m + SLACK  # the reference will move
        alpha = np.float32(1.0)
        if not done:
            mx = np.float32(x.max())
            if mx > m + SLACK:
                if m != -np.inf:
                    alpha = np.float32(np.exp2(np.float32(m) - mx))
                m = float(mx)
            p = np.exp2(x - np.float32(m))
        assert np.isfinite(p).all() and p.max() <= LIMIT < FP16_MAX
        p16 = p.astype(np.float16)
        l = l * alpha + p.astype(np.float32).sum(dtype=np.float32)
        o = o * alpha + p16.astype(np.float32) @ vt
    return o / l, redo


def exact(s_log2, v):
    w = np.exp2(s_log2 - s_log2.max())
    return (w[:, None] * v).sum(0) / w.sum()


@pytest.mark.parametrize("pattern", ["random", "rising", "jump", "sharp", "flat_high"])
def test_lagging_reference_rule(pattern):
    rng = np.random.default_rng(7)
    bk, n_tiles, d = 128, 24, 64
    n = bk * n_tiles
    if pattern == "random":
        s = rng.normal(0.0, 3.0, n)
    elif pattern == "rising":  # the row maximum grows tile after tile
        s = rng.normal(0.0, 1.0, n) + np.repeat(np.arange(n_tiles) * 1.5, bk)
    elif pattern == "jump":  # one late tile far above everything before it
        s = rng.normal(0.0, 2.0, n)
        s[17 * bk:18 * bk] += 40.0
    elif pattern == "sharp":  # a few huge logits inside otherwise small tiles
        s = rng.normal(0.0, 0.5, n)
        s[rng.choice(n, 5, replace=False)] += rng.uniform(10, 30, 5)
    else:  # every tile sits 7.9 above the first one: sums near 2^15 without a single large value
        s = np.full(n, 7.9) + rng.normal(0.0, 0.01, n)
        s[:bk] = rng.normal(0.0, 0.01, bk)
    v = rng.normal(0.0, 1.0, (n, d))
    got, redo = replay(s, v, bk)
    want = exact(s, v)
    err = np.abs(got - want)
    assert err.max() <= 1e-2 and err.sum() / np.abs(want).sum() <= 2e-3, (pattern, err.max())
    if pattern in ("jump", "rising"):
        assert redo >= 1  # the rule did have to move its reference
