"""Plain fp64 CPU oracle for the Sol-Attn forward operator.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may call it. It shares no code with the CUDA path.

What it computes (one query block i of one (batch, head) pair; rows R_i,
n_i = |R_i|; key blocks j with columns C_j, n_j = |C_j|; d = head dim):

1. Pool: q_i = mean of Q over R_i, k_j and v_j = means of K and V over C_j,
   over the valid rows only ("the proxy score for each query-key block pair is
   derived from the means of the corresponding query and key blocks":
   paperlayer summary "Sol-Attn: Accelerating Video Generation Inference via
   On-the-Fly Attention Sparsification", §2 Preliminaries, Block-Sparse
   Attention).
2. Proxy: s_ij = q_i . k_j / sqrt(d).
3. Visit order: key blocks are visited starting at the block holding query
   block i's first token, ascending with wrap-around. The pages do not state an
   order; this is the reading adopted for this build (local attention in video
   DiTs puts the largest proxies near the diagonal).
4. Threshold (on-the-fly block thresholding, paperlayer summary §3
   Methodology, "On-the-fly sparsification"; abstract "comparing block proxy
   scores against a threshold during online softmax"): M(t) is the running
   maximum of the proxies visited so far including the current one, and the
   visited block is kept iff s >= M(t) - tau. The pages' own threshold, a
   query-dependent mean + beta * std from pooled-key moments, is implemented
   beside it (``keep_sets_gaussian``, below).
5. Output, closed form (no online recurrence):
   keep_correct: O_r = [sum_{j kept} sum_{c in C_j} e^{s_rc} v_c
                        + sum_{j dropped} n_j e^{s_ij} v_j]
                       / [sum_{j kept} sum_{c in C_j} e^{s_rc}
                        + sum_{j dropped} n_j e^{s_ij}]
   (zeroth-order proxy-score reuse with pooled keys and summed values:
   paperlayer summary §3 Methodology, "Approximate correction", and App. B,
   "Approximation error"); keep_drop drops the dropped-block terms (abstract,
   "keep-or-drop sparsification"); dense keeps every block.
6. Stats: kept blocks per (b, h) = sum over query blocks of |K_i|.
7. Sinks (optional): the key blocks holding the first n_sink key tokens are kept by
   every query block (text tokens retained as sinks in the exact branch).
8. Token-to-block correction (optional): the dropped block's pseudo-key logit is
   q_r . k_j / sqrt(d) for each row r instead of the block proxy s_ij.

All arithmetic is float64 on the exact bf16 input values.
"""
from __future__ import annotations

import math

import numpy as np

MODES = {"dense": 0, "keep_drop": 1, "keep_correct": 2}
MODE_NAMES = {v: k for k, v in MODES.items()}


def _mode_name(mode):
    if isinstance(mode, str):
        if mode not in MODES:
            raise ValueError(f"unknown mode {mode!r}")
        return mode
    return MODE_NAMES[int(mode)]


def as_f64(x) -> np.ndarray:
    """A torch tensor (any dtype, any device) or array -> float64 numpy array."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------- step 1

def n_blocks(N: int, blk: int) -> int:
    return -(-N // blk)


def block_rows(N: int, blk: int, j: int) -> slice:
    """Rows of block j: [j*blk, min(N, (j+1)*blk))."""
    return slice(j * blk, min(N, (j + 1) * blk))


def valid_counts(N: int, blk: int) -> np.ndarray:
    """n_j: number of valid rows of each block (the last one may be ragged)."""
    return np.array([block_rows(N, blk, j).stop - j * blk for j in range(n_blocks(N, blk))],
                    dtype=np.int64)


def pool(x: np.ndarray, blk: int) -> np.ndarray:
    """Block means over the valid rows: [..., N, d] -> [..., nB, d] (float64)."""
    x = as_f64(x)
    N = x.shape[-2]
    out = np.empty(x.shape[:-2] + (n_blocks(N, blk), x.shape[-1]), dtype=np.float64)
    for j in range(n_blocks(N, blk)):
        rows = x[..., block_rows(N, blk, j), :]
        out[..., j, :] = rows.sum(axis=-2) / rows.shape[-2]
    return out


# ----------------------------------------------------------------- step 2

def proxy(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """s_ij = q_i . k_j / sqrt(d): [..., nQB, d] x [..., nKB, d] -> [..., nQB, nKB]."""
    d = qbar.shape[-1]
    return np.matmul(qbar, np.swapaxes(kbar, -1, -2)) / math.sqrt(d)


# ----------------------------------------------------------------- step 3

def diagonal_block(i: int, Bq: int, Bk: int, nKB: int) -> int:
    """The key block holding query block i's first token (clamped to the last block)."""
    return min((i * Bq) // Bk, nKB - 1)


def visit_order(i: int, nKB: int, Bq: int, Bk: int, order: str = "rotated") -> np.ndarray:
    """pi_i(t), t = 0..nKB-1: the key blocks in the order query block i visits them."""
    if order == "natural":
        return np.arange(nKB, dtype=np.int64)
    if order != "rotated":
        raise ValueError(order)
    j0 = diagonal_block(i, Bq, Bk, nKB)
    return (j0 + np.arange(nKB, dtype=np.int64)) % nKB


# ----------------------------------------------------------------- step 4

def keep_test(s_visited: np.ndarray, running_max: np.ndarray, tau: float) -> np.ndarray:
    """Keep iff the proxy clears the running maximum minus tau."""
    return s_visited >= running_max - tau


def route_row(s_row: np.ndarray, visit: np.ndarray, tau: float):
    """Keep flags and threshold margins of one query block.

    s_row: [nKB] proxies of query block i; visit: the visit order.
    Returns (keep [nKB] bool, margin [nKB] = s - (M(t) - tau) at visit time).
    """
    s_vis = s_row[visit]
    running_max = np.maximum.accumulate(s_vis)
    keep_vis = keep_test(s_vis, running_max, tau)
    keep = np.zeros(s_row.shape[0], dtype=bool)
    keep[visit] = keep_vis
    margin = np.empty(s_row.shape[0], dtype=np.float64)
    margin[visit] = s_vis - (running_max - tau)
    return keep, margin


def sink_blocks(n_sink: int, Bk: int) -> int:
    """Key blocks that hold any of the first n_sink key tokens (text tokens kept as sinks in
    the exact branch: paperlayer summary, App. A Additional Experimental Details). Reading:
    the sinks are a prefix of the key sequence and the blocks overlapping it are kept whole."""
    return -(-int(n_sink) // Bk)


def apply_sinks(keep: np.ndarray, margin: np.ndarray, n_sink: int, Bk: int):
    """Every query block keeps the sink blocks (margin +inf: no threshold decides them)."""
    ns = sink_blocks(n_sink, Bk)
    if ns:
        keep[..., :ns] = True
        margin[..., :ns] = np.inf
    return keep, margin


def keep_sets(q, k, Bq: int, Bk: int, tau: float, mode="keep_correct", order: str = "rotated", n_sink: int = 0):
    """Keep sets of every query block.

    Returns (keep [B, H, nQB, nKB] bool, margin [B, H, nQB, nKB] float64,
    sbar [B, H, nQB, nKB] float64). In dense mode every block is kept and the
    margin is +inf. The sink blocks of ``n_sink`` leading key tokens are kept too; their
    proxies still enter the running maximum, so the other decisions do not change.
    """
    mode = _mode_name(mode)
    q = as_f64(q)
    k = as_f64(k)
    B, H, N, d = q.shape
    nQB, nKB = n_blocks(N, Bq), n_blocks(N, Bk)
    sbar = proxy(pool(q, Bq), pool(k, Bk))
    keep = np.ones((B, H, nQB, nKB), dtype=bool)
    margin = np.full((B, H, nQB, nKB), np.inf)
    if mode == "dense" or tau == math.inf:
        return keep, margin, sbar
    for i in range(nQB):
        visit = visit_order(i, nKB, Bq, Bk, order)
        for b in range(B):
            for h in range(H):
                keep[b, h, i], margin[b, h, i] = route_row(sbar[b, h, i], visit, tau)
    keep, margin = apply_sinks(keep, margin, n_sink, Bk)
    return keep, margin, sbar


def kept_per_head(keep: np.ndarray) -> np.ndarray:
    """Sum of |K_i| over the query blocks of each (b, h): int64 [B, H]."""
    return keep.sum(axis=(-1, -2)).astype(np.int64)


# ----------------------------------------------------------------- step 5

def correction_terms(sbar_row: np.ndarray, dropped: np.ndarray, counts: np.ndarray,
                     vbar: np.ndarray):
    """Pseudo-key logits, weights and values of the dropped blocks of one query block.

    Each dropped block j enters as one pseudo-key with logit s_ij, multiplicity
    n_j and value v_j (its mean V): weight n_j * e^{s_ij}.
    Returns (logits [m], multiplicities [m], values [m, d]).
    """
    idx = np.nonzero(dropped)[0]
    return sbar_row[idx], counts[idx].astype(np.float64), vbar[idx]


def correction_terms_token(q_rows: np.ndarray, kbar: np.ndarray, dropped: np.ndarray, counts: np.ndarray,
                           vbar: np.ndarray):
    """Token-to-block pseudo-keys of the dropped blocks of one query block: the logit of
    row r is q_r . k_j / sqrt(d) with the pooled key k_j (paperlayer summary §3
    Methodology, "Unified execution": a token-to-block score tile determines the approximate
    correction). Returns (logits [n_i, m], multiplicities [m], values [m, d])."""
    idx = np.nonzero(dropped)[0]
    d = q_rows.shape[-1]
    return (q_rows @ kbar[idx].T) / math.sqrt(d), counts[idx].astype(np.float64), vbar[idx]


def attend_block(q_rows, k, v, kept_cols, pseudo):
    """Closed-form weighted softmax of one query block.

    q_rows [n_i, d]; k, v [N, d]; kept_cols: bool [N]; pseudo = (logits,
    multiplicities, values) of the pseudo-keys or None; the logits are one per pseudo-key
    ([m], the same for every row) or one per row and pseudo-key ([n_i, m]).
    """
    d = q_rows.shape[-1]
    s = (q_rows @ k[kept_cols].T) / math.sqrt(d)          # [n_i, n_kept]
    m = s.max(axis=1) if s.shape[1] else np.full(q_rows.shape[0], -np.inf)
    has_pseudo = pseudo is not None and pseudo[0].size
    if has_pseudo:
        logits = np.broadcast_to(pseudo[0], (q_rows.shape[0], pseudo[1].shape[0]))
        m = np.maximum(m, logits.max(axis=1))
    e = np.exp(s - m[:, None])
    num = e @ v[kept_cols]
    den = e.sum(axis=1)
    if has_pseudo:
        _, mult, vals = pseudo
        w = mult[None, :] * np.exp(logits - m[:, None])   # [n_i, m]
        num = num + w @ vals
        den = den + w.sum(axis=1)
    return num / den[:, None]


def forward(q, k, v, Bq: int, Bk: int, tau: float, mode="keep_correct", order: str = "rotated",
            keep: np.ndarray | None = None, qblocks=None, n_sink: int = 0, correction: str = "block"):
    """Sol-Attn output in float64.

    q, k, v: [B, H, N, d] (bf16 torch tensors or arrays; converted exactly).
    keep: optional [B, H, nQB, nKB] override of the keep sets (used to compare
    outputs on the GPU's own keep set where a near-threshold proxy flipped).
    qblocks: None for every query block, or an iterable of (b, h, i) triples.
    correction: "block" (pseudo-key logit s_ij, the same for every row of query block i)
    or "token" (logit q_r . k_j / sqrt(d) per row r).
    Returns (out [B, H, N, d] float64 with NaN rows for query blocks that were
    not computed, keep [B, H, nQB, nKB]).
    """
    if correction not in ("block", "token"):
        raise ValueError(correction)
    mode = _mode_name(mode)
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    B, H, N, d = q.shape
    nQB, nKB = n_blocks(N, Bq), n_blocks(N, Bk)
    if keep is None:
        keep, _, sbar = keep_sets(q, k, Bq, Bk, tau, mode, order, n_sink)
    else:
        keep = np.asarray(keep, dtype=bool)
        sbar = proxy(pool(q, Bq), pool(k, Bk))
    if mode == "dense":
        keep = np.ones_like(keep)
    counts = valid_counts(N, Bk)
    vbar = pool(v, Bk) if mode == "keep_correct" else None
    kbar = pool(k, Bk) if (mode == "keep_correct" and correction == "token") else None
    col_block = np.arange(N) // Bk
    out = np.full(q.shape, np.nan)
    if qblocks is None:
        qblocks = [(b, h, i) for b in range(B) for h in range(H) for i in range(nQB)]
    for b, h, i in qblocks:
        rows = block_rows(N, Bq, i)
        kept_cols = keep[b, h, i][col_block]
        pseudo = None
        if mode == "keep_correct" and correction == "token":
            pseudo = correction_terms_token(q[b, h, rows], kbar[b, h], ~keep[b, h, i], counts, vbar[b, h])
        elif mode == "keep_correct":
            pseudo = correction_terms(sbar[b, h, i], ~keep[b, h, i], counts, vbar[b, h])
        out[b, h, rows] = attend_block(q[b, h, rows], k[b, h], v[b, h], kept_cols, pseudo)
    return out, keep


# ----------------------------------------------------------------- query-dependent Gaussian threshold
#
# The pages' own routing rule (paperlayer summary "Sol-Attn: Accelerating Video
# Generation Inference via On-the-Fly Attention Sparsification", §2 Block-Sparse
# Attention, Figure 2: a threshold from the proxy-logit mean mu, standard deviation
# sigma and a standardized offset beta; §3 Methodology, "Dynamic threshold routing":
# query-dependent thresholds from proxy-score statistics with one shared standardized
# cutoff, the mean and variance taken from the pooled keys' first and second moments;
# App. "Threshold variance derivation" and "Diagonal threshold estimator": the exact
# variance from the pooled-key covariance, or its diagonal v_K = diag(Cov[K]) only).
# Readings (the pages do not fix them): the moments run over the key blocks with equal
# weight and 1/nKB normalisation; a block is kept iff its proxy is >= the threshold;
# the row's top block (largest proxy, lowest index on ties) is always kept, so no
# query block's exact set is empty.

def key_moments(kbar: np.ndarray):
    """Mean and covariance of the pooled keys over the key blocks:
    [..., nKB, d] -> (mean [..., d], cov [..., d, d]), normalised by 1/nKB."""
    m = kbar.mean(axis=-2)
    c = kbar - m[..., None, :]
    return m, np.swapaxes(c, -1, -2) @ c / kbar.shape[-2]


def threshold_variance(qbar: np.ndarray, cov: np.ndarray, variant: str) -> np.ndarray:
    """sigma_i^2 of the proxies of query block i: q_i^T Cov[K] q_i / d ("exact") or
    sum_e q_ie^2 Cov[K]_ee / d ("diag"): [..., nQB, d], [..., d, d] -> [..., nQB]."""
    d = qbar.shape[-1]
    if variant == "exact":
        return np.einsum("...id,...de,...ie->...i", qbar, cov, qbar) / d
    if variant == "diag":
        return np.einsum("...id,...d->...i", qbar * qbar, np.diagonal(cov, axis1=-2, axis2=-1)) / d
    raise ValueError(variant)


def gaussian_threshold(qbar: np.ndarray, kbar: np.ndarray, beta: float, variant: str = "exact") -> np.ndarray:
    """theta_i = mu_i + beta * sigma_i with mu_i = q_i . E[K] / sqrt(d): [..., nQB]."""
    d = qbar.shape[-1]
    m, cov = key_moments(kbar)
    mu = np.einsum("...id,...d->...i", qbar, m) / math.sqrt(d)
    sigma = np.sqrt(np.maximum(threshold_variance(qbar, cov, variant), 0.0))
    return mu + beta * sigma


def gaussian_keep(sbar: np.ndarray, theta: np.ndarray, n_sink_blocks: int = 0) -> np.ndarray:
    """Keep iff s_ij >= theta_i, plus the sink blocks; a row left empty keeps its top
    block: [..., nQB, nKB] bool."""
    keep = sbar >= theta[..., None]
    keep[..., :n_sink_blocks] = True
    top = np.argmax(sbar, axis=-1)
    empty = ~keep.any(axis=-1)
    top_keep = np.zeros_like(keep)
    np.put_along_axis(top_keep, top[..., None], True, axis=-1)
    return keep | (top_keep & empty[..., None])


def keep_sets_gaussian(q, k, Bq: int, Bk: int, beta: float, variant: str = "exact", mode="keep_correct",
                       n_sink: int = 0):
    """Keep sets under the Gaussian threshold.

    Returns (keep, margin = s - theta (+inf for a top block kept only because it is
    the top block), sbar), all [B, H, nQB, nKB]. In dense mode, or for beta = -inf,
    every block is kept.
    """
    mode = _mode_name(mode)
    q, k = as_f64(q), as_f64(k)
    N = q.shape[-2]
    qbar, kbar = pool(q, Bq), pool(k, Bk)
    sbar = proxy(qbar, kbar)
    if mode == "dense" or beta == -math.inf:
        return np.ones(sbar.shape, dtype=bool), np.full(sbar.shape, np.inf), sbar
    theta = gaussian_threshold(qbar, kbar, beta, variant)
    keep = gaussian_keep(sbar, theta, sink_blocks(n_sink, Bk))
    margin = sbar - theta[..., None]
    margin = np.where(keep & (margin < 0), np.inf, margin)
    keep, margin = apply_sinks(keep, margin, n_sink, Bk)
    return keep, margin, sbar


# ----------------------------------------------------------------- top-k and top-p routing
#
# The routing rules the pages compare Sol-Attn's on-the-fly thresholding against
# (paperlayer summary "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly
# Attention Sparsification", §2 Block-Sparse Attention: top-k keeps a fixed budget of the
# top-ranked blocks, top-p a dynamic one by cumulative probability mass, and both need
# the whole proxy row; §4 Experiments, "Efficient On-the-Fly Sparsification": routing
# measured against both). Readings (the pages do not fix them): top-k keeps the k blocks
# with the largest proxies of each query block's row; top-p keeps the smallest set of
# heaviest blocks whose share of the row's mass reaches p, where block j's mass is
# n_j e^{s_ij} (its attention mass under the same zeroth-order approximation as the
# correction; with equal block sizes this is the softmax of the proxies). Ties go to the
# lower block index in both.

def rank_desc(s_row: np.ndarray) -> np.ndarray:
    """Block indices of one proxy row, largest proxy first, lower index first on ties."""
    return np.lexsort((np.arange(s_row.shape[0]), -s_row))


def topk_keep(sbar: np.ndarray, k: int) -> np.ndarray:
    """Keep the min(k, nKB) largest proxies of every row: [..., nQB, nKB] -> bool."""
    keep = np.zeros(sbar.shape, dtype=bool)
    flat_s = sbar.reshape(-1, sbar.shape[-1])
    flat_k = keep.reshape(-1, sbar.shape[-1])
    for r in range(flat_s.shape[0]):
        flat_k[r, rank_desc(flat_s[r])[:k]] = True
    return keep


def topp_keep(sbar: np.ndarray, counts: np.ndarray, p: float) -> np.ndarray:
    """Rank the blocks of a row by mass n_j e^{s_ij} (largest first) and keep the shortest
    prefix whose mass reaches p of the row's total: a block is kept iff the mass ranked
    before it is < p * total."""
    keep = np.zeros(sbar.shape, dtype=bool)
    flat_s = sbar.reshape(-1, sbar.shape[-1])
    flat_k = keep.reshape(-1, sbar.shape[-1])
    log_n = np.log(counts)
    for r in range(flat_s.shape[0]):
        order = rank_desc(flat_s[r] + log_n)  # by mass, largest first
        w = np.exp(flat_s[r][order] + log_n[order] - (flat_s[r] + log_n).max())
        before = np.concatenate([[0.0], np.cumsum(w)[:-1]])
        flat_k[r, order[before < p * w.sum()]] = True
    return keep


def keep_sets_topk(q, k, Bq: int, Bk: int, kb: int):
    """Top-k keep sets from the block proxies (see above): [B, H, nQB, nKB] bool."""
    return topk_keep(proxy(pool(as_f64(q), Bq), pool(as_f64(k), Bk)), kb)


def keep_sets_topp(q, k, Bq: int, Bk: int, p: float):
    """Top-p keep sets from the block proxies (see above): [B, H, nQB, nKB] bool."""
    q, k = as_f64(q), as_f64(k)
    return topp_keep(proxy(pool(q, Bq), pool(k, Bk)), valid_counts(q.shape[-2], Bk).astype(np.float64), p)


def sample_qblocks(B, H, nQB, Bq, Bk, nKB, per_head=64, seed=0):
    """Seeded sample of query blocks per head, plus block 0, the last (ragged) one and
    the blocks whose diagonal is at the extremes."""
    rng = np.random.default_rng(seed)
    picks = []
    for b in range(B):
        for h in range(H):
            chosen = set(int(x) for x in rng.choice(nQB, size=min(per_head, nQB), replace=False))
            chosen.update({0, nQB - 1, nQB // 2})
            picks.extend((b, h, i) for i in sorted(chosen))
    return picks
