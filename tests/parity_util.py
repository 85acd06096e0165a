"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI and
compare it with the fp64 oracle on the same bf16 inputs."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import oracle.solattn_ref as ref

# Tolerances (bf16 inputs, fp32 accumulation, bf16 output):
#  * max-abs, by magnitude band of the oracle value o_ref:
#      |o_ref| <  BAND: |o - o_ref| <= MAX_ABS, the literal bound;
#      |o_ref| >= BAND: |o - o_ref| <= MAX_ABS + ulp_bf16(o_ref) / 2. The output is stored in
#      bf16, whose spacing is 2^-5 for |o| in [4, 8): rounding alone moves such an output
#      by up to 1.6e-2, so there the 1e-2 bound is applied to the error beyond the
#      half-ulp of the bf16 result.
#  * mean relative: sum|o - o_ref| / sum|o_ref| <= MEAN_REL over every checked element.
#  * kept sets: equal, except where the oracle's proxy lies within NEAR of the threshold.
# Setting SOLATTN_PARITY_LOG=<path> appends one JSON line of measured errors per case.
MAX_ABS = 1e-2
MEAN_REL = 2e-3
NEAR = 1e-3
BAND = 2.0


def half_ulp_bf16(x: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers (8 significant bits) at |x|."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 0.5 * np.exp2(e - 7)


def unpack_mask(mask: torch.Tensor, nKB: int) -> np.ndarray:
    m = mask.cpu().contiguous().numpy().view(np.uint32)
    bits = np.unpackbits(m.view(np.uint8), bitorder="little").reshape(m.shape[:-1] + (-1,))
    return bits[..., :nKB].astype(bool)


def run_gpu(q, k, v, Bq, Bk, tau, mode, gauss=None, n_sink=0, correction="block"):
    """gauss: None (running-max rule with tau) or (beta, variant) for the Gaussian threshold;
    n_sink > 0 or the token correction go through solattn_forward_ex."""
    from block_sparse_online_b200 import solattn
    dev = torch.device("cuda:0")
    qd, kd, vd = (t.to(dev).contiguous() for t in (q, k, v))
    ws = solattn.alloc_workspace(*qd.shape, Bq, Bk, dev)
    if n_sink or correction != "block":
        rule = "running_max" if gauss is None else f"gauss_{gauss[1]}"
        out, kept, mask = solattn.solattn_forward_ex(qd, kd, vd, Bq, Bk, mode, rule, tau=tau,
                                                     beta=0.0 if gauss is None else gauss[0], n_sink=n_sink,
                                                     correction=correction, keep_mask=True, workspace=ws)
    elif gauss is None:
        out, kept, mask = solattn.solattn_forward(qd, kd, vd, Bq, Bk, tau, mode, keep_mask=True, workspace=ws)
    else:
        out, kept, mask = solattn.solattn_forward_gaussian(qd, kd, vd, Bq, Bk, gauss[0], gauss[1], mode,
                                                           keep_mask=True, workspace=ws)
    st = solattn.solattn_get_status(ws)
    assert st == 0, f"device status {st}"
    torch.cuda.synchronize()
    return out.cpu(), kept.cpu(), mask


def extreme_blocks(keep: np.ndarray):
    """Per head, the query blocks that keep the most and the fewest key blocks (the heaviest
    and lightest tiles): [(b, h, i), ...]."""
    cnt = keep.sum(axis=-1)
    picks = []
    for b in range(cnt.shape[0]):
        for h in range(cnt.shape[1]):
            picks.append((b, h, int(np.argmax(cnt[b, h]))))
            picks.append((b, h, int(np.argmin(cnt[b, h]))))
    return picks


def _log(label, stats):
    path = os.environ.get("SOLATTN_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": label, **stats}) + "\n")


def check_case(q, k, v, Bq, Bk, tau, mode, qblocks=None, label="", gauss=None, n_sink=0, correction="block"):
    """Run one case on the GPU and compare keep sets, counts and outputs with the oracle.
    gauss: None (running-max rule with tau) or (beta, variant); n_sink: sink tokens.
    qblocks: None (every query block) or a list of (b, h, i); a sample is widened by each
    head's most- and least-kept query blocks of the GPU's keep set.
    Returns a dict of the measured errors."""
    B, H, N, d = q.shape
    nQB, nKB = -(-N // Bq), -(-N // Bk)
    out, kept, mask = run_gpu(q, k, v, Bq, Bk, tau, mode, gauss, n_sink, correction)
    gpu_keep = unpack_mask(mask, nKB)
    if gauss is None:
        ref_keep, margin, _ = ref.keep_sets(q, k, Bq, Bk, tau, mode, n_sink=n_sink)
    else:
        ref_keep, margin, _ = ref.keep_sets_gaussian(q, k, Bq, Bk, gauss[0], gauss[1], mode, n_sink=n_sink)
    diff = gpu_keep != ref_keep
    flips = int(diff.sum())
    if flips:
        worst = float(np.abs(margin[diff]).max())
        assert worst < NEAR, f"{label}: keep set differs away from the threshold (|margin| {worst})"
    # per-head kept counts equal the GPU's own mask popcounts, and the oracle's where no flip
    np.testing.assert_array_equal(kept.numpy(), gpu_keep.sum(axis=(-1, -2)))
    if not flips:
        np.testing.assert_array_equal(kept.numpy(), ref.kept_per_head(ref_keep))
    if qblocks is not None:
        qblocks = sorted(set(qblocks) | set(extreme_blocks(gpu_keep)))
    want, _ = ref.forward(q, k, v, Bq, Bk, tau, mode, keep=gpu_keep, qblocks=qblocks, correction=correction)
    got = out.to(torch.float64).numpy()
    sel = ~np.isnan(want[..., 0])
    w, g = want[sel], got[sel]
    assert np.isfinite(g).all(), f"{label}: non-finite output"
    err = np.abs(g - w)
    small = np.abs(w) < BAND
    max_small = float(err[small].max()) if small.any() else 0.0
    max_large = float(err[~small].max()) if (~small).any() else 0.0
    excess_large = float((err[~small] - half_ulp_bf16(w[~small])).max()) if (~small).any() else 0.0
    mean_rel = float(err.sum() / np.abs(w).sum())
    stats = {"flips": flips, "max_abs": float(err.max()), "max_abs_below_band": max_small,
             "max_abs_above_band": max_large, "max_abs_above_band_beyond_half_ulp": excess_large,
             "n_above_band": int((~small).sum()), "mean_rel": mean_rel, "keep_ratio": float(gpu_keep.mean()),
             "rows": int(sel.sum())}
    _log(label, stats)
    assert max_small <= MAX_ABS, f"{label}: max abs error {max_small} where |o| < {BAND}"
    assert excess_large <= MAX_ABS, f"{label}: max abs error beyond bf16 half-ulp {excess_large} where |o| >= {BAND}"
    assert mean_rel <= MEAN_REL, f"{label}: mean relative error {mean_rel}"
    return stats


def sampled_blocks(B, H, N, Bq, Bk, per_head, seed=0):
    nQB, nKB = -(-N // Bq), -(-N // Bk)
    return ref.sample_qblocks(B, H, nQB, Bq, Bk, nKB, per_head=per_head, seed=seed)


__all__ = ["check_case", "run_gpu", "unpack_mask", "sampled_blocks", "half_ulp_bf16", "extreme_blocks", "MAX_ABS",
           "MEAN_REL", "NEAR", "BAND"]
