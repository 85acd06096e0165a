"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI and
compare it with the fp64 oracle on the same bf16 inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle.solattn_ref as ref

# Tolerances (bf16 inputs, fp32 accumulation, bf16 output):
#  * max-abs: |o - o_ref| <= MAX_ABS + ulp_bf16(o_ref) / 2 elementwise. The output is
#    stored in bf16, whose spacing is 2^-5 for |o| in [4, 8): rounding alone moves such
#    an output by up to 1.6e-2, so the 1e-2 bound is applied to the error beyond the
#    half-ulp of the bf16 result.
#  * mean relative: sum|o - o_ref| / sum|o_ref| <= MEAN_REL over every checked element.
#  * kept sets: equal, except where the oracle's proxy lies within NEAR of the threshold.
MAX_ABS = 1e-2
MEAN_REL = 2e-3
NEAR = 1e-3


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


def check_case(q, k, v, Bq, Bk, tau, mode, qblocks=None, label="", gauss=None, n_sink=0, correction="block"):
    """Run one case on the GPU and compare keep sets, counts and outputs with the oracle.
    gauss: None (running-max rule with tau) or (beta, variant); n_sink: sink tokens.
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
    want, _ = ref.forward(q, k, v, Bq, Bk, tau, mode, keep=gpu_keep, qblocks=qblocks, correction=correction)
    got = out.to(torch.float64).numpy()
    sel = ~np.isnan(want[..., 0])
    w, g = want[sel], got[sel]
    assert np.isfinite(g).all(), f"{label}: non-finite output"
    err = np.abs(g - w)
    max_abs = float(err.max())
    excess = float((err - half_ulp_bf16(w)).max())
    mean_rel = float(err.sum() / np.abs(w).sum())
    assert excess <= MAX_ABS, f"{label}: max abs error beyond bf16 half-ulp {excess} (raw {max_abs})"
    assert mean_rel <= MEAN_REL, f"{label}: mean relative error {mean_rel}"
    return {"flips": flips, "max_abs": max_abs, "max_abs_beyond_half_ulp": excess, "mean_rel": mean_rel,
            "keep_ratio": float(gpu_keep.mean()), "rows": int(sel.sum())}


def sampled_blocks(B, H, N, Bq, Bk, per_head, seed=0):
    nQB, nKB = -(-N // Bq), -(-N // Bk)
    return ref.sample_qblocks(B, H, nQB, Bq, Bk, nKB, per_head=per_head, seed=seed)


__all__ = ["check_case", "run_gpu", "unpack_mask", "sampled_blocks", "half_ulp_bf16", "MAX_ABS", "MEAN_REL", "NEAR"]
