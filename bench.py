#!/usr/bin/env python
"""Benchmark of the Sol-Attn forward operator on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config video480] [--tau 6] [--mode keep_correct] [--no-sweep]

One step is one solattn_forward call (block pooling + the fused routed
attention kernel) over one batch of synthetic spatio-temporal Q/K/V of the
named configuration, inputs resident in HBM. The headline workload is the 480p
video shape (B=1, H=12, N=32760, d=128, 128x128 blocks), keep_correct at tau=6.
Prints ONE JSON line (rank 0). Multi-GPU runs are independent replicas (weak
scaling): the operator has no cross-GPU exchange.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload on the host cores (the baseline the pages' method is checked against).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ["block_sparse_online_b200/csrc/attn_kernel.cuh", "block_sparse_online_b200/csrc/ptx_sm100.cuh",
                  "block_sparse_online_b200/csrc/solattn_api.cu"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="video480")
    ap.add_argument("--tau", type=float, default=6.0)
    ap.add_argument("--mode", default="keep_correct", choices=["dense", "keep_drop", "keep_correct"])
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--all-configs", default="tiny,image,video480,video720,long",
                    help="configurations swept after the timed region (comma-separated; empty: none)")
    ap.add_argument("--heads", type=int, default=0,
                    help="use only this many heads of the configuration (small profiling captures)")
    return ap.parse_args()


def kernel_hash():
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        return float(m["bf16_tflops"]), float(m["hbm_gbs"]), "measured"
    return FALLBACK_BF16_TFLOPS, FALLBACK_HBM_GBS, "fallback"


def traffic_record():
    """DRAM bytes per attention-kernel launch from the committed ncu summary, if it was
    taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("kernel_hash") != kernel_hash():
        return None
    return rec


# ------------------------------------------------------------------ accounting

def block_sizes(N, blk):
    nb = -(-N // blk)
    return np.array([min(N, (i + 1) * blk) - i * blk for i in range(nb)], dtype=np.float64)


def executed_flops(mask_bits, N, Bq, Bk, d):
    """4 d sum over kept (i, j) of n_i n_j: the two matmuls on the kept blocks."""
    return 4.0 * d * float(np.einsum("bhij,i,j->", mask_bits.astype(np.float64),
                                     block_sizes(N, Bq), block_sizes(N, Bk)))


def unpack(mask, nKB):
    m = mask.cpu().contiguous().numpy().view(np.uint32)
    bits = np.unpackbits(m.view(np.uint8), bitorder="little").reshape(m.shape[:-1] + (-1,))
    return bits[..., :nKB].astype(bool)


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """SM clock and clock-event reasons of the benchmarked GPU, sampled in a background
    thread every ``period_s`` seconds through NVML (so that even a timed region of a few
    tens of milliseconds gets samples), or by ``nvidia-smi -lms 50`` where NVML is absent.
    The GPU is found by its UUID, so the index mapping of CUDA_VISIBLE_DEVICES does not
    matter. Read-only: no clock or other GPU setting is changed."""
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index, period_s=0.001):
        self.index = index
        self.period = period_s
        self.samples = []  # (sm_mhz, max_mhz, set of reason names)
        self.proc = None
        self.thread = None
        self.stop_flag = threading.Event()
        self.source = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(self.index).uuid)
        if not uuid.startswith("GPU-"):
            uuid = "GPU-" + uuid
        return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid)

    def _poll_nvml(self, nv, h):
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        while not self.stop_flag.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, mx, {n for n, b in bits.items() if r & b}))
            except nv.NVMLError:
                pass
            time.sleep(self.period)

    def _read_smi(self):
        for line in self.proc.stdout:
            f = [x.strip() for x in line.strip().split(",")]
            if len(f) < 9:
                continue
            try:
                sm, mx = float(f[1]), float(f[2])
            except ValueError:
                continue
            self.samples.append((sm, mx, {n for n, val in zip(self.NAMES, f[5:9])
                                          if val.lower().startswith("active")}))

    def start(self):
        """Start sampling and wait (up to 10 s) for the first sample, so that the samples
        taken after mark() fall inside the region being timed."""
        try:
            nv, h = self._nvml_handle()
            self.thread = threading.Thread(target=self._poll_nvml, args=(nv, h), daemon=True)
            self.source = f"nvml every {self.period * 1e3:.0f} ms"
        except Exception:  # no NVML: fall back to nvidia-smi
            try:
                self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                                              "--format=csv,noheader,nounits", "-lms", "50"],
                                             stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except (OSError, ValueError):
                return
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
            self.source = "nvidia-smi -lms 50"
        self.thread.start()
        t0 = time.time()
        while not self.samples and time.time() - t0 < 10:
            time.sleep(0.005)

    def mark(self):
        """Index of the next sample: samples from here on fall in the region being timed."""
        return len(self.samples)

    def stop(self, first=0, last=None):
        if self.thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"], "samples": 0}
        self.stop_flag.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.thread.join(timeout=5)
        sel = self.samples[first:last]
        sm = [x[0] for x in sel]
        reasons = set().union(*[x[2] for x in sel]) if sel else set()
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": sel[-1][1] if sel else None,
                "reasons": sorted(reasons), "samples": len(sm), "source": self.source}


# ------------------------------------------------------------------ CPU baseline (oracle)

def cpu_oracle_rate(cfg, q, k, v, tau, mode, budget_s, seed=0):
    """Time the fp64 oracle on a bounded sample of the workload and extrapolate.

    The sample: the keep sets of one head (pooling, proxies and routing of all its query
    blocks) plus the attention of query blocks of that head, as many as fit in
    ``budget_s`` seconds. Returns (dense-equiv TFLOP/s of the extrapolated full step,
    description, extrapolated seconds per full step, seconds actually timed).
    """
    import oracle.solattn_ref as ref
    B, H, N, d = q.shape
    nQB = -(-N // cfg.Bq)
    rng = np.random.default_rng(seed)
    qh, kh, vh = q[:1, :1], k[:1, :1], v[:1, :1]
    t0 = time.perf_counter()
    keep, _, _ = ref.keep_sets(qh, kh, cfg.Bq, cfg.Bk, tau, mode)
    t_route = time.perf_counter() - t0
    order = rng.permutation(nQB)
    done, t_att = 0, 0.0
    while done < nQB and t_att < budget_s:
        blk = [(0, 0, int(order[done]))]
        t1 = time.perf_counter()
        ref.forward(qh, kh, vh, cfg.Bq, cfg.Bk, tau, mode, keep=keep, qblocks=blk)
        t_att += time.perf_counter() - t1
        done += 1
    per_head = t_route + t_att / done * nQB
    total = per_head * B * H
    dense = cfg.dense_flops()
    desc = (f"oracle keep sets of 1 of {B * H} heads ({t_route:.2f} s) + attention of {done} of {nQB} query "
            f"blocks of that head ({t_att:.2f} s), extrapolated linearly to {B * H} heads x {nQB} blocks")
    return dense / total / 1e12, desc, total, t_route + t_att


def cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


# ------------------------------------------------------------------ main

def rank_config(cfg, rank):
    """Each rank of a multi-GPU run solves an independent problem of the same shape
    (weak scaling): the same configuration with its own input seed."""
    import dataclasses
    return cfg if rank == 0 else dataclasses.replace(cfg, seed=cfg.seed + 7919 * rank)


def max_over_ranks(x, world, device="cpu"):
    """The largest value of x over the ranks (device times are reduced this way)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, flops_per_rank, ms):
    """Throughput of the whole job: the work all ranks did over the slowest rank's time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


METRIC = "sparse-attn dense-equiv TFLOP/s (ms/call, executed TFLOP/s and keep ratio alongside)"
UNIT = "TFLOP/s (dense-equivalent)"


def config_dict(args, cfg, world):
    """The workload description both arms print."""
    B, H, N, d = cfg.shape()
    elem = B * H * N * d
    return {"workload": f"{args.config}: {cfg.note}", "mode": args.mode, "tau": args.tau,
            "B": B, "H": H, "N": N, "d": d, "Bq": cfg.Bq, "Bk": cfg.Bk,
            "l2": "inputs larger than L2 (q, k, v = %.0f MB)" % (3 * elem * 2 / 1e6),
            "parallelism": f"replicas x{world}"}


def reference_arm(args, world, rank):
    if rank != 0:
        return
    from block_sparse_online_b200 import synth
    cfg = synth.CONFIGS[args.config]
    q, k, v = synth.make_inputs(cfg)
    vals, timed, full, desc = [], [], [], ""
    budget = max(2.0, min(args.cpu_seconds, 120.0 / max(1, args.steps + args.warmup)))
    for step in range(args.warmup + args.steps):
        rate, desc, sec_full, sec_timed = cpu_oracle_rate(cfg, q, k, v, args.tau, args.mode, budget, seed=step)
        if step >= args.warmup:
            vals.append(rate)
            timed.append(sec_timed)
            full.append(sec_full)
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value,
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        # Each reference step is a bounded sample of the workload (the oracle would take
        # minutes per full step): ms_per_step is the time actually measured per sampled
        # step; value is the rate extrapolated from it to the full step (below).
        "ms_per_step": statistics.median(timed) * 1e3,
        "step_is_sample": True,
        "extrapolated_full_step_ms": statistics.median(full) * 1e3,
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(args, cfg, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores(), "kind": "oracle",
                         "sample": desc + " (one such sample per step)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def issued_flops(mask_bits, N, Bq, Bk, d):
    """FLOPs the tensor cores issue: every 128-row query tile runs Q K^T and P V over the
    union of its query blocks' kept key blocks, full 128 x Bk tiles (ragged rows and columns
    and rows of a query block that did not keep the entry are computed and masked)."""
    B, H, nQB, nKB = mask_bits.shape
    sub = 128 // Bq
    pad = (-nQB) % sub
    m = np.concatenate([mask_bits, np.zeros((B, H, pad, nKB), dtype=bool)], axis=2) if pad else mask_bits
    union = m.reshape(B, H, -1, sub, nKB).any(axis=3)
    return 4.0 * 128 * Bk * d * float(union.sum())


def quantiles(x):
    x = np.asarray(x, dtype=np.float64)
    return {q: round(float(np.quantile(x, p)), 5) for q, p in
            (("min", 0.0), ("p10", 0.1), ("p50", 0.5), ("p90", 0.9), ("max", 1.0))} | {"mean": round(float(x.mean()), 5)}


# Spin of the GPU (clock cycles, ~10 ms) before a timed group of calls, so that the host's
# enqueue latency does not show up as idle GPU time between the events.
SPIN_CYCLES = 20_000_000


def device_ms(fn, stream, reps=5, warm=2, rounds=3):
    """Device time per call of `fn` in ms: `reps` back-to-back calls between two CUDA events
    on `stream`, recorded behind a spin kernel that keeps the GPU busy while the host enqueues
    them; the median over `rounds` groups, after `warm` untimed calls."""
    import torch
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(rounds):
        torch.cuda._sleep(SPIN_CYCLES)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(reps):
            fn()
        a1.record(stream)
        torch.cuda.synchronize()
        ts.append(a0.elapsed_time(a1) / reps)
    return statistics.median(ts)


def config_sweep(name, dev, stream, peak_tf, reps=5):
    """One configuration: every (mode, tau) of its sweep timed as whole solattn_forward calls
    (median of `reps` after 2 warm-up calls), with keep ratios (block and token-weighted),
    executed, issued and dense-equivalent TFLOP/s, the correction ablation against the dense
    output at identical keep sets (rel-l2 and cosine similarity of keep_drop and keep_correct,
    paperlayer summary §4 "Ablations"), the keep-ratio distribution per head and per query
    block, and torch's bf16 SDPA on the same inputs for context."""
    import torch
    from block_sparse_online_b200 import solattn, synth
    cfg = synth.CONFIGS[name]
    B, H, N, d = cfg.shape()
    q, k, v = synth.make_inputs(cfg)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    del q, k, v
    ws = solattn.alloc_workspace(B, H, N, d, cfg.Bq, cfg.Bk, dev)
    out = torch.empty_like(qd)
    kept = torch.empty((B, H), dtype=torch.int64, device=dev)
    dense_flops = cfg.dense_flops()
    bq, bk = block_sizes(N, cfg.Bq), block_sizes(N, cfg.Bk)

    def timed(fn):
        return device_ms(fn, stream, reps=reps)

    dense_out, _, _ = solattn.solattn_forward(qd, kd, vd, cfg.Bq, cfg.Bk, 0.0, "dense", workspace=ws)
    dense_out = dense_out.float()
    rows = []
    for mode in ("dense", "keep_drop", "keep_correct"):
        for tau in ((0.0,) if mode == "dense" else cfg.taus):
            o, _, m = solattn.solattn_forward(qd, kd, vd, cfg.Bq, cfg.Bk, tau, mode, keep_mask=True, workspace=ws)
            if solattn.solattn_get_status(ws) != 0:
                raise RuntimeError(f"{name} {mode} {tau}: device status")
            bits = unpack(m, cfg.nKB)
            ms = timed(lambda: solattn.solattn_forward(qd, kd, vd, cfg.Bq, cfg.Bk, tau, mode, out=out,
                                                       kept_per_head=kept, workspace=ws))
            ef = executed_flops(bits, N, cfg.Bq, cfg.Bk, d)
            row = {"mode": mode, "tau": None if (mode == "dense" or math.isinf(tau)) else tau, "ms": round(ms, 4),
                   "keep_ratio": round(float(bits.mean()), 5),
                   "keep_ratio_tokens": round(float(np.einsum("bhij,i,j->", bits.astype(np.float64), bq, bk)
                                                    / (B * H * N * N)), 5),
                   "exec_tflops": round(ef / (ms * 1e-3) / 1e12, 2),
                   "exec_frac_of_peak": round(ef / (ms * 1e-3) / 1e12 / peak_tf, 4),
                   "dense_equiv_tflops": round(dense_flops / (ms * 1e-3) / 1e12, 2)}
            if cfg.Bq == 64:
                isf = issued_flops(bits, N, cfg.Bq, cfg.Bk, d)
                row["issued_tflops"] = round(isf / (ms * 1e-3) / 1e12, 2)
                row["issued_over_executed"] = round(isf / ef, 4)
            if mode != "dense":
                x, y = o.float().flatten(), dense_out.flatten()
                row["rel_l2_vs_dense"] = round(float(torch.linalg.vector_norm(x - y) / torch.linalg.vector_norm(y)), 6)
                row["cos_sim_vs_dense"] = round(float(torch.nn.functional.cosine_similarity(x, y, dim=0)), 6)
                if mode == "keep_correct":
                    per_head = bits.mean(axis=(-1, -2)).reshape(-1)
                    per_qb = bits.mean(axis=-1).reshape(-1)
                    row["keep_ratio_per_head"] = quantiles(per_head)
                    row["keep_ratio_per_query_block"] = quantiles(per_qb)
                    row["keep_ratio_per_query_block_hist"] = np.histogram(per_qb, bins=10, range=(0.0, 1.0))[0].tolist()
            rows.append(row)
    # Context: torch's fused bf16 attention on the same inputs. The unfused math backend would
    # materialise N x N scores (hundreds of GB at the long shape), so it is excluded.
    from torch.nn.attention import SDPBackend, sdpa_kernel
    try:
        with sdpa_kernel([SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION, SDPBackend.EFFICIENT_ATTENTION]):
            sdpa_ms = timed(lambda: torch.nn.functional.scaled_dot_product_attention(qd, kd, vd))
        sdpa = {"ms": round(sdpa_ms, 4), "tflops": round(dense_flops / (sdpa_ms * 1e-3) / 1e12, 2),
                "note": "torch.nn.functional.scaled_dot_product_attention, bf16, same inputs (library kernel; "
                        "context only)"}
    except RuntimeError as e:
        sdpa = {"unavailable": str(e).splitlines()[0][:200]}
    res = {"workload": cfg.note, "shape": [B, H, N, d], "Bq": cfg.Bq, "Bk": cfg.Bk, "rows": rows,
           "torch_sdpa_bf16": sdpa}
    del qd, kd, vd, ws, out, dense_out
    torch.cuda.empty_cache()
    return res


def routing_overhead(cfg, qd, kd, tau, stream):
    """The routing stage alone on the pooled blocks of the timed inputs (paperlayer summary
    §4, "Efficient On-the-Fly Sparsification"): the running-max rule with the proxies kept on
    chip, against top-k and top-p routers that first write the proxy map to HBM. k is the
    mean number of blocks our rule keeps per query block at this tau; top-p is timed at two
    masses. CUDA events, median of 10 after 3 warm-up calls each."""
    import torch
    from block_sparse_online_b200 import solattn
    N = cfg.N
    qb, kb = solattn.solattn_pool(qd, cfg.Bq), solattn.solattn_pool(kd, cfg.Bk)
    mask = solattn.solattn_route_keep(qb, kb, N, cfg.Bq, cfg.Bk, tau)
    bits = unpack(mask, cfg.nKB)
    kk = max(1, int(round(float(bits.sum(-1).mean()))))
    smap = torch.empty(solattn.solattn_proxy_map_bytes(cfg.B, cfg.H, N, cfg.Bq, cfg.Bk) // 4, dtype=torch.float32,
                       device=qd.device)

    def timed(fn):
        return device_ms(fn, stream, reps=10, warm=3)

    ours = timed(lambda: solattn.solattn_route_keep(qb, kb, N, cfg.Bq, cfg.Bk, tau, keep_mask=mask))
    topk = timed(lambda: solattn.solattn_route_topk(qb, kb, N, cfg.Bq, cfg.Bk, kk, keep_mask=mask, proxy_map=smap))
    out = {"tau": tau, "keep_ratio": round(float(bits.mean()), 5), "ours_ms": round(ours, 4),
           "topk": {"k": kk, "ms": round(topk, 4), "slowdown_vs_ours": round(topk / ours, 2)}, "topp": [],
           "proxy_map_bytes": int(smap.numel() * 4),
           "pages": "routing 11.5x faster than top-k and 32.7x faster than top-p (paperlayer summary, section 4)"}
    for pm in (0.9, 0.99):
        t = timed(lambda: solattn.solattn_route_topp(qb, kb, N, cfg.Bq, cfg.Bk, pm, keep_mask=mask, proxy_map=smap))
        kr = float(unpack(mask, cfg.nKB).mean())
        out["topp"].append({"p": pm, "ms": round(t, 4), "keep_ratio": round(kr, 5),
                            "slowdown_vs_ours": round(t / ours, 2)})
    return out


def e2e_measure(args, cfg, q, k, v, dev, stream, world, barrier, dense_flops, elem):
    """Same metric through the host entry point: pinned host q/k/v in, host output out,
    host<->device copies inside the timed region."""
    import torch
    import torch.distributed as dist
    from block_sparse_online_b200 import solattn
    B, H, N, d = cfg.shape()
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    outh = torch.empty_like(q).pin_memory()
    kh_cnt = torch.empty((B, H), dtype=torch.int64)
    scratch = torch.empty(solattn.solattn_host_workspace_size(B, H, N, d, cfg.Bq, cfg.Bk), dtype=torch.uint8,
                          device=dev)
    e2e_steps = max(3, min(args.steps, 10))
    for _ in range(2):
        solattn.solattn_forward_host(qh, kh, vh, cfg.Bq, cfg.Bk, args.tau, args.mode, out=outh, kept_per_head=kh_cnt,
                                     scratch=scratch)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        solattn.solattn_forward_host(qh, kh, vh, cfg.Bq, cfg.Bk, args.tau, args.mode, out=outh, kept_per_head=kh_cnt,
                                     scratch=scratch)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, dev)
    return {"value": round(whole_job_rate(world, dense_flops, e2e_ms), 3), "unit": "TFLOP/s (dense-equivalent)",
            "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": 3 * elem * 2,
            "d2h_bytes_per_step": elem * 2 + B * H * 8, "steps": e2e_steps}


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        reference_arm(args, world, rank)
        return
    import torch
    import torch.distributed as dist
    from block_sparse_online_b200 import solattn, synth

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    cfg = rank_config(synth.CONFIGS[args.config], rank)
    if args.heads:
        import dataclasses
        cfg = dataclasses.replace(cfg, H=args.heads, note=cfg.note + f" [reduced to H={args.heads}]")
    B, H, N, d = cfg.shape()
    q, k, v = synth.make_inputs(cfg)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    out = torch.empty_like(qd)
    kept = torch.empty((B, H), dtype=torch.int64, device=dev)
    ws = solattn.alloc_workspace(B, H, N, d, cfg.Bq, cfg.Bk, dev)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            dist.barrier()

    # keep set of the headline call (for executed FLOPs); off the timed path
    _, _, mask = solattn.solattn_forward(qd, kd, vd, cfg.Bq, cfg.Bk, args.tau, args.mode, keep_mask=True, workspace=ws)
    st = solattn.solattn_get_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st}")
    bits = unpack(mask, cfg.nKB)
    exec_flops = executed_flops(bits, N, cfg.Bq, cfg.Bk, d)
    dense_flops = cfg.dense_flops()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    ka = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for _ in range(args.warmup):
        solattn.solattn_forward(qd, kd, vd, cfg.Bq, cfg.Bk, args.tau, args.mode, out=out, kept_per_head=kept,
                                workspace=ws)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    first_sample = clocks.mark()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        solattn.solattn_forward(qd, kd, vd, cfg.Bq, cfg.Bk, args.tau, args.mode, out=out, kept_per_head=kept,
                                workspace=ws, events=ka[i])
        ev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    last_sample = clocks.mark()
    barrier()
    clk = clocks.stop(first_sample, max(last_sample, first_sample + 1))
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
    st = solattn.solattn_get_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st}")
    ms_step = total_ms / args.steps
    step_ms = [a.elapsed_time(b) for a, b in ev]
    attn_ms = [a.elapsed_time(b) for a, b in ka]
    attn_avg = sum(attn_ms) / len(attn_ms)
    value = whole_job_rate(world, dense_flops, ms_step)
    peak_tf, peak_hbm, peak_kind = measured_peaks()
    achieved = exec_flops / (attn_avg * 1e-3) / 1e12
    trec = traffic_record()

    # end to end through the host entry point (pinned host buffers, copies inside the timed region)
    elem = B * H * N * d
    e2e = None
    if not args.no_e2e:
        e2e = e2e_measure(args, cfg, q, k, v, dev, stream, world, barrier, dense_flops, elem)

    sweep = []
    routing = None
    configs = {}
    if not args.no_sweep and rank == 0:
        for mode in ("keep_drop", "keep_correct"):
            for tau in cfg.taus:
                _, _, m = solattn.solattn_forward(qd, kd, vd, cfg.Bq, cfg.Bk, tau, mode, keep_mask=True, workspace=ws)
                b = unpack(m, cfg.nKB)
                ef = executed_flops(b, N, cfg.Bq, cfg.Bk, d)
                ms = device_ms(lambda: solattn.solattn_forward(qd, kd, vd, cfg.Bq, cfg.Bk, tau, mode, out=out,
                                                               kept_per_head=kept, workspace=ws), stream)
                sweep.append({"mode": mode, "tau": None if math.isinf(tau) else tau, "ms": round(ms, 4),
                              "keep_ratio": round(float(b.mean()), 5),
                              "exec_tflops": round(ef / (ms * 1e-3) / 1e12, 2),
                              "dense_equiv_tflops": round(dense_flops / (ms * 1e-3) / 1e12, 2)})
        # keep_correct with the token-to-block correction (pooled-key tiles on the tensor cores).
        for tau in (3.0, 6.0):
            _, _, m = solattn.solattn_forward_ex(qd, kd, vd, cfg.Bq, cfg.Bk, "keep_correct", tau=tau,
                                                 correction="token", keep_mask=True, workspace=ws)
            b = unpack(m, cfg.nKB)
            ef = executed_flops(b, N, cfg.Bq, cfg.Bk, d)
            ms = device_ms(lambda: solattn.solattn_forward_ex(qd, kd, vd, cfg.Bq, cfg.Bk, "keep_correct", tau=tau,
                                                              correction="token", out=out, kept_per_head=kept,
                                                              workspace=ws), stream)
            sweep.append({"mode": "keep_correct", "correction": "token", "tau": tau, "ms": round(ms, 4),
                          "keep_ratio": round(float(b.mean()), 5),
                          "exec_tflops": round(ef / (ms * 1e-3) / 1e12, 2),
                          "dense_equiv_tflops": round(dense_flops / (ms * 1e-3) / 1e12, 2)})
        # The pages' query-dependent Gaussian threshold (theta = mu + beta * sigma), keep_correct.
        for variant in ("exact", "diag"):
            for beta in (0.5, 1.0, 1.5):
                _, _, m = solattn.solattn_forward_gaussian(qd, kd, vd, cfg.Bq, cfg.Bk, beta, variant, "keep_correct",
                                                           keep_mask=True, workspace=ws)
                b = unpack(m, cfg.nKB)
                ef = executed_flops(b, N, cfg.Bq, cfg.Bk, d)
                ms = device_ms(lambda: solattn.solattn_forward_gaussian(qd, kd, vd, cfg.Bq, cfg.Bk, beta, variant,
                                                                        "keep_correct", out=out, kept_per_head=kept,
                                                                        workspace=ws), stream)
                sweep.append({"mode": "keep_correct", "threshold": f"gaussian-{variant}", "beta": beta,
                              "ms": round(ms, 4), "keep_ratio": round(float(b.mean()), 5),
                              "exec_tflops": round(ef / (ms * 1e-3) / 1e12, 2),
                              "dense_equiv_tflops": round(dense_flops / (ms * 1e-3) / 1e12, 2)})
        ms = device_ms(lambda: solattn.solattn_forward(qd, kd, vd, cfg.Bq, cfg.Bk, 0.0, "dense", out=out,
                                                       kept_per_head=kept, workspace=ws), stream, reps=3)
        sweep.append({"mode": "dense", "tau": None, "ms": round(ms, 4), "keep_ratio": 1.0,
                      "exec_tflops": round(dense_flops / (ms * 1e-3) / 1e12, 2),
                      "dense_equiv_tflops": round(dense_flops / (ms * 1e-3) / 1e12, 2)})
        routing = routing_overhead(cfg, qd, kd, args.tau, stream)
        peak_tf0, _, _ = measured_peaks()
        for name in (args.all_configs.split(",") if args.all_configs else []):
            configs[name] = config_sweep(name, dev, stream, peak_tf0)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, desc, _, _ = cpu_oracle_rate(cfg, q, k, v, args.tau, args.mode, args.cpu_seconds)
        cpu = {"value": rate, "unit": "TFLOP/s (dense-equivalent)", "cores": cores(), "kind": "oracle",
               "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_dict(args, cfg, world),
            "keep_ratio": round(float(bits.mean()), 5),
            "exec_tflops": round(exec_flops / (ms_step * 1e-3) / 1e12, 2),
            "step_ms_median": round(statistics.median(step_ms), 4),
            "attn_kernel_ms": round(attn_avg, 4),
            "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak_tf, "unit": "TFLOP/s",
                         "frac": round(achieved / peak_tf, 4), "peak_source": f"{peak_kind} bf16 dense (burst)",
                         "traffic": None if trec is None else trec["dram_bytes_per_launch"],
                         "kernel": "solattn_fwd_kernel (executed FLOPs per launch / CUDA-event duration)"},
            "e2e": e2e,
            # per step: pool_kernel (block means and the fp16 copy of V; the copy alone in
            # dense mode), plan_kernel (keep modes) and solattn_fwd_kernel
            "gpu_launches": args.steps * (2 if args.mode == "dense" else 3),
            "clocks": clk,
            "cpu_baseline": cpu,
            "sweep": sweep,
            "routing_overhead": routing,
            "configs": configs,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
