"""fp64 CPU oracle for the Sol-Attn forward operator: test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It shares no code with the CUDA path.
"""
from .solattn_ref import (MODES, forward, gaussian_threshold, keep_sets, keep_sets_gaussian,  # noqa: F401
                          keep_sets_topk, keep_sets_topp, kept_per_head, pool, proxy, sample_qblocks, topk_keep,
                          topp_keep, valid_counts, visit_order)
