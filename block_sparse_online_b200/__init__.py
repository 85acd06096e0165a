"""block_sparse_online_b200: a B200-native (sm_100a) Sol-Attn forward operator.

The compute path is ``libsolattn.so`` (hand-written CUDA for sm_100a behind a
C ABI, declared in ``include/solattn.h``); ``block_sparse_online_b200.solattn``
is its thin ctypes binding. ``synth`` makes seeded synthetic inputs.
"""
__all__ = ["synth", "solattn"]
