"""Oracle jobs that test processes hand to spawned workers.

Kept apart from the GPU test modules so that a worker imports only numpy, the
oracle and the seeded input generator (no torch, no CUDA).
"""

from __future__ import annotations

import oracle
import sikv_inputs as gen


def encode_segment(cfg: int, b: int, h: int):
    """Oracle prefill encode of segment (b, h) of workload ``cfg``, regenerated
    from the seeded inputs.  Returns (b, h, mu, code, centroids)."""
    w = gen.config(cfg)
    hi = gen.head_inputs(w, b, h)
    K = gen.storage_to_f64(hi.keys, w.dtype)
    mu, code, cent, _ = oracle.encode_keys(K, w.num_sinks)
    return b, h, mu, code, cent
