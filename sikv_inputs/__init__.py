"""Seeded synthetic inputs for the Self-Indexing KVCache decode hot path.

This module holds the workload shapes and the random draws that both the CUDA
path and the CPU oracle consume.  It contains none of the method's arithmetic
(no channel mean, no sign code, no codebook, no scoring, no selection, no
attention): only Gaussian draws, a sinusoidal drift, planted "needle" rows and
the round-to-nearest-even conversion to the storage dtype.

Workloads stand in for the pages' evaluation (RULER 32K at 7.5 % token
retention and LongBench on Llama3.1-8B / Qwen2.5-14B, "Self-Indexing KVCache:
Predicting Sparse Attention from Compressed Keys", technical summary §4), which
needs datasets and trained weights that are not available: the head shapes are
Llama-3-8B's (32 query heads, 8 KV heads, head_dim 128) and the retention is the
pages' 7.5 %.

Recipe for one (sequence b, KV head h), all draws from
``numpy.random.default_rng(SeedSequence([seed, b, h, role, extra]))``:

* keys: per-channel mean ``m_c ~ N(0, 1.5)`` plus ``N(0, 1)`` noise per token
  (the second argument of N is a standard deviation throughout); four channels
  drawn per head are outliers whose per-token deviation is multiplied by 8;
  with ``drift`` the mean moves as ``m_c + 0.1 sin(2 pi t / 8192)`` (same phase
  on every channel);
* values: ``N(0, 1)``;
* queries of the G query heads of the group, at decode step s:
  ``0.8 * unit(mean over all tokens of the key rows) + N(0, 0.3)`` per head;
* needles: ``needles_per_head`` rows at positions drawn uniformly without
  replacement from ``[num_sinks, N)`` are overwritten with ``3 * q``, where q
  is the query that selects for the KV head at step 0: the single query when
  the group has one head, the sum of the group's queries otherwise (a GQA group
  shares one selection scored with its summed query);
* everything is rounded to the storage dtype (fp32 or bf16, round to nearest
  even) before use, and the rounded bytes are what both sides read.
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np

ROLE_KEYS = 1
ROLE_VALUES = 2
ROLE_QUERY = 3
ROLE_NEEDLES = 4
ROLE_LENGTHS = 5
ROLE_SCORES = 6
ROLE_INDICES = 7
ROLE_KMEANS_INIT = 8


# ----------------------------------------------------------------------------
# storage dtype helpers (rounding only)
# ----------------------------------------------------------------------------

def f32_to_bf16_bits(x) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    u = np.array(x, dtype=np.float32, copy=True, order="C").view(np.uint32)
    bias = u >> 16
    bias &= 1
    bias += 0x7FFF
    u += bias
    u >>= 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_storage(x, dtype: str) -> np.ndarray:
    """Round to the storage dtype; returns float32 array (f32) or uint16 bits (bf16)."""
    x32 = np.asarray(x, dtype=np.float32)
    if dtype == "f32":
        return np.ascontiguousarray(x32)
    if dtype == "bf16":
        return f32_to_bf16_bits(x32)
    raise ValueError(f"unknown dtype {dtype!r}")


def storage_to_f64(a, dtype: str) -> np.ndarray:
    """Exact value of stored elements as float64."""
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    if dtype == "bf16":
        return bf16_bits_to_f32(a).astype(np.float64)
    raise ValueError(f"unknown dtype {dtype!r}")


def storage_np_dtype(dtype: str):
    return np.float32 if dtype == "f32" else np.uint16


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

@dataclass(frozen=True)
class Workload:
    """Shape and generator settings of one decode workload."""

    name: str
    dtype: str                 # "f32" or "bf16" for K, V, q and out
    batch: int
    num_q_heads: int
    num_kv_heads: int
    seq_lens: tuple            # N_b per sequence
    topk: tuple                # k_b per sequence (non-sink tokens selected)
    num_sinks: int = 64
    head_dim: int = 128
    needles_per_head: int = 8
    drift: bool = False
    steps: int = 1             # decode steps, queries redrawn each step
    seed: int = 0
    max_seq_len_override: int = 0

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def max_seq_len(self) -> int:
        return max(self.max_seq_len_override, max(self.seq_lens))

    @property
    def max_topk(self) -> int:
        return max(max(self.topk), 1)

    @property
    def segments(self) -> int:
        return self.batch * self.num_kv_heads


def retention_topk(n: int, frac: float = 0.075) -> int:
    """k = ceil(frac * N); 7.5 % retention of a 32K context gives 2458."""
    return int(math.ceil(frac * n - 1e-9))


def _ragged_lengths(seed: int, batch: int, lo: int, hi: int) -> tuple:
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0, 0, ROLE_LENGTHS, 0]))
    return tuple(int(v) for v in rng.integers(lo, hi + 1, size=batch))


def config(cfg: int) -> Workload:
    """The five configurations of the decode hot path (index 0..4)."""
    if cfg == 0:
        return Workload("tiny-1head-f32-N4096", "f32", 1, 1, 1, (4096,), (256,),
                        needles_per_head=8, seed=0)
    if cfg == 1:
        n = 32768
        return Workload("llama3-8b-layer-bf16-N32768", "bf16", 1, 32, 8, (n,),
                        (retention_topk(n),), needles_per_head=32, seed=1)
    if cfg == 2:
        n = 131072
        return Workload("long-context-bf16-B4-N131072", "bf16", 4, 32, 8, (n,) * 4,
                        (2048,) * 4, needles_per_head=32, drift=True, steps=256, seed=2)
    if cfg == 3:
        lens = _ragged_lengths(3, 32, 8192, 32768)
        return Workload("ragged-bf16-B32-N8K-32K", "bf16", 32, 32, 8, lens,
                        tuple(retention_topk(n) for n in lens), needles_per_head=32, seed=3)
    if cfg == 4:
        n = 524288
        return Workload("extreme-bf16-B1-N524288", "bf16", 1, 32, 8, (n,), (4096,),
                        needles_per_head=32, drift=True, seed=4)
    raise ValueError(f"no config {cfg}")


def small(cfg: int, n: int = 2048 + 37, k: int | None = None, batch: int | None = None,
          num_q_heads: int | None = None, num_kv_heads: int | None = None) -> Workload:
    """A config's generator and head layout at a size the oracle finishes in seconds."""
    w = config(cfg)
    b = batch if batch is not None else min(w.batch, 2)
    hq = num_q_heads if num_q_heads is not None else w.num_q_heads
    hkv = num_kv_heads if num_kv_heads is not None else w.num_kv_heads
    if cfg == 3:
        lens = tuple(int(n * (0.5 + 0.5 * i / max(b - 1, 1))) for i in range(b))
    else:
        lens = (n,) * b
    if k is None:
        ks = tuple(max(1, retention_topk(x)) for x in lens)
    else:
        ks = (k,) * b
    ks = tuple(min(kk, max(x - w.num_sinks, 0)) for kk, x in zip(ks, lens))
    return replace(w, name=w.name + f"-small{n}", batch=b, num_q_heads=hq, num_kv_heads=hkv,
                   seq_lens=lens, topk=ks, needles_per_head=min(w.needles_per_head, 8), steps=2)


# ----------------------------------------------------------------------------
# per-head generation
# ----------------------------------------------------------------------------

def _rng(w: Workload, b: int, h: int, role: int, extra: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([w.seed, b, h, role, extra]))


@dataclass
class HeadInputs:
    """Stored bytes of one (sequence, KV head): K and V rows plus the step queries."""

    keys: np.ndarray           # [N][D] storage dtype
    values: np.ndarray         # [N][D] storage dtype
    mean_dir: np.ndarray       # [D] float64 unit vector used for the queries
    needle_pos: np.ndarray     # positions of the planted rows
    queries: dict = field(default_factory=dict)   # step -> [G][D] storage dtype


def _head_keys_f32(w: Workload, b: int, h: int, n: int) -> np.ndarray:
    d = w.head_dim
    rng = _rng(w, b, h, ROLE_KEYS)
    mean = rng.normal(0.0, 1.5, size=d)
    outliers = rng.choice(d, size=min(4, d), replace=False)
    keys = rng.standard_normal((n, d), dtype=np.float32)
    keys[:, outliers] *= np.float32(8.0)
    if w.drift:
        t = np.arange(n, dtype=np.float64)
        keys += (0.1 * np.sin(2.0 * np.pi * t / 8192.0)).astype(np.float32)[:, None]
    keys += mean[None, :].astype(np.float32)
    return keys


def head_queries(w: Workload, b: int, h: int, step: int, mean_dir: np.ndarray) -> np.ndarray:
    rng = _rng(w, b, h, ROLE_QUERY, step)
    q = 0.8 * mean_dir[None, :] + rng.normal(0.0, 0.3, size=(w.group, w.head_dim))
    return to_storage(q, w.dtype)


def head_inputs(w: Workload, b: int, h: int, steps=(0,)) -> HeadInputs:
    """Generate the stored K, V and queries of sequence b, KV head h."""
    n = w.seq_lens[b]
    keys = to_storage(_head_keys_f32(w, b, h, n), w.dtype)
    kf = storage_to_f64(keys, w.dtype)
    m = kf.mean(axis=0) if n > 0 else np.zeros(w.head_dim)
    nrm = float(np.linalg.norm(m))
    mean_dir = m / nrm if nrm > 0 else np.zeros_like(m)
    q0 = head_queries(w, b, h, 0, mean_dir)
    span = n - w.num_sinks
    npos = min(w.needles_per_head, max(span, 0))
    rng = _rng(w, b, h, ROLE_NEEDLES)
    pos = np.sort(rng.choice(span, size=npos, replace=False) + w.num_sinks) if npos > 0 \
        else np.zeros(0, dtype=np.int64)
    if npos > 0:
        needle = 3.0 * storage_to_f64(q0, w.dtype).sum(axis=0)
        keys[pos] = to_storage(needle[None, :], w.dtype)
    vals = to_storage(_rng(w, b, h, ROLE_VALUES).standard_normal((n, w.head_dim),
                                                                 dtype=np.float32), w.dtype)
    qs = {s: (q0 if s == 0 else head_queries(w, b, h, s, mean_dir)) for s in steps}
    return HeadInputs(keys, vals, mean_dir, pos, qs)


# ----------------------------------------------------------------------------
# whole-workload tensors (host, storage dtype)
# ----------------------------------------------------------------------------

@dataclass
class Batch:
    """Host arrays of a whole workload in the library's layouts."""

    w: Workload
    K: np.ndarray              # [B][Hkv][Nmax][D]
    V: np.ndarray              # [B][Hkv][Nmax][D]
    q: dict                    # step -> [B][Hq][D]
    seq_lens: np.ndarray       # int32 [B]
    topk: np.ndarray           # int32 [B]
    mean_dirs: np.ndarray      # [B][Hkv][D] float64
    needles: dict              # (b, h) -> positions


def make_batch(w: Workload, steps=(0,), threads: int | None = None) -> Batch:
    """All heads of a workload; rows past N_b are zero padding that is never read."""
    nmax, d = w.max_seq_len, w.head_dim
    npd = storage_np_dtype(w.dtype)
    K = np.zeros((w.batch, w.num_kv_heads, nmax, d), dtype=npd)
    V = np.zeros_like(K)
    q = {s: np.zeros((w.batch, w.num_q_heads, d), dtype=npd) for s in steps}
    dirs = np.zeros((w.batch, w.num_kv_heads, d))
    needles = {}

    def one(bh):
        b, h = bh
        hi = head_inputs(w, b, h, steps)
        n = w.seq_lens[b]
        K[b, h, :n] = hi.keys
        V[b, h, :n] = hi.values
        dirs[b, h] = hi.mean_dir
        needles[(b, h)] = hi.needle_pos
        for s in steps:
            q[s][b, h * w.group:(h + 1) * w.group] = hi.queries[s]

    jobs = [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]
    nthreads = threads or min(len(jobs), os.cpu_count() or 1, 32)
    if nthreads > 1:
        with ThreadPoolExecutor(nthreads) as ex:
            list(ex.map(one, jobs))
    else:
        for j in jobs:
            one(j)
    return Batch(w, K, V, q, np.asarray(w.seq_lens, dtype=np.int32),
                 np.asarray(w.topk, dtype=np.int32), dirs, needles)


def step_queries(w: Workload, step: int, mean_dirs: np.ndarray) -> np.ndarray:
    """Queries [B][Hq][D] of one decode step (redrawn each step)."""
    npd = storage_np_dtype(w.dtype)
    q = np.zeros((w.batch, w.num_q_heads, w.head_dim), dtype=npd)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            q[b, h * w.group:(h + 1) * w.group] = head_queries(w, b, h, step, mean_dirs[b, h])
    return q


# ----------------------------------------------------------------------------
# direct inputs for the selection and attention steps
# ----------------------------------------------------------------------------

def random_scores(seed: int, segments: int, nmax: int, ties: bool = True) -> np.ndarray:
    """fp32 score rows [segments][nmax] with planted exact ties, +0.0 and -0.0."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0, 0, ROLE_SCORES, 0]))
    s = rng.normal(0.0, 40.0, size=(segments, nmax)).astype(np.float32)
    if ties and nmax > 8:
        # a coarse grid makes many exact duplicates
        coarse = rng.random((segments, nmax)) < 0.3
        s[coarse] = np.round(s[coarse] / 8.0).astype(np.float32) * np.float32(8.0)
        z = rng.random((segments, nmax))
        s[z < 0.01] = np.float32(0.0)
        s[(z >= 0.01) & (z < 0.02)] = np.float32(-0.0)
    return s


def random_indices(seed: int, seq_len: int, num_sinks: int, k: int) -> np.ndarray:
    """k distinct token positions in [num_sinks, seq_len), in random order."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, seq_len, k, ROLE_INDICES, 0]))
    return (rng.choice(seq_len - num_sinks, size=k, replace=False) + num_sinks).astype(np.int32)


def kmeans_init(w: Workload, seq_lens, clusters: int = 16) -> np.ndarray:
    """Starting tokens of the k-means baseline: for every (sequence b, KV head
    h), ``clusters`` distinct positions drawn uniformly from [num_sinks,
    seq_lens[b]), in random order; int32 [B][Hkv][clusters]."""
    out = np.zeros((w.batch, w.num_kv_heads, clusters), dtype=np.int32)
    for b in range(w.batch):
        n = int(seq_lens[b]) - w.num_sinks
        if n < clusters:
            raise ValueError(f"sequence {b} has {n} non-sink tokens, fewer than {clusters}")
        for h in range(w.num_kv_heads):
            out[b, h] = _rng(w, b, h, ROLE_KMEANS_INIT).choice(n, size=clusters, replace=False) + w.num_sinks
    return out
