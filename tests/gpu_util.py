"""Helpers shared by the GPU parity tests.

Inputs come from ``sikv_inputs`` (seeded, synthetic); expected values come
from ``oracle`` run on the same host bytes.  Nothing computed by the CUDA path
is ever fed to the oracle.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

import long_context_decode_sikv_b200 as sk
import oracle
import sikv_inputs as gen

# Tolerances of the decode path (bf16 I/O).
SCORE_RTOL = 1e-4          # |gpu - oracle| <= 1e-4 * condition scale of the score sum
TIE_BAND = 1e-5            # selection may differ only among scores this close (relative) to the k-th
ATTN_ATOL_BF16, ATTN_RTOL_BF16 = 2e-2, 1e-2
ATTN_ATOL_F32, ATTN_RTOL_F32 = 1e-5, 1e-5


def device() -> torch.device:
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    return torch.device("cuda:0")


def attn_tol(dtype: str):
    return (ATTN_ATOL_BF16, ATTN_RTOL_BF16) if dtype == "bf16" else (ATTN_ATOL_F32, ATTN_RTOL_F32)


@dataclass
class OracleHead:
    K: np.ndarray
    V: np.ndarray
    mu: np.ndarray
    code: np.ndarray
    cent: np.ndarray
    counts: np.ndarray


def oracle_head(w: gen.Workload, bt: gen.Batch, b: int, h: int) -> OracleHead:
    n = w.seq_lens[b]
    K = gen.storage_to_f64(bt.K[b, h, :n], w.dtype)
    V = gen.storage_to_f64(bt.V[b, h, :n], w.dtype)
    mu, code, cent, counts = oracle.encode_keys(K, w.num_sinks)
    return OracleHead(K, V, mu, code, cent, counts)


def oracle_queries(w: gen.Workload, bt: gen.Batch, step: int, b: int, h: int) -> np.ndarray:
    g = w.group
    return gen.storage_to_f64(bt.q[step][b, h * g:(h + 1) * g], w.dtype)


class DeviceWorkload:
    """A workload uploaded to cuda:0 with its cache and workspaces."""

    def __init__(self, w: gen.Workload, steps=(0,), bt: gen.Batch | None = None, decode_path: int = 0):
        dev = device()
        self.w = w
        self.bt = bt if bt is not None else gen.make_batch(w, steps)
        self.p = sk.make_params(w.dtype, w.batch, w.num_q_heads, w.num_kv_heads, w.max_seq_len, w.num_sinks,
                                w.max_topk, decode_path=decode_path)
        self.K = sk.to_device(self.bt.K, w.dtype, dev)
        self.V = sk.to_device(self.bt.V, w.dtype, dev)
        self.q = {s: sk.to_device(self.bt.q[s], w.dtype, dev) for s in self.bt.q}
        self.seq_lens = torch.from_numpy(self.bt.seq_lens).to(dev)
        self.k = torch.from_numpy(self.bt.topk).to(dev)
        self.cache = sk.SikvCache(self.p, self.K, self.V, self.seq_lens)
        self.dev = dev

    def encode(self):
        self.cache.encode()
        torch.cuda.synchronize()
        assert self.cache.ws_encode.check() == 0

    def decode(self, step=0):
        tdt = self.p.torch_dtype
        B, Hq, Hkv, N = self.w.batch, self.w.num_q_heads, self.w.num_kv_heads, self.w.max_seq_len
        out = torch.empty((B, Hq, 128), dtype=tdt, device=self.dev)
        idx = torch.full((B, Hkv, self.w.max_topk), -7, dtype=torch.int32, device=self.dev)
        sc = torch.full((B, Hkv, N), 12345.0, dtype=torch.float32, device=self.dev)
        self.cache.decode(self.q[step], self.k, out=out, idx_out=idx, scores_out=sc)
        torch.cuda.synchronize()
        assert self.cache.ws_decode.check() == 0
        return out, idx, sc


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_selection(gpu_idx: np.ndarray, want_idx: np.ndarray, oracle_scores: np.ndarray, cond: np.ndarray, k: int):
    """Selected sets equal, except tokens whose oracle score ties the k-th within the band."""
    got, want = set(gpu_idx.tolist()), set(want_idx.tolist())
    assert len(got) == len(gpu_idx) == k, (len(got), k)
    diff = got ^ want
    if not diff:
        return 0
    kth = float(np.min(oracle_scores[want_idx])) if k else 0.0
    for t in diff:
        band = TIE_BAND * float(cond[t])
        assert abs(float(oracle_scores[t]) - kth) <= band, (t, oracle_scores[t], kth, band)
    return len(diff)
