"""Parity over the long-context workload's consecutive decode steps.

The bench times 256 decode steps of the 4 x 128K workload with the queries
redrawn every step.  Here the same 256 steps run through sikv_decode, and the
oracle recomputes:

* steps 0, 1 and 255 on eight (sequence, KV head) segments, two per sequence;
* two more segments on every step, drawn by a seeded generator from all 32.

Each check covers every scored token's score, the selected set (identical up
to ties within the band of the k-th score), needle recall and the attention
output of the group's heads.  The oracle's prefill encodes run in spawned
worker processes while the GPU works.
"""

from __future__ import annotations

import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np
import pytest
import torch

import oracle
import sikv_inputs as gen
from tests import gpu_util as gu
from tests import oracle_jobs

pytestmark = pytest.mark.gpu

CFG = 2
STEPS = 256
FULL_STEPS = (0, 1, STEPS - 1)
FULL_SEGMENTS = [(0, 0), (0, 5), (1, 2), (1, 7), (2, 1), (2, 4), (3, 3), (3, 6)]


def _random_segments(w):
    rng = np.random.default_rng(np.random.SeedSequence([CFG, 0, 0, 99, 0]))
    segs = [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]
    return {s: [segs[i] for i in rng.choice(len(segs), size=2, replace=False)] for s in range(STEPS)}


def test_long_context_steps_match_oracle():
    w = gen.config(CFG)
    draws = _random_segments(w)
    wanted = sorted(set(FULL_SEGMENTS) | {bh for v in draws.values() for bh in v})
    workers = max(1, min(16, (os.cpu_count() or 2) - 1))
    pool = ProcessPoolExecutor(workers, mp_context=mp.get_context("spawn"))
    futures = [pool.submit(oracle_jobs.encode_segment, CFG, b, h) for (b, h) in wanted]

    dw = gu.DeviceWorkload(w, steps=tuple(range(STEPS)))
    dw.encode()
    B, Hq, Hkv, N, kmax = w.batch, w.num_q_heads, w.num_kv_heads, w.max_seq_len, w.max_topk
    outs = torch.empty((STEPS, B, Hq, 128), dtype=dw.p.torch_dtype, device=dw.dev)
    idxs = torch.full((STEPS, B, Hkv, kmax), -7, dtype=torch.int32, device=dw.dev)
    sc = torch.empty((B, Hkv, N), dtype=torch.float32, device=dw.dev)
    kept_scores = {}
    for s in range(STEPS):
        dw.cache.decode(dw.q[s], dw.k, out=outs[s], idx_out=idxs[s], scores_out=sc)
        segs = set(draws[s]) | (set(FULL_SEGMENTS) if s in FULL_STEPS else set())
        for (b, h) in segs:
            kept_scores[(s, b, h)] = sc[b, h].clone()
    torch.cuda.synchronize()
    assert dw.cache.ws_decode.check() == 0
    outs = gu.to_f64(outs)
    idxs = idxs.cpu().numpy()
    kept_scores = {key: v.cpu().numpy().astype(np.float64) for key, v in kept_scores.items()}
    mu_gpu = dw.cache.mu.cpu().numpy()
    enc = {}
    for f in futures:
        b, h, mu, code, cent = f.result()
        enc[(b, h)] = (mu, code, cent)
        assert np.array_equal(mu_gpu[b, h].view(np.uint32), mu.view(np.uint32)), (b, h)
        assert np.array_equal(dw.cache.codes[b, h].cpu().numpy(), oracle.pack_codes(code)), (b, h)
    pool.shutdown()

    S = w.num_sinks
    checked = 0
    by_segment = {}
    for (s, b, h) in kept_scores:
        by_segment.setdefault((b, h), []).append(s)
    for (b, h), steps in sorted(by_segment.items()):
        n, k = w.seq_lens[b], w.topk[b]
        K = gen.storage_to_f64(dw.bt.K[b, h, :n], w.dtype)
        V = gen.storage_to_f64(dw.bt.V[b, h, :n], w.dtype)
        mu, code, cent = enc[(b, h)]
        for s in sorted(steps):
            got_sc = kept_scores[(s, b, h)]
            q = gu.oracle_queries(w, dw.bt, s, b, h)
            o_out, o_idx, o_sc, cond = oracle.decode_step(q, K, V, mu, cent, code, k, S)
            assert np.all(np.abs(got_sc[S:n] - o_sc[S:]) <= gu.SCORE_RTOL * cond[S:]), (s, b, h)
            sel = idxs[s, b, h, :k]
            assert np.all(np.diff(sel) > 0) and np.all(idxs[s, b, h, k:] == -1), (s, b, h)
            gu.check_selection(sel, o_idx, o_sc, cond, k)
            if s == 0:
                needles = set(dw.bt.needles[(b, h)].tolist())
                assert needles <= set(o_idx.tolist()) and needles <= set(sel.tolist()), (b, h)
            g = outs[s, b, h * w.group:(h + 1) * w.group]
            assert np.allclose(g, o_out, atol=gu.ATTN_ATOL_BF16, rtol=gu.ATTN_RTOL_BF16), \
                (s, b, h, float(np.abs(g - o_out).max()))
            checked += 1
    assert checked == len(kept_scores) >= STEPS * 2
    del dw
    torch.cuda.empty_cache()
