"""The dense comparison baselines (not the method) against the oracle's plain
definitions: full-precision scoring and dense decode attention."""

from dataclasses import replace

import numpy as np
import pytest
import torch

import long_context_decode_sikv_b200 as sk
import oracle
import sikv_inputs as gen
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

SHAPES = {
    "gqa4-ragged": lambda: gen.small(3, n=5000, batch=3, num_q_heads=8, num_kv_heads=2),
    "gqa5": lambda: gen.small(1, n=3100, batch=2, num_q_heads=10, num_kv_heads=2),
    "gqa8": lambda: gen.small(2, n=2600, batch=1, num_q_heads=16, num_kv_heads=2),
    "f32-one-head": lambda: gen.small(0, n=4100),
    "short": lambda: replace(gen.small(1, n=300, batch=2, num_q_heads=4, num_kv_heads=1), seq_lens=(40, 300)),
}


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_dense_baselines_match_oracle(name):
    w = SHAPES[name]()
    dw = gu.DeviceWorkload(w)
    p, dev, g = dw.p, dw.dev, w.group
    sc = torch.full((w.batch, w.num_kv_heads, w.max_seq_len), 12345.0, dtype=torch.float32, device=dev)
    sk.sikv_dense_score(p, dw.q[0], dw.K, dw.seq_lens, sc).check()
    out = torch.empty_like(dw.q[0])
    sk.sikv_dense_attn(p, dw.q[0], dw.K, dw.V, dw.seq_lens, out).check()
    torch.cuda.synchronize()
    sc = sc.cpu().numpy().astype(np.float64)
    out = gu.to_f64(out)
    atol, rtol = gu.attn_tol(w.dtype)
    for b in range(w.batch):
        n = w.seq_lens[b]
        for h in range(w.num_kv_heads):
            K = gen.storage_to_f64(dw.bt.K[b, h, :n], w.dtype)
            V = gen.storage_to_f64(dw.bt.V[b, h, :n], w.dtype)
            q = gu.oracle_queries(w, dw.bt, 0, b, h)
            want = oracle.dense_scores(q, K, w.num_sinks)
            s = min(w.num_sinks, n)
            assert np.all(np.isneginf(sc[b, h, :s]))
            cond = np.abs(K[s:] * q.sum(axis=0)[None, :]).sum(axis=1)
            assert np.all(np.abs(sc[b, h, s:n] - want[s:]) <= 1e-5 * cond + 1e-30), (name, b, h)
            assert np.all(sc[b, h, n:] == 12345.0)
            o = oracle.dense_attention(q, K, V)
            assert np.allclose(out[b, h * g:(h + 1) * g], o, atol=atol, rtol=rtol), (name, b, h)
