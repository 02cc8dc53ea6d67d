"""Parity at the full workload sizes, in the launch configuration bench.py
times (one sikv_decode per step), on sampled (sequence, KV head) segments that
the oracle recomputes one by one.  Also checks properties that hold at any
size on every segment: ascending, in-range, duplicate-free selections of
exactly k tokens, and finite outputs.
"""

import numpy as np
import pytest
import torch

import oracle
import sikv_inputs as gen
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

SAMPLES = {0: [(0, 0)], 1: [(0, 0), (0, 7)], 2: [(0, 0), (3, 5)], 3: [(0, 1), (17, 6), (31, 3)], 4: [(0, 2)]}


@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4])
def test_full_size_decode_matches_oracle_on_samples(cfg):
    w = gen.config(cfg)
    dw = gu.DeviceWorkload(w)
    dw.encode()
    out, idx, sc = dw.decode()
    # the call bench.py times (no selection or score outputs) gives the same bytes
    bench_out = torch.empty_like(out)
    dw.cache.decode(dw.q[0], dw.k, out=bench_out)
    torch.cuda.synchronize()
    assert dw.cache.ws_decode.check() == 0
    assert torch.equal(bench_out, out)
    idx = idx.cpu().numpy()
    out = gu.to_f64(out)
    assert np.isfinite(out).all()
    for b in range(w.batch):
        n, k = w.seq_lens[b], w.topk[b]
        sel = idx[b, :, :k]
        assert np.all(np.diff(sel, axis=1) > 0)
        assert sel.min() >= w.num_sinks and sel.max() < n
        assert np.all(idx[b, :, k:] == -1)
    for (b, h) in SAMPLES[cfg]:
        n, k = w.seq_lens[b], w.topk[b]
        o = gu.oracle_head(w, dw.bt, b, h)
        mu_gpu = dw.cache.mu[b, h].cpu().numpy()
        assert np.array_equal(mu_gpu.view(np.uint32), o.mu.view(np.uint32))
        codes = dw.cache.codes[b, h, :n].cpu().numpy()
        assert np.array_equal(codes, oracle.pack_codes(o.code))
        q = gu.oracle_queries(w, dw.bt, 0, b, h)
        o_out, o_idx, o_sc, cond = oracle.decode_step(q, o.K, o.V, o.mu, o.cent, o.code, k, w.num_sinks)
        s = w.num_sinks
        got_sc = sc[b, h, :n].cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got_sc[s:] - o_sc[s:]) <= gu.SCORE_RTOL * cond[s:])
        gu.check_selection(idx[b, h, :k], o_idx, o_sc, cond, k)
        needles = set(dw.bt.needles[(b, h)].tolist())
        assert needles <= set(o_idx.tolist())
        assert needles <= set(idx[b, h, :k].tolist())
        g = out[b, h * w.group:(h + 1) * w.group]
        atol, rtol = gu.attn_tol(w.dtype)
        assert np.allclose(g, o_out, atol=atol, rtol=rtol), (cfg, b, h, float(np.abs(g - o_out).max()))
        if cfg == 0:
            # the tiny fp32 workload is checked on every element: scores of
            # every token, the selected set, and the output row
            assert len(needles) == w.needles_per_head
    del dw
    torch.cuda.empty_cache()


def test_full_size_decode_qv_matches_oracle_on_samples():
    """2-bit values at the long-context workload (4 x 128K), sampled segments."""
    w = gen.config(2)
    dw = gu.DeviceWorkload(w)
    dw.encode()
    dw.cache.quantize_values()
    out = torch.empty((w.batch, w.num_q_heads, 128), dtype=dw.p.torch_dtype, device=dw.dev)
    dw.cache.decode_qv(dw.q[0], dw.k, out=out)
    torch.cuda.synchronize()
    assert dw.cache.ws_decode.check() == 0 and dw.cache.ws_encode.check() == 0
    out = gu.to_f64(out)
    assert np.isfinite(out).all()
    for (b, h) in SAMPLES[2]:
        k = w.topk[b]
        o = gu.oracle_head(w, dw.bt, b, h)
        q = gu.oracle_queries(w, dw.bt, 0, b, h)
        vq = dw.cache.vq[b, h, :w.seq_lens[b]].cpu().numpy()
        packed = oracle.quantize_values(o.V)
        assert np.array_equal(vq, packed)
        o_out, _, _, _ = oracle.decode_step_qv(q, o.K, o.V, packed, o.mu, o.cent, o.code, k, w.num_sinks)
        g = out[b, h * w.group:(h + 1) * w.group]
        assert np.allclose(g, o_out, atol=2e-2, rtol=1e-2), (b, h, float(np.abs(g - o_out).max()))
    del dw
    torch.cuda.empty_cache()
