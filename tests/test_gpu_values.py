"""2-bit values (sikv_quantize_values, sikv_decode_qv, sikv_sparse_attn_qv)
against the oracle.

The quantized rows are byte work decided in fp32 on both sides, so they must
match the oracle bit for bit; rows past a sequence's end are left alone.  A
decode step reading the selected tokens' values from those rows (sinks keep
their full-precision rows) must select what the oracle selects and produce
its output within the attention tolerance, in the single-launch kernel and
in the composed attention kernel.
"""

from dataclasses import replace

import numpy as np
import pytest
import torch

import long_context_decode_sikv_b200 as sk
import oracle
import sikv_inputs as gen
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_quantized_rows_match_oracle(dtype):
    base = gen.small(3, n=1500, batch=3, num_q_heads=8, num_kv_heads=2)
    w = replace(base, dtype=dtype, name=base.name + "-qv")
    bt = gen.make_batch(w)
    dev = gu.device()
    p = sk.make_params(w.dtype, w.batch, w.num_q_heads, w.num_kv_heads, w.max_seq_len, w.num_sinks, w.max_topk)
    V = sk.to_device(bt.V, w.dtype, dev)
    vq = torch.full((w.batch, w.num_kv_heads, w.max_seq_len, 48), 0xCD, dtype=torch.uint8, device=dev)
    ws = sk.sikv_quantize_values(p, V, torch.tensor(w.seq_lens, dtype=torch.int32, device=dev), vq)
    torch.cuda.synchronize()
    assert ws.check() == 0
    got = vq.cpu().numpy()
    for b in range(w.batch):
        n = w.seq_lens[b]
        for h in range(w.num_kv_heads):
            want = oracle.quantize_values(gen.storage_to_f64(bt.V[b, h, :n], w.dtype))
            assert np.array_equal(got[b, h, :n], want), (b, h)
            assert np.all(got[b, h, n:] == 0xCD)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_qv_matches_oracle(dtype):
    base = gen.small(3, n=3000, batch=3, num_q_heads=8, num_kv_heads=2)
    w = replace(base, dtype=dtype, name=base.name + "-qv-decode")
    dw = gu.DeviceWorkload(w)
    dw.encode()
    dw.cache.quantize_values()
    B, Hq, Hkv = w.batch, w.num_q_heads, w.num_kv_heads
    out = torch.empty((B, Hq, 128), dtype=dw.p.torch_dtype, device=dw.dev)
    idx = torch.full((B, Hkv, w.max_topk), -7, dtype=torch.int32, device=dw.dev)
    dw.cache.decode_qv(dw.q[0], dw.k, out=out, idx_out=idx)
    torch.cuda.synchronize()
    assert dw.cache.ws_decode.check() == 0 and dw.cache.ws_encode.check() == 0
    out, idx = gu.to_f64(out), idx.cpu().numpy()
    atol, rtol = gu.attn_tol(w.dtype)
    for b in range(B):
        k = w.topk[b]
        for h in range(Hkv):
            o = gu.oracle_head(w, dw.bt, b, h)
            q = gu.oracle_queries(w, dw.bt, 0, b, h)
            packed = oracle.quantize_values(o.V)
            o_out, o_idx, o_sc, cond = oracle.decode_step_qv(q, o.K, o.V, packed, o.mu, o.cent, o.code, k,
                                                             w.num_sinks)
            gu.check_selection(idx[b, h, :k], o_idx, o_sc, cond, k)
            g = out[b, h * w.group:(h + 1) * w.group]
            assert np.allclose(g, o_out, atol=atol, rtol=rtol), (b, h, float(np.abs(g - o_out).max()))
            # and it would fail as the full-precision result: the 2-bit rows were read
            f_out = oracle.sparse_attention(q, o.K, o.V, o.mu, o.cent, o.code, o_idx, w.num_sinks)
            assert not np.allclose(g, f_out, atol=atol, rtol=rtol), (b, h)


def test_sparse_attn_qv_matches_oracle():
    """The composed attention kernel with 2-bit values, on the oracle's
    selection (sinks, ragged lengths, GQA groups of 4)."""
    base = gen.small(3, n=2500, batch=2, num_q_heads=16, num_kv_heads=4)
    w = replace(base, name=base.name + "-qv-attn")
    dw = gu.DeviceWorkload(w)
    dw.encode()
    dw.cache.quantize_values()
    B, Hkv = w.batch, w.num_kv_heads
    sel = np.full((B, Hkv, w.max_topk), -1, dtype=np.int32)
    want = {}
    for b in range(B):
        k = w.topk[b]
        for h in range(Hkv):
            o = gu.oracle_head(w, dw.bt, b, h)
            q = gu.oracle_queries(w, dw.bt, 0, b, h)
            sc, _ = oracle.scores(q, o.mu, o.cent, o.code, w.num_sinks)
            ti = oracle.topk(sc, k, w.num_sinks)
            sel[b, h, :k] = ti
            want[(b, h)] = oracle.sparse_attention_qv(q, o.K, o.V, oracle.quantize_values(o.V), o.mu, o.cent,
                                                      o.code, ti, w.num_sinks)
    out = torch.empty((B, w.num_q_heads, 128), dtype=dw.p.torch_dtype, device=dw.dev)
    ws = sk.sikv_sparse_attn_qv(dw.p, dw.q[0], dw.K, dw.V, dw.cache.vq, dw.cache.codes, dw.cache.codebook,
                                dw.cache.mu, torch.from_numpy(sel).to(dw.dev), dw.k, dw.seq_lens, out)
    torch.cuda.synchronize()
    assert ws.check() == 0
    out = gu.to_f64(out)
    atol, rtol = gu.attn_tol(w.dtype)
    for (b, h), o_out in want.items():
        g = out[b, h * w.group:(h + 1) * w.group]
        assert np.allclose(g, o_out, atol=atol, rtol=rtol), (b, h, float(np.abs(g - o_out).max()))
