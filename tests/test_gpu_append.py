"""Decode-time append (sikv_append_codes) against the oracle.

Keys written into the cache after prefill are coded against the frozen
prefill mean (readings R19, R20): the appended code rows must equal the
oracle's bit for bit, every other row must be left alone, out-of-range
requests must set SIKV_DEVERR_APPEND without writing, and a decode step over
the grown sequence must match the oracle run on the prefill codebook plus the
appended codes.
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

PREFILL = (2500, 3000, 3896)
COUNT = (1, 37, 200)


def _setup(dtype="bf16"):
    base = gen.small(1, n=4096, batch=3, num_q_heads=8, num_kv_heads=2)
    w = replace(base, dtype=dtype, name=base.name + "-append")
    bt = gen.make_batch(w)
    dev = gu.device()
    p = sk.make_params(w.dtype, w.batch, w.num_q_heads, w.num_kv_heads, w.max_seq_len, w.num_sinks, w.max_topk)
    K = sk.to_device(bt.K, w.dtype, dev)
    V = sk.to_device(bt.V, w.dtype, dev)
    lens0 = torch.tensor(PREFILL, dtype=torch.int32, device=dev)
    cache = sk.SikvCache(p, K, V, lens0.clone())
    cache.encode()
    torch.cuda.synchronize()
    assert cache.ws_encode.check() == 0
    return w, bt, p, cache, dev


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_appended_codes_match_oracle(dtype):
    w, bt, p, cache, dev = _setup(dtype)
    before = cache.codes.clone()
    start = torch.tensor(PREFILL, dtype=torch.int32, device=dev)
    count = torch.tensor(COUNT, dtype=torch.int32, device=dev)
    cache.append(start, count)
    torch.cuda.synchronize()
    assert cache.ws_encode.check() == 0
    after = cache.codes.cpu().numpy()
    prev = before.cpu().numpy()
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            Kb = gen.storage_to_f64(bt.K[b, h], w.dtype)
            mu = oracle.channel_mean(Kb[:PREFILL[b]], w.num_sinks)
            assert np.array_equal(cache.mu[b, h].cpu().numpy().view(np.uint32), mu.view(np.uint32))
            want = oracle.append_codes(prev[b, h], Kb, mu, PREFILL[b], COUNT[b])
            assert np.array_equal(after[b, h], want), (b, h)


def test_out_of_range_append_is_flagged_and_skipped():
    w, bt, p, cache, dev = _setup()
    before = cache.codes.clone()
    start = torch.tensor([-1, 4000, 100], dtype=torch.int32, device=dev)
    count = torch.tensor([1, 200, 5], dtype=torch.int32, device=dev)
    cache.append(start, count)
    with pytest.raises(sk.SikvError) as e:
        cache.ws_encode.check()
    assert e.value.flags & sk.SIKV_DEVERR_APPEND
    after = cache.codes
    assert torch.equal(after[0], before[0]) and torch.equal(after[1], before[1])
    Kb = gen.storage_to_f64(bt.K[2, 0], w.dtype)
    mu = cache.mu[2, 0].cpu().numpy()
    want = oracle.append_codes(before[2, 0].cpu().numpy(), Kb, mu, 100, 5)
    assert np.array_equal(after[2, 0].cpu().numpy(), want)


def test_decode_sees_appended_tokens():
    """A needle written after prefill and appended is selected, and the decode
    step over the grown sequences matches the oracle on the frozen codebook."""
    w, bt, p, cache, dev = _setup()
    g, S = w.group, w.num_sinks
    # plant a needle (3 x the summed group query) at the first appended row of (0, 1)
    q = bt.q[0]
    qbar = gen.storage_to_f64(q[0, g:2 * g], w.dtype).sum(axis=0)
    needle = torch.from_numpy(gen.to_storage(3.0 * qbar, "bf16").view(np.int16)).view(torch.bfloat16)
    cache.K[0, 1, PREFILL[0]] = needle.to(dev)
    bt.K[0, 1, PREFILL[0]] = gen.to_storage(3.0 * qbar, "bf16")
    start = torch.tensor(PREFILL, dtype=torch.int32, device=dev)
    count = torch.tensor(COUNT, dtype=torch.int32, device=dev)
    cache.append(start, count)
    grown = [a + c for a, c in zip(PREFILL, COUNT)]
    cache.seq_lens.copy_(torch.tensor(grown, dtype=torch.int32))
    ks = [min(w.max_topk, n - S) for n in grown]
    kk = torch.tensor(ks, dtype=torch.int32, device=dev)
    qd = sk.to_device(q, w.dtype, dev)
    out = torch.empty_like(qd)
    idx = torch.full((w.batch, w.num_kv_heads, w.max_topk), -7, dtype=torch.int32, device=dev)
    cache.decode(qd, kk, out=out, idx_out=idx)
    torch.cuda.synchronize()
    assert cache.ws_decode.check() == 0 and cache.ws_encode.check() == 0
    idx = idx.cpu().numpy()
    out = gu.to_f64(out)
    assert PREFILL[0] in set(idx[0, 1, :ks[0]].tolist())
    atol, rtol = gu.attn_tol(w.dtype)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            Kb = gen.storage_to_f64(bt.K[b, h, :grown[b]], w.dtype)
            Vb = gen.storage_to_f64(bt.V[b, h, :grown[b]], w.dtype)
            mu, code0, cent, _ = oracle.encode_keys(Kb[:PREFILL[b]], S)      # frozen prefill statistics
            packed = oracle.pack_codes(oracle.sign_codes(Kb, mu))
            packed[:PREFILL[b]] = oracle.pack_codes(code0)
            packed = oracle.append_codes(packed, Kb, mu, PREFILL[b], COUNT[b])
            code = oracle.unpack_codes(packed)
            qg = gen.storage_to_f64(q[b, h * g:(h + 1) * g], w.dtype)
            o_out, o_idx, o_sc, cond = oracle.decode_step(qg, Kb, Vb, mu, cent, code, ks[b], S)
            gu.check_selection(idx[b, h, :ks[b]], o_idx, o_sc, cond, ks[b])
            assert np.allclose(out[b, h * g:(h + 1) * g], o_out, atol=atol, rtol=rtol), (b, h)
