"""CUDA path against the CPU oracle, element by element, at sizes the oracle
finishes in seconds (several tiles and ragged tails).

Bars: codes, packed layout, cluster sizes and the channel mean bit-exact;
scores within 1e-4 of the condition scale of their sum; top-k sets identical
(exact on shared fp32 inputs, up to ties within 1e-5 of the k-th score
end to end); attention within 2e-2 abs / 1e-2 rel (bf16) or 1e-5 (fp32).
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


def _edge_workload():
    # lengths below, at and just past the sinks, plus a ragged tail
    return replace(gen.config(1), name="edge", batch=5, num_q_heads=8, num_kv_heads=2,
                   seq_lens=(40, 64, 65, 97, 300), topk=(0, 0, 1, 33, 200), needles_per_head=2,
                   max_seq_len_override=320)


WORKLOADS = {
    "cfg0-f32": lambda: gen.small(0, n=2085),
    "cfg1-gqa4": lambda: gen.small(1, n=2085, batch=1, num_q_heads=8, num_kv_heads=2),
    "cfg3-ragged": lambda: gen.small(3, n=1500, batch=3, num_q_heads=8, num_kv_heads=2),
    "gqa5": lambda: gen.small(1, n=1000, batch=2, num_q_heads=10, num_kv_heads=2),
    "gqa8": lambda: gen.small(2, n=1200, batch=1, num_q_heads=16, num_kv_heads=2),
    "gqa1-bf16": lambda: gen.small(1, n=700, batch=2, num_q_heads=2, num_kv_heads=2),
    "edge": _edge_workload,
}

_CACHE = {}


def _dw(name):
    if name not in _CACHE:
        _CACHE[name] = gu.DeviceWorkload(WORKLOADS[name](), steps=(0, 1))
    return _CACHE[name]


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_encode_bit_exact(name):
    dw = _dw(name)
    w = dw.w
    dw.cache.codes.fill_(0xAB)
    dw.encode()
    mu = dw.cache.mu.cpu().numpy()
    codes = dw.cache.codes.cpu().numpy()
    cb = dw.cache.codebook.cpu().numpy()
    counts = dw.cache.counts.cpu().numpy()
    for b in range(w.batch):
        n = w.seq_lens[b]
        for h in range(w.num_kv_heads):
            o = gu.oracle_head(w, dw.bt, b, h)
            assert np.array_equal(mu[b, h].view(np.uint32), o.mu.view(np.uint32)), (b, h)
            assert np.array_equal(codes[b, h, :n], oracle.pack_codes(o.code)), (b, h)
            assert np.all(codes[b, h, n:] == 0xAB), "rows past N were written"
            assert np.array_equal(counts[b, h], o.counts), (b, h)
            scale = max(1.0, float(np.abs(o.cent).max()))
            assert np.allclose(cb[b, h], o.cent, rtol=1e-5, atol=1e-6 * scale), (b, h)


def test_encode_mean_exact_outside_the_fast_window():
    """bf16 keys with values the encoder's plain fp64 channel sums cannot take
    exactly (zeros of both signs, subnormals, values just outside
    [2^-20, 2^17), very small and very large values) among ordinary ones, a
    head whose every value is tiny, and a head of values at the window's two
    edges only: the channel mean stays bit-exact, the codes and cluster sizes
    exact."""
    w = gen.small(1, n=4096 + 700, batch=1, num_q_heads=12, num_kv_heads=3)
    bt = gen.make_batch(w, steps=(0,))
    n = w.seq_lens[0]
    rng = np.random.default_rng(np.random.SeedSequence([4096, 700, 3]))
    K = gen.storage_to_f64(bt.K, w.dtype).astype(np.float32)
    special = np.array([0.0, -0.0, 2.0 ** -130, -(2.0 ** -133), 2.0 ** -21, -(2.0 ** -21), 2.0 ** -20,
                        -(2.0 ** -20), 2.0 ** 17, -(2.0 ** 17), 130560.0, -130560.0, 1e-30, -1e-30, 1e20,
                        -3e19], np.float32)
    h0 = K[0, 0, :n]
    hit = rng.random(h0.shape) < 2e-4
    h0[hit] = rng.choice(special, size=int(hit.sum()))
    K[0, 1, :n] *= np.float32(2.0 ** -30)
    edge = np.where(rng.random((n, 128)) < 0.5, np.float32(2.0 ** -20), np.float32(130560.0))
    K[0, 2, :n] = edge * rng.choice(np.array([-1.0, 1.0], np.float32), size=(n, 128))
    bt.K = gen.to_storage(K, w.dtype)
    dw = gu.DeviceWorkload(w, steps=(0,), bt=bt)
    dw.encode()
    mu = dw.cache.mu.cpu().numpy()
    codes = dw.cache.codes.cpu().numpy()
    counts = dw.cache.counts.cpu().numpy()
    cb = dw.cache.codebook.cpu().numpy()
    for h in range(w.num_kv_heads):
        o = gu.oracle_head(w, bt, 0, h)
        assert np.array_equal(mu[0, h].view(np.uint32), o.mu.view(np.uint32)), h
        assert np.array_equal(codes[0, h, :n], oracle.pack_codes(o.code)), h
        assert np.array_equal(counts[0, h], o.counts), h
        scale = max(1.0, float(np.abs(o.cent).max()))
        assert np.allclose(cb[0, h], o.cent, rtol=1e-5, atol=1e-6 * scale), h
    del dw
    torch.cuda.empty_cache()


def _upload_oracle_encode(dw):
    """Oracle encode outputs (mu, packed codes, fp32 centroids) as device tensors."""
    w, dev = dw.w, dw.dev
    mu = np.zeros((w.batch, w.num_kv_heads, 128), np.float32)
    codes = np.full((w.batch, w.num_kv_heads, w.max_seq_len, 16), 0xCD, np.uint8)
    cb = np.zeros((w.batch, w.num_kv_heads, 32, 16, 4), np.float32)
    heads = {}
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            o = gu.oracle_head(w, dw.bt, b, h)
            heads[b, h] = o
            mu[b, h] = o.mu
            codes[b, h, :w.seq_lens[b]] = oracle.pack_codes(o.code)
            cb[b, h] = o.cent.astype(np.float32)
    t = lambda a: torch.from_numpy(a).to(dev)
    return heads, t(mu), t(codes), t(cb)


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_score_matches_oracle(name):
    dw = _dw(name)
    w = dw.w
    heads, mu, codes, cb = _upload_oracle_encode(dw)
    sc = torch.full((w.batch, w.num_kv_heads, w.max_seq_len), 777.0, device=dw.dev)
    ws = sk.sikv_score(dw.p, dw.q[1], codes, cb, mu, dw.seq_lens, sc)
    assert ws.check() == 0
    sc = sc.cpu().numpy().astype(np.float64)
    for (b, h), o in heads.items():
        n = w.seq_lens[b]
        want, cond = oracle.scores(gu.oracle_queries(w, dw.bt, 1, b, h), o.mu, o.cent, o.code, w.num_sinks)
        got = sc[b, h, :n]
        s = min(w.num_sinks, n)
        assert np.all(np.isneginf(got[:s]))
        err = np.abs(got[s:] - want[s:])
        assert np.all(err <= gu.SCORE_RTOL * cond[s:]), (b, h, float((err / cond[s:]).max()))
        assert np.all(sc[b, h, n:] == 777.0)


@pytest.mark.parametrize("n,k,s", [(5000, 1, 64), (5000, 4936, 64), (5000, 0, 64), (4099, 300, 64),
                                   (131072, 2048, 64), (20000, 777, 0), (50, 0, 64), (64, 0, 64), (65, 1, 64)])
def test_topk_exact_on_shared_scores(n, k, s):
    dev = gu.device()
    segs, kmax = 3, max(k, 1)
    scores = gen.random_scores(n * 7 + k, segs, n)
    p = sk.make_params("bf16", segs, 1, 1, n, s, kmax)
    seq = torch.full((segs,), n, dtype=torch.int32, device=dev)
    kk = torch.full((segs,), k, dtype=torch.int32, device=dev)
    idx = torch.full((segs, 1, kmax), -9, dtype=torch.int32, device=dev)
    ws = sk.sikv_topk(p, torch.from_numpy(scores).to(dev).view(segs, 1, n), seq, kk, idx)
    assert ws.check() == 0
    got = idx.cpu().numpy()
    for g in range(segs):
        want = oracle.topk(scores[g].astype(np.float64), k, s)
        assert np.array_equal(got[g, 0, :k], want), g
        assert np.all(got[g, 0, k:] == -1)


def test_topk_all_equal_scores_takes_lowest_indices():
    """Every score tied: the threshold bin overflows shared memory (fallback path)."""
    dev = gu.device()
    n, k = 30000, 1234
    scores = torch.full((1, 1, n), 3.25, device=dev)
    scores[0, 0, 100] = -0.0
    p = sk.make_params("bf16", 1, 1, 1, n, 64, k)
    idx = torch.empty((1, 1, k), dtype=torch.int32, device=dev)
    sk.sikv_topk(p, scores, torch.tensor([n], dtype=torch.int32, device=dev),
                 torch.tensor([k], dtype=torch.int32, device=dev), idx).check()
    want = oracle.topk(scores[0, 0].cpu().numpy().astype(np.float64), k, 64)
    assert np.array_equal(idx[0, 0].cpu().numpy(), want)


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_sparse_attention_matches_oracle(name):
    dw = _dw(name)
    w = dw.w
    heads, mu, codes, cb = _upload_oracle_encode(dw)
    idx = np.full((w.batch, w.num_kv_heads, w.max_topk), -1, np.int32)
    for (b, h), o in heads.items():
        k = w.topk[b]
        if k:
            # a random selection (not the top-k) exercises arbitrary order
            idx[b, h, :k] = gen.random_indices(b * 31 + h, w.seq_lens[b], w.num_sinks, k)
    out = torch.empty((w.batch, w.num_q_heads, 128), dtype=dw.p.torch_dtype, device=dw.dev)
    ws = sk.sikv_sparse_attn(dw.p, dw.q[0], dw.K, dw.V, codes, cb, mu, torch.from_numpy(idx).to(dw.dev),
                             dw.k, dw.seq_lens, out)
    assert ws.check() == 0
    got = gu.to_f64(out)
    atol, rtol = gu.attn_tol(w.dtype)
    for (b, h), o in heads.items():
        k = w.topk[b]
        want = oracle.sparse_attention(gu.oracle_queries(w, dw.bt, 0, b, h), o.K, o.V, o.mu, o.cent, o.code,
                                       idx[b, h, :k], w.num_sinks)
        g = got[b, h * w.group:(h + 1) * w.group]
        assert np.allclose(g, want, atol=atol, rtol=rtol), (b, h, float(np.abs(g - want).max()))


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_decode_end_to_end(name):
    dw = _dw(name)
    w = dw.w
    dw.encode()
    out, idx, sc = dw.decode(step=0)
    out, idx, sc = gu.to_f64(out), idx.cpu().numpy(), sc.cpu().numpy().astype(np.float64)
    atol, rtol = gu.attn_tol(w.dtype)
    for b in range(w.batch):
        n, k = w.seq_lens[b], w.topk[b]
        for h in range(w.num_kv_heads):
            o = gu.oracle_head(w, dw.bt, b, h)
            q = gu.oracle_queries(w, dw.bt, 0, b, h)
            o_out, o_idx, o_sc, cond = oracle.decode_step(q, o.K, o.V, o.mu, o.cent, o.code, k, w.num_sinks)
            s = min(w.num_sinks, n)
            assert np.all(np.abs(sc[b, h, s:n] - o_sc[s:]) <= gu.SCORE_RTOL * cond[s:])
            gi = idx[b, h, :k]
            assert np.all(np.diff(gi) > 0), "selection not in ascending order"
            gu.check_selection(gi, o_idx, o_sc, cond, k)
            assert np.all(idx[b, h, k:] == -1)
            needles = set(dw.bt.needles[(b, h)].tolist())
            assert (needles <= set(gi.tolist())) == (needles <= set(o_idx.tolist()))
            g = out[b, h * w.group:(h + 1) * w.group]
            assert np.allclose(g, o_out, atol=atol, rtol=rtol), (b, h, float(np.abs(g - o_out).max()))


def test_decode_is_deterministic():
    dw = _dw("cfg3-ragged")
    dw.encode()
    a = [t.clone() for t in dw.decode(step=1)]
    b = dw.decode(step=1)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_device_checks_flag_and_skip():
    """Out-of-range lengths, k and indices set status bits instead of faulting."""
    dw = _dw("cfg1-gqa4")
    w, dev = dw.w, dw.dev
    dw.encode()
    bad_len = torch.tensor([w.max_seq_len + 5], dtype=torch.int32, device=dev)
    sc = torch.zeros((1, w.num_kv_heads, w.max_seq_len), device=dev)
    ws = sk.sikv_score(dw.p, dw.q[0], dw.cache.codes, dw.cache.codebook, dw.cache.mu, bad_len, sc)
    with pytest.raises(sk.SikvError) as e:
        ws.check()
    assert e.value.flags & sk.SIKV_DEVERR_SEQ_LEN
    bad_k = torch.tensor([w.seq_lens[0]], dtype=torch.int32, device=dev)        # > N - S
    idx = torch.zeros((1, w.num_kv_heads, w.max_topk), dtype=torch.int32, device=dev)
    ws = sk.sikv_topk(dw.p, sc, dw.seq_lens, bad_k, idx)
    with pytest.raises(sk.SikvError) as e:
        ws.check()
    assert e.value.flags & sk.SIKV_DEVERR_TOPK
    idx.fill_(3)                                                                  # a sink, not a selectable token
    out = torch.empty((1, w.num_q_heads, 128), dtype=dw.p.torch_dtype, device=dev)
    ws = sk.sikv_sparse_attn(dw.p, dw.q[0], dw.K, dw.V, dw.cache.codes, dw.cache.codebook, dw.cache.mu, idx,
                             dw.k, dw.seq_lens, out)
    with pytest.raises(sk.SikvError) as e:
        ws.check()
    assert e.value.flags & sk.SIKV_DEVERR_INDEX
    assert torch.isfinite(out.float()).all()
