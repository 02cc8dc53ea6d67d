"""K-means codebook baseline (sikv_kmeans_codebook) against the oracle.

Lloyd's iterations make their nearest-centroid decision in fp32 in a fixed
order and move centroids to exact means rounded once, on both sides, so the
codes, the centroids (as fp32 bit patterns) and the counts must match the
oracle exactly, on ragged batches, for both storage dtypes.  At a full-size
workload the outputs are checked by properties that hold at any size.
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


def _setup(w):
    bt = gen.make_batch(w)
    dev = gu.device()
    p = sk.make_params(w.dtype, w.batch, w.num_q_heads, w.num_kv_heads, w.max_seq_len, w.num_sinks, w.max_topk)
    mu = np.zeros((w.batch, w.num_kv_heads, 128), dtype=np.float32)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            mu[b, h] = oracle.channel_mean(gen.storage_to_f64(bt.K[b, h, :w.seq_lens[b]], w.dtype), w.num_sinks)
    return bt, dev, p, mu


def _run(w, bt, dev, p, mu, init, iters, lens=None):
    lens = w.seq_lens if lens is None else lens
    K = sk.to_device(bt.K, w.dtype, dev)
    codes = torch.full((w.batch, w.num_kv_heads, w.max_seq_len, 16), 0xAB, dtype=torch.uint8, device=dev)
    cent = torch.empty((w.batch, w.num_kv_heads, 32, 16, 4), dtype=torch.float32, device=dev)
    counts = torch.full((w.batch, w.num_kv_heads, 32, 16), -1, dtype=torch.int32, device=dev)
    ws = sk.sikv_kmeans_codebook(p, K, torch.tensor(lens, dtype=torch.int32, device=dev),
                                 torch.from_numpy(mu).to(dev), torch.from_numpy(np.ascontiguousarray(init)).to(dev),
                                 codes, cent, counts, iters=iters)
    torch.cuda.synchronize()
    return ws, codes.cpu().numpy(), cent.cpu().numpy(), counts.cpu().numpy()


@pytest.mark.parametrize("dtype,iters", [("bf16", 20), ("f32", 3), ("bf16", 1)])
def test_kmeans_matches_oracle_bit_for_bit(dtype, iters):
    base = gen.small(3, n=3000, batch=3, num_q_heads=8, num_kv_heads=2)
    w = replace(base, dtype=dtype, name=base.name + "-kmeans")
    bt, dev, p, mu = _setup(w)
    init = gen.kmeans_init(w, w.seq_lens)
    ws, codes, cent, counts = _run(w, bt, dev, p, mu, init, iters)
    assert ws.check() == 0
    S = w.num_sinks
    for b in range(w.batch):
        n = w.seq_lens[b]
        for h in range(w.num_kv_heads):
            Kb = gen.storage_to_f64(bt.K[b, h, :n], w.dtype)
            o_code, o_cent, o_cnt = oracle.kmeans_codebook(Kb, mu[b, h], init[b, h], iters, S)
            assert np.array_equal(cent[b, h].view(np.uint32), o_cent.view(np.uint32)), (b, h)
            assert np.array_equal(counts[b, h], o_cnt), (b, h)
            assert np.array_equal(codes[b, h, S:n], oracle.pack_codes(o_code[S:])), (b, h)
            assert np.all(codes[b, h, :S] == 0xAB) and np.all(codes[b, h, n:] == 0xAB)   # untouched rows


def test_kmeans_edge_cases_are_flagged_or_zero():
    """A sequence with no non-sink token gets zero centroids and counts; a
    start token outside [S, N_b) sets SIKV_DEVERR_INDEX and its centroid starts
    at 0; the other sequences are unaffected."""
    base = gen.small(3, n=1200, batch=3, num_q_heads=4, num_kv_heads=1)
    w = replace(base, seq_lens=(1200, 64, 900), needles_per_head=0, name=base.name + "-kmeans-edge")
    bt, dev, p, mu = _setup(w)
    init = np.zeros((3, 1, 16), dtype=np.int32)
    init[0] = gen.kmeans_init(replace(w, batch=1, seq_lens=(1200,)), (1200,))[0]
    init[2] = gen.kmeans_init(replace(w, batch=1, seq_lens=(900,)), (900,))[0]
    good = init.copy()
    init[2, 0, 5] = 900                                             # one past the end
    ws, codes, cent, counts = _run(w, bt, dev, p, mu, init, 4)
    with pytest.raises(sk.SikvError) as e:
        ws.check()
    assert e.value.flags == sk.SIKV_DEVERR_INDEX
    S = w.num_sinks
    assert np.all(cent[1] == 0) and np.all(counts[1] == 0)
    Kb = gen.storage_to_f64(bt.K[0, 0, :1200], w.dtype)
    o_code, o_cent, o_cnt = oracle.kmeans_codebook(Kb, mu[0, 0], good[0, 0], 4, S)
    assert np.array_equal(cent[0, 0].view(np.uint32), o_cent.view(np.uint32))
    assert np.array_equal(counts[0, 0], o_cnt) and np.array_equal(codes[0, 0, S:1200], oracle.pack_codes(o_code[S:]))
    assert counts[2, 0].sum(axis=1).tolist() == [900 - S] * 32       # every point still assigned


def test_kmeans_full_size_properties():
    """The 32K-token Llama-3-8B layer shape (8 KV heads), 20 iterations: every
    point is counted once, the codes agree with the counts, and every
    non-empty centroid is the mean of the points its code names."""
    w = gen.config(1)
    bt, dev, p, mu = _setup(w)
    init = gen.kmeans_init(w, w.seq_lens)
    ws, codes, cent, counts = _run(w, bt, dev, p, mu, init, 20)
    assert ws.check() == 0
    S, n = w.num_sinks, w.seq_lens[0]
    for h in range(w.num_kv_heads):
        assert np.all(counts[0, h].sum(axis=1) == n - S)
        nib = oracle.unpack_codes(codes[0, h, S:n])                  # [n - S][32]
        x = (gen.storage_to_f64(bt.K[0, h, S:n], w.dtype).astype(np.float32) - mu[0, h]).astype(np.float64)
        for s in range(0, 32, 7):
            lab = nib[:, s]
            assert np.array_equal(np.bincount(lab, minlength=16), counts[0, h, s])
            for j in range(16):
                if counts[0, h, s, j]:
                    m = x[lab == j, 4 * s:4 * s + 4].mean(axis=0)
                    assert np.allclose(cent[0, h, s, j], m, rtol=1e-6, atol=1e-6), (h, s, j)


def _f32(bits):
    return np.array(bits, dtype=np.uint32).view(np.float32)


def test_kmeans_rounding_sensitive_tie_goes_to_lower_cluster():
    """A point at exactly the same fp32 distance from centroids 4 and 5 when
    every operation is rounded (a fused multiply-add would make centroid 5
    nearer) joins cluster 4 on both sides.  The point and the two centroids
    are fp32 values the oracle met on a seeded workload; the other 14
    centroids are far away."""
    x = _f32([0x3f76fb20, 0x3c101bce, 0x3f8644b6, 0xbec1a272])
    c4 = _f32([0x3f0d5b72, 0xbf466c27, 0x3fc98590, 0xbf9a6621])
    c5 = _f32([0x3f1df7db, 0xbd0f9a78, 0x3e223a96, 0x3f087c5a])
    rows = [np.array([100.0 + j, 100.0, 100.0, 100.0], dtype=np.float32) for j in range(16)]
    rows[4], rows[5] = c4, c5
    rows.append(x)
    K = np.stack([np.tile(r, 32) for r in rows]).astype(np.float32)          # [17][128], mu = 0
    mu = np.zeros(128, dtype=np.float32)
    init = np.arange(16, dtype=np.int32)
    o_code, o_cent, o_cnt = oracle.kmeans_codebook(K.astype(np.float64), mu, init, 1, 0)
    assert np.all(o_code[16] == 4)
    dev = gu.device()
    p = sk.make_params("f32", 1, 1, 1, 17, 0, 0)
    codes = torch.zeros((1, 1, 17, 16), dtype=torch.uint8, device=dev)
    cent = torch.empty((1, 1, 32, 16, 4), dtype=torch.float32, device=dev)
    counts = torch.empty((1, 1, 32, 16), dtype=torch.int32, device=dev)
    ws = sk.sikv_kmeans_codebook(p, torch.from_numpy(K).reshape(1, 1, 17, 128).to(dev),
                                 torch.tensor([17], dtype=torch.int32, device=dev),
                                 torch.from_numpy(mu).reshape(1, 1, 128).to(dev),
                                 torch.from_numpy(init).reshape(1, 1, 16).to(dev), codes, cent, counts, iters=1)
    torch.cuda.synchronize()
    assert ws.check() == 0
    assert np.array_equal(codes[0, 0].cpu().numpy(), oracle.pack_codes(o_code))
    assert np.array_equal(counts[0, 0].cpu().numpy(), o_cnt)
    assert np.array_equal(cent[0, 0].cpu().numpy().view(np.uint32), o_cent.view(np.uint32))
