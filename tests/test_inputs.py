"""Seeded input generator: shapes, determinism and storage rounding."""

import numpy as np
import torch

import sikv_inputs as gen


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(100_000) * np.exp2(rng.integers(-20, 20, 100_000))).astype(np.float32)
    x[:4] = [0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8]      # exact ties
    ours = gen.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(gen.bf16_bits_to_f32(ours), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_config_shapes():
    assert gen.config(1).topk == (2458,)
    w2 = gen.config(2)
    assert (w2.batch, w2.num_q_heads, w2.num_kv_heads, w2.max_seq_len, w2.topk[0]) == (4, 32, 8, 131072, 2048)
    w3 = gen.config(3)
    assert w3.batch == 32 and all(8192 <= n <= 32768 for n in w3.seq_lens)
    assert all(k == int(np.ceil(0.075 * n - 1e-9)) for n, k in zip(w3.seq_lens, w3.topk))
    assert gen.config(4).max_seq_len == 524288
    assert gen.config(0).dtype == "f32" and gen.config(0).group == 1


def test_heads_deterministic_and_independent():
    w = gen.small(1, n=700, batch=1, num_q_heads=8, num_kv_heads=2)
    a = gen.head_inputs(w, 0, 0)
    b = gen.head_inputs(w, 0, 0)
    c = gen.head_inputs(w, 0, 1)
    assert np.array_equal(a.keys, b.keys) and np.array_equal(a.queries[0], b.queries[0])
    assert not np.array_equal(a.keys, c.keys)
    assert len(a.needle_pos) == w.needles_per_head
    assert a.needle_pos.min() >= w.num_sinks and len(set(a.needle_pos.tolist())) == len(a.needle_pos)


def test_make_batch_layout():
    w = gen.small(3, n=600, batch=3)
    bt = gen.make_batch(w, steps=(0, 1))
    assert bt.K.shape == (3, w.num_kv_heads, w.max_seq_len, 128) and bt.K.dtype == np.uint16
    for b in range(3):
        n = w.seq_lens[b]
        assert np.all(bt.K[b, :, n:] == 0)
        hi = gen.head_inputs(w, b, 1, steps=(0, 1))
        assert np.array_equal(bt.K[b, 1, :n], hi.keys)
        assert np.array_equal(bt.q[1][b, w.group:2 * w.group], hi.queries[1])
    assert not np.array_equal(bt.q[0], bt.q[1])
