"""The single-launch decode kernels against the standalone entry points and
the oracle.

sikv_decode runs the whole step in one launch: on thread-block clusters (one
cluster per segment) when a segment fits 16 CTAs, else as a cooperative
kernel when every CTA of the step fits on the device at once.  Each test
runs both kernels (forced through sikv_params.decode_path).  Their scores must
be bit-identical to sikv_score's (same table, same order of additions per
token), their selection identical to sikv_topk's on those scores, and their
attention within the attention tolerance of sikv_sparse_attn's over that
selection.
"""

import ctypes
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
    "two-chunks": lambda: gen.small(1, n=2085, batch=1, num_q_heads=8, num_kv_heads=2),
    "many-chunks": lambda: replace(gen.config(1), name="many", batch=1, num_q_heads=8, num_kv_heads=2,
                                   seq_lens=(40000,), topk=(3000,), needles_per_head=8),
    "ragged-empty-chunks": lambda: gen.small(3, n=9000, batch=4, num_q_heads=8, num_kv_heads=2),
    "gqa8": lambda: gen.small(2, n=5000, batch=1, num_q_heads=16, num_kv_heads=2),
    "gqa5": lambda: gen.small(1, n=4100, batch=2, num_q_heads=10, num_kv_heads=2),
    "f32-one-head": lambda: gen.small(0, n=6000),
    "k-equals-n": lambda: replace(gen.config(1), name="kn", batch=2, num_q_heads=4, num_kv_heads=1,
                                  seq_lens=(3000, 2500), topk=(2936, 2436), needles_per_head=2),
}


PATHS = {"cluster": sk.SIKV_DECODE_CLUSTER, "cooperative": sk.SIKV_DECODE_COOPERATIVE}


def _fused_runs(p):
    return int(sk.lib().sikv_decode_launches(ctypes.byref(p))) == 1


def _standalone(dw, step):
    w, dev, c = dw.w, dw.dev, dw.cache
    sc = torch.full((w.batch, w.num_kv_heads, w.max_seq_len), 12345.0, device=dev)
    sk.sikv_score(dw.p, dw.q[step], c.codes, c.codebook, c.mu, dw.seq_lens, sc).check()
    idx = torch.full((w.batch, w.num_kv_heads, w.max_topk), -7, dtype=torch.int32, device=dev)
    sk.sikv_topk(dw.p, sc, dw.seq_lens, dw.k, idx).check()
    out = torch.empty((w.batch, w.num_q_heads, 128), dtype=dw.p.torch_dtype, device=dev)
    sk.sikv_sparse_attn(dw.p, dw.q[step], dw.K, dw.V, c.codes, c.codebook, c.mu, idx, dw.k, dw.seq_lens,
                        out).check()
    return out, idx, sc


@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("name", sorted(SHAPES))
def test_fused_matches_standalone_entry_points(name, path):
    dw = gu.DeviceWorkload(SHAPES[name](), steps=(0, 1), decode_path=PATHS[path])
    assert _fused_runs(dw.p), "the single-launch kernel should cover this shape"
    dw.encode()
    atol, rtol = gu.attn_tol(dw.w.dtype)
    for step in (0, 1):
        out_f, idx_f, sc_f = dw.decode(step=step)
        out_s, idx_s, sc_s = _standalone(dw, step)
        for b in range(dw.w.batch):
            n = dw.w.seq_lens[b]
            assert torch.equal(sc_f[b, :, :n], sc_s[b, :, :n]), (name, step, b)
        assert torch.equal(idx_f, idx_s), (name, step)
        assert np.allclose(gu.to_f64(out_f), gu.to_f64(out_s), atol=atol, rtol=rtol), name


@pytest.mark.parametrize("path", sorted(PATHS))
def test_fused_repeated_calls_leave_clean_state(path):
    """Repeated calls agree bit for bit (the cooperative kernel resets its
    per-segment counters; the cluster kernel keeps no state between calls)."""
    dw = gu.DeviceWorkload(SHAPES["many-chunks"](), steps=(0, 1), decode_path=PATHS[path])
    dw.encode()
    first = [t.clone() for t in dw.decode(step=1)]
    for _ in range(3):
        dw.decode(step=0)
        again = dw.decode(step=1)
        for x, y in zip(first, again):
            assert torch.equal(x, y)


@pytest.mark.parametrize("path", sorted(PATHS))
def test_fused_all_scores_tied_takes_lowest_indices(path):
    """Identical keys: every score ties, the threshold bin holds every token
    (the candidate list does not fit in shared memory) and the selection falls
    back to the lowest token indices."""
    dev = gu.device()
    n, k, S = 20000, 1500, 64
    w = replace(gen.config(1), name="ties", batch=1, num_q_heads=4, num_kv_heads=1, seq_lens=(n,), topk=(k,),
                needles_per_head=0)
    rng = np.random.default_rng(5)
    row = gen.to_storage(rng.standard_normal(128), "bf16")
    K = np.broadcast_to(row, (1, 1, n, 128)).copy()
    V = gen.to_storage(rng.standard_normal((1, 1, n, 128)), "bf16")
    q = gen.to_storage(rng.standard_normal((1, 4, 128)), "bf16")
    bt = gen.Batch(w, K, V, {0: q}, np.array([n], np.int32), np.array([k], np.int32), None, {(0, 0): np.zeros(0)})
    dw = gu.DeviceWorkload(w, bt=bt, decode_path=PATHS[path])
    assert _fused_runs(dw.p)
    dw.encode()
    out, idx, sc = dw.decode()
    Kf = gen.storage_to_f64(K[0, 0], "bf16")
    Vf = gen.storage_to_f64(V[0, 0], "bf16")
    qf = gen.storage_to_f64(q[0], "bf16")
    mu, code, cent, _ = oracle.encode_keys(Kf, S)
    o_out, o_idx, o_sc, cond = oracle.decode_step(qf, Kf, Vf, mu, cent, code, k, S)
    assert np.array_equal(o_idx, np.arange(S, S + k))
    assert np.array_equal(idx[0, 0].cpu().numpy(), o_idx)
    assert np.allclose(gu.to_f64(out)[0], o_out, atol=2e-2, rtol=1e-2)


@pytest.mark.parametrize("name", ["gqa5", "ragged-empty-chunks", "f32-one-head"])
def test_decode_host_matches_device_decode(name):
    """sikv_decode_host (query and output in host memory: page-locked, the
    query copied in by a kernel (staged when unaligned) and the output
    written in place; pageable, staged) and its plan (a captured graph whose
    copies each call points at its buffers) give exactly what sikv_decode
    gives on device buffers."""
    dw = gu.DeviceWorkload(SHAPES[name](), steps=(0, 1))
    dw.encode()
    c, p = dw.cache, dw.p
    # one plan (a captured graph) for both steps: each call re-points its copies
    plan = sk.DecodeHostPlan(p, c.K, c.V, c.codes, c.codebook, c.mu, dw.seq_lens, dw.k)
    for step in (0, 1):
        out_d = torch.empty_like(dw.q[step])
        sk.sikv_decode(p, dw.q[step], c.K, c.V, c.codes, c.codebook, c.mu, dw.seq_lens, dw.k, out_d).check()
        qh = dw.q[step].cpu().pin_memory()
        oh = torch.full(tuple(qh.shape), 7.0, dtype=qh.dtype).pin_memory()
        ws = sk.sikv_decode_host(p, qh, c.K, c.V, c.codes, c.codebook, c.mu, dw.seq_lens, dw.k, oh)
        torch.cuda.synchronize()
        assert ws.check() == 0
        assert torch.equal(oh, out_d.cpu()), (name, step)
        # pageable host memory takes the staged-copy path
        qp = dw.q[step].cpu()
        op = torch.full(tuple(qp.shape), 7.0, dtype=qp.dtype)
        assert not qp.is_pinned()
        sk.sikv_decode_host(p, qp, c.K, c.V, c.codes, c.codebook, c.mu, dw.seq_lens, dw.k, op, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(op, out_d.cpu()), (name, step)
        # page-locked but not 16-byte aligned (one element into the buffer):
        # the query takes the staged-copy path, the output is written in place
        n_el = qh.numel()
        qa = torch.empty(n_el + 1, dtype=qh.dtype).pin_memory()
        oa = torch.full((n_el + 1,), 7.0, dtype=qh.dtype).pin_memory()
        qu, ou = qa[1:].view(qh.shape), oa[1:].view(qh.shape)
        qu.copy_(qh)
        assert qu.is_pinned() and ou.is_pinned() and qu.data_ptr() % 16 and ou.data_ptr() % 16
        sk.sikv_decode_host(p, qu, c.K, c.V, c.codes, c.codebook, c.mu, dw.seq_lens, dw.k, ou, workspace=ws)
        torch.cuda.synchronize()
        assert ws.check() == 0
        assert torch.equal(ou, out_d.cpu()), (name, step)
        oh2 = torch.zeros_like(oh).pin_memory()
        plan(qh, oh2)
        plan(qh, oh2)                                   # repeated calls: same answer
        torch.cuda.synchronize()
        assert plan.workspace.check() == 0
        assert torch.equal(oh2, out_d.cpu()), (name, step)
        # buffers the graph does not take (unaligned, pageable): the staged path
        ou.fill_(7.0)
        plan(qu, ou)
        op.fill_(7.0)
        plan(qp, op)
        torch.cuda.synchronize()
        assert torch.equal(ou, out_d.cpu()) and torch.equal(op, out_d.cpu()), (name, step)
    plan.close()


@pytest.mark.parametrize("path", sorted(PATHS))
def test_batch_split_into_sub_launches_matches_oracle(path):
    """More segments than one co-resident launch holds at this length.  The
    cooperative kernel runs the batch as consecutive single-launch
    sub-batches (here 18 + 1 sequences); the cluster kernel runs it as one
    launch whose clusters do not all fit at once (later ones run in later
    waves).  Checked against the oracle on sampled segments.  Repeated
    calls on the same workspace must give the same bytes: each sub-launch
    leaves only its own segments' coordination state zeroed, so all of them
    must share one layout (the segments sampled in sequences 1 and 2 sit
    where a layout sized for the 1-sequence launch would put its counters
    and candidates)."""
    dev = gu.device()
    B, H, N, S, k = 19, 8, 16896, 64, 842
    p = sk.make_params("bf16", B, H, H, N, S, k, decode_path=PATHS[path])
    assert int(sk.lib().sikv_decode_launches(ctypes.byref(p))) == (2 if path == "cooperative" else 1)
    g = torch.Generator().manual_seed(31)
    K = torch.randn((B, H, N, 128), generator=g).to(torch.bfloat16)
    V = torch.randn((B, H, N, 128), generator=g).to(torch.bfloat16)
    q = torch.randn((B, H, 128), generator=g).to(torch.bfloat16)
    seq = torch.full((B,), N, dtype=torch.int32, device=dev)
    kk = torch.full((B,), k, dtype=torch.int32, device=dev)
    c = sk.SikvCache(p, K.to(dev), V.to(dev), seq)
    c.encode()
    qd = q.to(dev)
    outs = []
    for call in range(3):
        out = torch.empty((B, H, 128), dtype=torch.bfloat16, device=dev)
        idx = torch.full((B, H, k), -7, dtype=torch.int32, device=dev)
        if call == 1:
            c.decode(qd, kk, out=out)                  # the call a serving loop makes
        else:
            c.decode(qd, kk, out=out, idx_out=idx)
        torch.cuda.synchronize()
        c.check()
        outs.append(out.clone())
    assert all(torch.equal(outs[0], o) for o in outs[1:])
    idx = idx.cpu().numpy()
    out = gu.to_f64(outs[-1])
    for b, h in ((0, 0), (1, 0), (2, 4), (17, 5), (18, 7)):
        Kb = K[b, h].double().numpy()
        Vb = V[b, h].double().numpy()
        qb = q[b, h:h + 1].double().numpy()
        mu, code, cent, _ = oracle.encode_keys(Kb, S)
        o_out, o_idx, o_sc, cond = oracle.decode_step(qb, Kb, Vb, mu, cent, code, k, S)
        assert np.all(np.diff(idx[b, h]) > 0)
        gu.check_selection(idx[b, h], o_idx, o_sc, cond, k)
        assert np.allclose(out[b, h:h + 1], o_out, atol=2e-2, rtol=1e-2), (b, h)
