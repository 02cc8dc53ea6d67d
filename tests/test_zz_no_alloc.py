"""sikv_sparse_attn_static: sparse attention for callers that cannot allocate.

Some callers have no way to call cudaMalloc: a serving engine that plans all
of its device memory once at start-up and may not allocate inside the decode
loop, or a plugin host that hands the kernel only its inputs and outputs.
They cannot pass the workspace that sikv_sparse_attn needs, so the library
offers a variant whose scratch lives in a fixed 8 MiB array compiled into the
library.  These tests call that variant through the C ABI and check that it
returns what sikv_sparse_attn returns, on two calls in a row (the array keeps
the previous call's contents) and what the oracle's attention gives over the
same selection, that it reports device-side errors, and that
sizes beyond its limit are refused before anything is launched.

This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes when run on its own.
"""

import ctypes

import numpy as np
import pytest
import torch

import long_context_decode_sikv_b200 as sk
import oracle
import sikv_inputs as gen
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _static_entry():
    fn = sk.lib().sikv_sparse_attn_static
    fn.argtypes = [ctypes.POINTER(sk.Params)] + [ctypes.c_void_p] * 12
    fn.restype = ctypes.c_int
    return fn


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _indices(w):
    idx = np.full((w.batch, w.num_kv_heads, w.max_topk), -1, np.int32)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            k = w.topk[b]
            idx[b, h, :k] = gen.random_indices(100 + 7 * b + h, w.seq_lens[b], w.num_sinks, k)
    return idx


def test_static_scratch_matches_workspace_variant_twice():
    dev = gu.device()
    w = gen.small(3, n=3000, batch=3, num_q_heads=8, num_kv_heads=2)      # ragged lengths
    dw = gu.DeviceWorkload(w, steps=(0, 1))
    dw.encode()
    c = dw.cache
    idx = torch.from_numpy(_indices(w)).to(dev)
    fn = _static_entry()
    flags = torch.full((1,), -1, dtype=torch.int32, device=dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    atol, rtol = gu.attn_tol(w.dtype)
    heads = {(b, h): gu.oracle_head(w, dw.bt, b, h) for b in range(w.batch) for h in range(w.num_kv_heads)}
    for step in (0, 1):
        ref = torch.empty((w.batch, w.num_q_heads, 128), dtype=dw.p.torch_dtype, device=dev)
        sk.sikv_sparse_attn(dw.p, dw.q[step], dw.K, dw.V, c.codes, c.codebook, c.mu, idx, dw.k, dw.seq_lens,
                            ref).check()
        out = torch.full_like(ref, float("nan"))
        st = fn(ctypes.byref(dw.p), _p(dw.q[step]), _p(dw.K), _p(dw.V), _p(c.codes), _p(c.codebook), _p(c.mu),
                _p(idx), _p(dw.k), _p(dw.seq_lens), _p(out), _p(flags), stream)
        assert st == 0, sk.lib().sikv_status_string(st)
        torch.cuda.synchronize()
        assert flags.item() == 0
        assert torch.isfinite(out.float()).all()
        assert np.allclose(gu.to_f64(out), gu.to_f64(ref), atol=atol, rtol=rtol), step
        # and directly against the oracle's attention over the same selection
        got = gu.to_f64(out)
        idx_h = idx.cpu().numpy()
        for b in range(w.batch):
            k = w.topk[b]
            for h in range(w.num_kv_heads):
                o = heads[(b, h)]
                q = gu.oracle_queries(w, dw.bt, step, b, h)
                want = oracle.sparse_attention(q, o.K, o.V, o.mu, o.cent, o.code, idx_h[b, h, :k], w.num_sinks)
                g = got[b, h * w.group:(h + 1) * w.group]
                assert np.allclose(g, want, atol=atol, rtol=rtol), (step, b, h, float(np.abs(g - want).max()))


def test_static_scratch_reports_device_errors():
    dev = gu.device()
    w = gen.small(1, n=800, batch=1, num_q_heads=4, num_kv_heads=1)
    dw = gu.DeviceWorkload(w)
    dw.encode()
    c = dw.cache
    idx = torch.full((1, 1, w.max_topk), 5, dtype=torch.int32, device=dev)     # sinks are not selectable
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    out = torch.empty((1, w.num_q_heads, 128), dtype=dw.p.torch_dtype, device=dev)
    st = _static_entry()(ctypes.byref(dw.p), _p(dw.q[0]), _p(dw.K), _p(dw.V), _p(c.codes), _p(c.codebook),
                         _p(c.mu), _p(idx), _p(dw.k), _p(dw.seq_lens), _p(out), _p(flags),
                         ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    assert flags.item() & sk.SIKV_DEVERR_INDEX


def test_static_scratch_refuses_sizes_beyond_its_limit():
    # 2048 segments x 17 splits x 4 heads x 520 B is far above 8 MiB: refused
    # on the host, before any launch (the pointers are never dereferenced).
    p = sk.make_params("bf16", 256, 32, 8, 131072, 64, 2048)
    fake = ctypes.c_void_p(1 << 20)
    st = _static_entry()(ctypes.byref(p), *([fake] * 10), ctypes.c_void_p(0), ctypes.c_void_p(0))
    assert st == 3                                       # SIKV_ERR_WORKSPACE
