"""The C-ABI library loads, exports what include/sikv.h declares, and rejects
bad arguments on the host before touching the GPU (no CUDA device needed)."""

import ctypes
import os
import re

import pytest

import long_context_decode_sikv_b200 as sk
from long_context_decode_sikv_b200 import _binding as bnd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"SIKV_API\s+[^;(]*?\b(sikv_\w+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported():
    decl = _declared()
    assert {"sikv_encode_keys", "sikv_score", "sikv_topk", "sikv_sparse_attn", "sikv_decode"} <= decl
    lib = sk.lib()
    for name in sorted(decl):
        assert hasattr(lib, name), name
    assert decl <= set(bnd.EXPORTED) | {"sikv_status_string", "sikv_version"}


def test_version_and_status_strings():
    assert sk.version() >= 100
    for code in range(6):
        s = sk.lib().sikv_status_string(code).decode()
        assert s.startswith("SIKV_")


def _p(**kw):
    base = dict(dtype="bf16", batch=2, num_q_heads=8, num_kv_heads=2, max_seq_len=4096, num_sinks=64, max_topk=256)
    base.update(kw)
    return sk.make_params(**base)


@pytest.mark.parametrize("kw,ok", [
    ({}, True),
    ({"head_dim": 64}, False),
    ({"num_q_heads": 7}, False),
    ({"num_q_heads": 32, "num_kv_heads": 2}, False),      # group 16 > 8
    ({"batch": 0}, False),
    ({"max_seq_len": 0}, False),
    ({"num_sinks": -1}, False),
    ({"max_topk": -1}, False),
    ({"dtype": 7}, False),
    ({"decode_path": 1}, True),
    ({"decode_path": 3}, True),
    ({"decode_path": 4}, False),
    ({"decode_path": -1}, False),
])
def test_workspace_size_validates_params(kw, ok):
    p = _p(**kw)
    n = sk.lib().sikv_decode_workspace_size(ctypes.byref(p))
    assert (n > 0) == ok


def test_workspace_sizes_grow_with_shape():
    small, big = _p(), _p(max_seq_len=65536, max_topk=4096)
    for kind in ("sparse_attn", "decode"):
        assert sk.workspace_size(kind, big) > sk.workspace_size(kind, small) >= 256
    assert sk.workspace_size("encode", big) >= sk.workspace_size("encode", small) > 256


def test_host_rejects_bad_arguments_without_launch():
    """Null pointers, unsupported shapes and short workspaces return a status."""
    lib = sk.lib()
    p = _p()
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(1 << 20)          # never dereferenced: validation fails first
    st = lib.sikv_score(ctypes.byref(p), null, fake, fake, fake, fake, fake, fake, 1 << 20, null)
    assert st == 1                             # SIKV_ERR_INVALID_ARG
    bad = _p(head_dim=64)
    st = lib.sikv_score(ctypes.byref(bad), fake, fake, fake, fake, fake, fake, fake, 1 << 20, null)
    assert st == 2                             # SIKV_ERR_UNSUPPORTED
    mis = ctypes.c_void_p((1 << 20) + 4)
    st = lib.sikv_score(ctypes.byref(p), mis, fake, fake, fake, fake, fake, fake, 1 << 20, null)
    assert st == 2                             # misaligned q
    st = lib.sikv_decode(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake, fake, null, null,
                         fake, 1024, null)
    assert st == 3                             # SIKV_ERR_WORKSPACE (too small)
    st = lib.sikv_encode_keys(ctypes.byref(p), fake, fake, fake, fake, fake, null,
                              ctypes.c_void_p((1 << 20) + 16), 1 << 30, null)
    assert st == 3                             # workspace not 256-byte aligned


def test_binding_refuses_host_tensors():
    import torch
    p = _p()
    with pytest.raises(ValueError, match="CUDA"):
        sk.sikv_topk(p, torch.zeros(2, 2, 4096), torch.zeros(2, dtype=torch.int32),
                     torch.zeros(2, dtype=torch.int32), torch.zeros(2, 2, 256, dtype=torch.int32))


def test_decode_host_validates_without_launch():
    """sikv_decode_host: its workspace holds the decode workspace plus device
    copies of q and out; null host buffers are refused before any copy."""
    p = _p()
    L = sk.lib()
    n_dec = L.sikv_decode_workspace_size(ctypes.byref(p))
    n_host = L.sikv_decode_host_workspace_size(ctypes.byref(p))
    q_bytes = p.batch * p.num_q_heads * p.head_dim * 2
    assert n_host >= n_dec + 2 * q_bytes
    bad = sk.make_params("bf16", 2, 7, 2, 4096, 64, 256)
    assert L.sikv_decode_host_workspace_size(ctypes.byref(bad)) == 0
    fake = ctypes.c_void_p(1 << 20)
    st = L.sikv_decode_host(ctypes.byref(p), None, fake, fake, fake, fake, fake, fake, fake, fake, fake,
                            n_host, None)
    assert st == 1                                       # SIKV_ERR_INVALID_ARG: q_host is null
    st = L.sikv_decode_host(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake, None, fake,
                            n_host, None)
    assert st == 1                                       # out_host is null
    st = L.sikv_decode_host(ctypes.byref(bad), fake, fake, fake, fake, fake, fake, fake, fake, fake, fake,
                            n_host, None)
    assert st == 1                                       # invalid parameters


def test_decode_host_plan_validates_without_capture():
    """sikv_decode_host_plan_create refuses bad arguments before any CUDA
    call (a null handle pointer, invalid parameters, null or misaligned
    device pointers, a missing or short workspace); run refuses a null plan
    or null host buffers; destroy accepts NULL."""
    p = _p()
    L = sk.lib()
    n_host = L.sikv_decode_host_workspace_size(ctypes.byref(p))
    fake = ctypes.c_void_p(1 << 20)
    ws = ctypes.c_void_p(1 << 21)
    h = ctypes.c_void_p()
    args = [fake] * 7
    assert L.sikv_decode_host_plan_create(ctypes.byref(p), *args, ws, n_host, None) == 1
    bad = sk.make_params("bf16", 2, 7, 2, 4096, 64, 256)
    assert L.sikv_decode_host_plan_create(ctypes.byref(bad), *args, ws, n_host, ctypes.byref(h)) == 1
    assert not h.value
    assert L.sikv_decode_host_plan_create(ctypes.byref(p), None, *args[1:], ws, n_host, ctypes.byref(h)) == 1
    odd = ctypes.c_void_p((1 << 20) + 4)
    assert L.sikv_decode_host_plan_create(ctypes.byref(p), odd, *args[1:], ws, n_host, ctypes.byref(h)) == 2
    assert L.sikv_decode_host_plan_create(ctypes.byref(p), *args, None, n_host, ctypes.byref(h)) == 3
    assert L.sikv_decode_host_plan_create(ctypes.byref(p), *args, ws, n_host - 256, ctypes.byref(h)) == 3
    assert not h.value
    assert L.sikv_decode_host_plan_run(None, fake, fake, None) == 1
    L.sikv_decode_host_plan_destroy(None)


def test_decode_host_binding_refuses_device_or_misshapen_buffers():
    p = _p()
    import torch
    with pytest.raises((TypeError, ValueError)):
        bnd._host_ptr(torch.zeros(2, 8, 64, dtype=torch.bfloat16), "q_host", p.torch_dtype, (2, 8, 128))
    with pytest.raises(TypeError):
        bnd._host_ptr(torch.zeros(2, 8, 128, dtype=torch.float32), "q_host", p.torch_dtype, (2, 8, 128))
    assert bnd._host_ptr(torch.zeros(2, 8, 128, dtype=torch.bfloat16), "q_host", p.torch_dtype, (2, 8, 128))


def test_append_validates_without_launch():
    p = _p()
    L = sk.lib()
    assert L.sikv_append_workspace_size(ctypes.byref(p)) == 256
    fake = ctypes.c_void_p(1 << 20)
    assert L.sikv_append_codes(ctypes.byref(p), None, fake, fake, fake, fake, fake, 256, None) == 1
    assert L.sikv_append_codes(ctypes.byref(p), fake, None, fake, fake, fake, fake, 256, None) == 1
    assert L.sikv_append_codes(ctypes.byref(p), fake, fake, fake, fake, None, fake, 256, None) == 1
    assert L.sikv_append_codes(ctypes.byref(p), fake, fake, fake, fake, fake, fake, 16, None) == 3   # workspace too small


def test_kmeans_validates_without_launch():
    p = _p()
    L = sk.lib()
    assert L.sikv_kmeans_workspace_size(ctypes.byref(p)) > 256
    fake = ctypes.c_void_p(1 << 20)
    ws = L.sikv_kmeans_workspace_size(ctypes.byref(p))
    args = [fake, fake, fake, fake]
    assert L.sikv_kmeans_codebook(ctypes.byref(p), None, *args[1:], 20, fake, fake, None, fake, ws, None) == 1
    assert L.sikv_kmeans_codebook(ctypes.byref(p), *args[:3], None, 20, fake, fake, None, fake, ws, None) == 1
    assert L.sikv_kmeans_codebook(ctypes.byref(p), *args, 20, None, fake, None, fake, ws, None) == 1
    assert L.sikv_kmeans_codebook(ctypes.byref(p), *args, 0, fake, fake, None, fake, ws, None) == 1      # iters < 1
    assert L.sikv_kmeans_codebook(ctypes.byref(p), *args, 1001, fake, fake, None, fake, ws, None) == 1   # iters > 1000
    assert L.sikv_kmeans_codebook(ctypes.byref(p), *args, 20, fake, fake, ctypes.c_void_p((1 << 20) + 2),
                                  fake, ws, None) == 2                                                  # misaligned counts
    assert L.sikv_kmeans_codebook(ctypes.byref(p), *args, 20, fake, fake, None, fake, 256, None) == 3   # workspace too small


def test_value_quantization_entry_points_validate_without_launch():
    p = _p()
    L = sk.lib()
    assert L.sikv_quantize_values_workspace_size(ctypes.byref(p)) == 256
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)                   # not 16-byte aligned
    assert L.sikv_quantize_values(ctypes.byref(p), fake, fake, None, fake, 256, None) == 1
    assert L.sikv_quantize_values(ctypes.byref(p), fake, fake, odd, fake, 256, None) == 2
    assert L.sikv_quantize_values(ctypes.byref(p), fake, fake, fake, fake, 16, None) == 3
    ws = L.sikv_decode_workspace_size(ctypes.byref(p))
    args = [fake] * 9
    assert L.sikv_decode_qv(ctypes.byref(p), fake, fake, fake, None, *args[:6], None, None, fake, ws, None) == 1
    assert L.sikv_decode_qv(ctypes.byref(p), fake, fake, fake, odd, *args[:6], None, None, fake, ws, None) == 2
    wa = L.sikv_sparse_attn_workspace_size(ctypes.byref(p))
    assert L.sikv_sparse_attn_qv(ctypes.byref(p), fake, fake, fake, None, *args[:7], fake, wa, None) == 1
    assert L.sikv_sparse_attn_qv(ctypes.byref(p), fake, fake, fake, odd, *args[:7], fake, wa, None) == 2


def test_static_attention_entry_validates_without_launch():
    """sikv_sparse_attn_static refuses null or misaligned pointers, invalid
    parameters and sizes beyond its fixed scratch array on the host, before
    it looks up the array or launches anything."""
    fn = sk.lib().sikv_sparse_attn_static
    fn.argtypes = [ctypes.POINTER(sk.Params)] + [ctypes.c_void_p] * 12
    fn.restype = ctypes.c_int
    p = _p()
    fake = ctypes.c_void_p(1 << 20)
    null = ctypes.c_void_p(0)
    args = [fake] * 10                       # q, K, V, codes, codebook, mu, idx, k_per_seq, seq_lens, out
    assert fn(ctypes.byref(p), null, *args[1:], null, null) == 1          # null q
    assert fn(ctypes.byref(p), *args[:9], null, null, null) == 1          # null out
    assert fn(ctypes.byref(p), *args[:6], null, *args[7:], null, null) == 1   # null idx with kmax > 0
    bad = _p(num_q_heads=7)
    assert fn(ctypes.byref(bad), *args, null, null) == 1                  # invalid parameters
    odd16 = ctypes.c_void_p((1 << 20) + 8)
    assert fn(ctypes.byref(p), odd16, *args[1:], null, null) == 2          # q not 16-byte aligned
    odd4 = ctypes.c_void_p((1 << 20) + 2)
    assert fn(ctypes.byref(p), *args, odd4, null) == 2                    # device_flags not 4-byte aligned
    big = sk.make_params("bf16", 256, 32, 8, 131072, 64, 2048)
    assert fn(ctypes.byref(big), *args, null, null) == 3                  # partials beyond the 8 MiB array
