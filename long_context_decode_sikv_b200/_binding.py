"""ctypes binding of libsikv (argument marshalling only).

Every function takes torch tensors that live on a CUDA device, checks that
their dtype, shape and contiguity match the C ABI documented in
``include/sikv.h``, and passes raw pointers and sizes to the library.  All the
work runs in the library's CUDA kernels; there is no CPU path.  A missing
library is built on first use with nvcc; a missing CUDA device or a failed
launch raises :class:`SikvError`.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

from . import build as _build

SIKV_DTYPE_F32 = 0
SIKV_DTYPE_BF16 = 1

SIKV_DEVERR_SEQ_LEN = 0x1
SIKV_DEVERR_TOPK = 0x2
SIKV_DEVERR_INDEX = 0x4
SIKV_DEVERR_TIMEOUT = 0x8
SIKV_DEVERR_APPEND = 0x10

# sikv_params.decode_path: which kernels a decode step runs
SIKV_DECODE_AUTO = 0
SIKV_DECODE_CLUSTER = 1
SIKV_DECODE_COOPERATIVE = 2
SIKV_DECODE_COMPOSED = 3

_STATUS = {0: "SIKV_OK", 1: "SIKV_ERR_INVALID_ARG", 2: "SIKV_ERR_UNSUPPORTED", 3: "SIKV_ERR_WORKSPACE",
           4: "SIKV_ERR_CUDA", 5: "SIKV_ERR_DEVICE"}

EXPORTED = ("sikv_version", "sikv_status_string", "sikv_workspace_init", "sikv_check_device_status",
            "sikv_encode_workspace_size", "sikv_score_workspace_size", "sikv_topk_workspace_size",
            "sikv_sparse_attn_workspace_size", "sikv_decode_workspace_size", "sikv_encode_keys",
            "sikv_score", "sikv_topk", "sikv_sparse_attn", "sikv_decode", "sikv_decode_launches",
            "sikv_decode_resolved_path",
            "sikv_sparse_attn_static", "sikv_decode_host_workspace_size", "sikv_decode_host",
            "sikv_append_workspace_size", "sikv_append_codes", "sikv_dense_attn_workspace_size",
            "sikv_dense_score", "sikv_dense_attn", "sikv_kmeans_workspace_size", "sikv_kmeans_codebook",
            "sikv_quantize_values_workspace_size", "sikv_quantize_values", "sikv_decode_qv", "sikv_sparse_attn_qv",
            "sikv_decode_host_plan_create", "sikv_decode_host_plan_run", "sikv_decode_host_plan_destroy")

VQ_ROW_BYTES = 48     # a token's 2-bit value row: 32 bytes of levels + 4 (min, step) fp16 pairs


class SikvError(RuntimeError):
    def __init__(self, status: int, where: str, flags: int = 0):
        self.status = status
        self.flags = flags
        msg = f"{where}: {_STATUS.get(status, status)}"
        if flags:
            msg += f" (device flags 0x{flags:x})"
        super().__init__(msg)


class Params(ctypes.Structure):
    """Mirror of ``sikv_params``."""

    _fields_ = [("dtype", ctypes.c_int32), ("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("max_seq_len", ctypes.c_int32),
                ("num_sinks", ctypes.c_int32), ("max_topk", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
                ("decode_path", ctypes.c_int32), ("reserved", ctypes.c_int32 * 2)]

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def segments(self) -> int:
        return self.batch * self.num_kv_heads

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == SIKV_DTYPE_F32 else torch.bfloat16


def make_params(dtype, batch, num_q_heads, num_kv_heads, max_seq_len, num_sinks=64, max_topk=0,
                head_dim=128, softmax_scale=0.0, decode_path=0) -> Params:
    if isinstance(dtype, str):
        dtype = {"f32": SIKV_DTYPE_F32, "bf16": SIKV_DTYPE_BF16}[dtype]
    elif isinstance(dtype, torch.dtype):
        dtype = {torch.float32: SIKV_DTYPE_F32, torch.bfloat16: SIKV_DTYPE_BF16}[dtype]
    return Params(int(dtype), int(batch), int(num_q_heads), int(num_kv_heads), int(head_dim), int(max_seq_len),
                  int(num_sinks), int(max_topk), float(softmax_scale), int(decode_path),
                  (ctypes.c_int32 * 2)(0, 0))


_LIB = None


def lib() -> ctypes.CDLL:
    """Load libsikv.so (building it in-tree first if it is missing or stale)."""
    global _LIB
    if _LIB is None:
        if not _build.up_to_date():
            _build.build()
        L = ctypes.CDLL(_build.LIB)
        vp, sz, i32, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int
        pp = ctypes.POINTER(Params)
        L.sikv_version.restype = i32
        L.sikv_status_string.restype = ctypes.c_char_p
        L.sikv_status_string.argtypes = [st]
        L.sikv_workspace_init.argtypes = [vp, sz, vp]
        L.sikv_check_device_status.argtypes = [vp, sz, vp, ctypes.POINTER(i32)]
        for n in ("sikv_encode_workspace_size", "sikv_score_workspace_size", "sikv_topk_workspace_size",
                  "sikv_sparse_attn_workspace_size", "sikv_decode_workspace_size",
                  "sikv_decode_host_workspace_size", "sikv_append_workspace_size",
                  "sikv_dense_attn_workspace_size", "sikv_kmeans_workspace_size",
                  "sikv_quantize_values_workspace_size"):
            getattr(L, n).restype = sz
            getattr(L, n).argtypes = [pp]
        L.sikv_decode_launches.restype = i32
        L.sikv_decode_launches.argtypes = [pp]
        L.sikv_decode_resolved_path.restype = i32
        L.sikv_decode_resolved_path.argtypes = [pp]
        L.sikv_encode_keys.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sikv_score.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sikv_topk.argtypes = [pp, vp, vp, vp, vp, vp, sz, vp]
        L.sikv_sparse_attn.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sikv_decode.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sikv_decode_host.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sikv_decode_host_plan_create.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, sz, ctypes.POINTER(vp)]
        L.sikv_decode_host_plan_run.argtypes = [vp, vp, vp, vp]
        L.sikv_decode_host_plan_destroy.argtypes = [vp]
        L.sikv_decode_host_plan_destroy.restype = None
        L.sikv_append_codes.argtypes = [pp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sikv_dense_score.argtypes = [pp, vp, vp, vp, vp, vp, sz, vp]
        L.sikv_dense_attn.argtypes = [pp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sikv_kmeans_codebook.argtypes = [pp, vp, vp, vp, vp, i32, vp, vp, vp, vp, sz, vp]
        L.sikv_quantize_values.argtypes = [pp, vp, vp, vp, vp, sz, vp]
        L.sikv_decode_qv.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sikv_sparse_attn_qv.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        for n in ("sikv_workspace_init", "sikv_check_device_status", "sikv_encode_keys", "sikv_score",
                  "sikv_topk", "sikv_sparse_attn", "sikv_decode", "sikv_decode_host", "sikv_append_codes",
                  "sikv_dense_score", "sikv_dense_attn", "sikv_kmeans_codebook", "sikv_quantize_values",
                  "sikv_decode_qv", "sikv_sparse_attn_qv", "sikv_decode_host_plan_create",
                  "sikv_decode_host_plan_run"):
            getattr(L, n).restype = st
        _LIB = L
    return _LIB


def library_path() -> str:
    return _build.LIB


def version() -> int:
    return int(lib().sikv_version())


# ----------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------

def _ptr(t, name, dtype=None, shape=None, device=None, optional=False):
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (libsikv has no CPU path)")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _host_ptr(t, name, dtype, shape):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor; pin it for asynchronous copies")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(status: int, where: str):
    if status != 0:
        raise SikvError(status, where)


class Workspace:
    """A device workspace (torch allocation) with its header zeroed."""

    def __init__(self, nbytes: int, device, stream=None):
        self.nbytes = max(int(nbytes), 256)
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        if self.buf.data_ptr() % 256:
            raise RuntimeError("workspace allocation is not 256-byte aligned")
        _check(lib().sikv_workspace_init(ctypes.c_void_p(self.buf.data_ptr()), self.nbytes,
                                         _stream(stream, self.buf.device)), "sikv_workspace_init")

    @property
    def ptr(self):
        return ctypes.c_void_p(self.buf.data_ptr())

    def check(self, stream=None) -> int:
        """Synchronize, read and clear the device status word; raise on error."""
        flags = ctypes.c_int32(0)
        st = lib().sikv_check_device_status(self.ptr, self.nbytes, _stream(stream, self.buf.device),
                                            ctypes.byref(flags))
        if st != 0:
            raise SikvError(st, "device status", flags.value)
        return flags.value


def workspace_size(kind: str, p: Params) -> int:
    n = getattr(lib(), f"sikv_{kind}_workspace_size")(ctypes.byref(p))
    if n == 0:
        raise SikvError(1, f"sikv_{kind}_workspace_size (invalid parameters)")
    return int(n)


def _ws(kind, p, workspace, device, stream):
    if workspace is None:
        workspace = Workspace(workspace_size(kind, p), device, stream)
    return workspace


# ----------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ----------------------------------------------------------------------------

def sikv_encode_keys(p: Params, K, seq_lens, mu, codes, codebook, counts=None, workspace=None, stream=None):
    dev = K.device
    B, H, N, D = p.batch, p.num_kv_heads, p.max_seq_len, p.head_dim
    args = (_ptr(K, "K", p.torch_dtype, (B, H, N, D), dev), _ptr(seq_lens, "seq_lens", torch.int32, (B,), dev),
            _ptr(mu, "mu", torch.float32, (B, H, D), dev), _ptr(codes, "codes", torch.uint8, (B, H, N, D // 8), dev),
            _ptr(codebook, "codebook", torch.float32, (B, H, D // 4, 16, 4), dev),
            _ptr(counts, "counts", torch.int32, (B, H, D // 4, 16), dev, optional=True))
    ws = _ws("encode", p, workspace, dev, stream)
    _check(lib().sikv_encode_keys(ctypes.byref(p), *args, ws.ptr, ws.nbytes, _stream(stream, dev)), "sikv_encode_keys")
    return ws


def sikv_append_codes(p: Params, K, start, count, mu, codes, workspace=None, stream=None):
    """Decode-time append: code rows [start[b], start[b] + count[b]) of every
    KV head of sequence b against the frozen mean (K rows already written)."""
    dev = K.device
    B, H, N, D = p.batch, p.num_kv_heads, p.max_seq_len, p.head_dim
    args = (_ptr(K, "K", p.torch_dtype, (B, H, N, D), dev), _ptr(start, "start", torch.int32, (B,), dev),
            _ptr(count, "count", torch.int32, (B,), dev), _ptr(mu, "mu", torch.float32, (B, H, D), dev),
            _ptr(codes, "codes", torch.uint8, (B, H, N, D // 8), dev))
    ws = _ws("append", p, workspace, dev, stream)
    _check(lib().sikv_append_codes(ctypes.byref(p), *args, ws.ptr, ws.nbytes, _stream(stream, dev)),
           "sikv_append_codes")
    return ws


def sikv_kmeans_codebook(p: Params, K, seq_lens, mu, init_idx, codes, codebook, counts=None, iters=20,
                         workspace=None, stream=None):
    """Comparison baseline: ``iters`` Lloyd's k-means iterations on the
    normalized sub-vectors from the start tokens ``init_idx`` [B][Hkv][16];
    codes, centroids and counts in the layouts of :func:`sikv_encode_keys`."""
    dev = K.device
    B, H, N, D = p.batch, p.num_kv_heads, p.max_seq_len, p.head_dim
    args = (_ptr(K, "K", p.torch_dtype, (B, H, N, D), dev), _ptr(seq_lens, "seq_lens", torch.int32, (B,), dev),
            _ptr(mu, "mu", torch.float32, (B, H, D), dev), _ptr(init_idx, "init_idx", torch.int32, (B, H, 16), dev))
    outs = (_ptr(codes, "codes", torch.uint8, (B, H, N, D // 8), dev),
            _ptr(codebook, "codebook", torch.float32, (B, H, D // 4, 16, 4), dev),
            _ptr(counts, "counts", torch.int32, (B, H, D // 4, 16), dev, optional=True))
    ws = _ws("kmeans", p, workspace, dev, stream)
    _check(lib().sikv_kmeans_codebook(ctypes.byref(p), *args, int(iters), *outs, ws.ptr, ws.nbytes,
                                      _stream(stream, dev)), "sikv_kmeans_codebook")
    return ws


def sikv_score(p: Params, q, codes, codebook, mu, seq_lens, scores, workspace=None, stream=None):
    dev = q.device
    B, H, N, D = p.batch, p.num_kv_heads, p.max_seq_len, p.head_dim
    args = (_ptr(q, "q", p.torch_dtype, (B, p.num_q_heads, D), dev),
            _ptr(codes, "codes", torch.uint8, (B, H, N, D // 8), dev),
            _ptr(codebook, "codebook", torch.float32, (B, H, D // 4, 16, 4), dev),
            _ptr(mu, "mu", torch.float32, (B, H, D), dev), _ptr(seq_lens, "seq_lens", torch.int32, (B,), dev),
            _ptr(scores, "scores", torch.float32, (B, H, N), dev))
    ws = _ws("score", p, workspace, dev, stream)
    _check(lib().sikv_score(ctypes.byref(p), *args, ws.ptr, ws.nbytes, _stream(stream, dev)), "sikv_score")
    return ws


def sikv_topk(p: Params, scores, seq_lens, k_per_seq, idx, workspace=None, stream=None):
    dev = scores.device
    B, H, N = p.batch, p.num_kv_heads, p.max_seq_len
    args = (_ptr(scores, "scores", torch.float32, (B, H, N), dev), _ptr(seq_lens, "seq_lens", torch.int32, (B,), dev),
            _ptr(k_per_seq, "k_per_seq", torch.int32, (B,), dev),
            _ptr(idx, "idx", torch.int32, (B, H, p.max_topk), dev, optional=p.max_topk == 0))
    ws = _ws("topk", p, workspace, dev, stream)
    _check(lib().sikv_topk(ctypes.byref(p), *args, ws.ptr, ws.nbytes, _stream(stream, dev)), "sikv_topk")
    return ws


def sikv_sparse_attn(p: Params, q, K, V, codes, codebook, mu, idx, k_per_seq, seq_lens, out,
                     workspace=None, stream=None):
    dev = q.device
    B, H, N, D = p.batch, p.num_kv_heads, p.max_seq_len, p.head_dim
    args = (_ptr(q, "q", p.torch_dtype, (B, p.num_q_heads, D), dev), _ptr(K, "K", p.torch_dtype, (B, H, N, D), dev),
            _ptr(V, "V", p.torch_dtype, (B, H, N, D), dev), _ptr(codes, "codes", torch.uint8, (B, H, N, D // 8), dev),
            _ptr(codebook, "codebook", torch.float32, (B, H, D // 4, 16, 4), dev),
            _ptr(mu, "mu", torch.float32, (B, H, D), dev),
            _ptr(idx, "idx", torch.int32, (B, H, p.max_topk), dev, optional=p.max_topk == 0),
            _ptr(k_per_seq, "k_per_seq", torch.int32, (B,), dev), _ptr(seq_lens, "seq_lens", torch.int32, (B,), dev),
            _ptr(out, "out", p.torch_dtype, (B, p.num_q_heads, D), dev))
    ws = _ws("sparse_attn", p, workspace, dev, stream)
    _check(lib().sikv_sparse_attn(ctypes.byref(p), *args, ws.ptr, ws.nbytes, _stream(stream, dev)),
           "sikv_sparse_attn")
    return ws


def sikv_decode(p: Params, q, K, V, codes, codebook, mu, seq_lens, k_per_seq, out, idx_out=None,
                scores_out=None, workspace=None, stream=None):
    dev = q.device
    B, H, N, D = p.batch, p.num_kv_heads, p.max_seq_len, p.head_dim
    args = (_ptr(q, "q", p.torch_dtype, (B, p.num_q_heads, D), dev), _ptr(K, "K", p.torch_dtype, (B, H, N, D), dev),
            _ptr(V, "V", p.torch_dtype, (B, H, N, D), dev), _ptr(codes, "codes", torch.uint8, (B, H, N, D // 8), dev),
            _ptr(codebook, "codebook", torch.float32, (B, H, D // 4, 16, 4), dev),
            _ptr(mu, "mu", torch.float32, (B, H, D), dev), _ptr(seq_lens, "seq_lens", torch.int32, (B,), dev),
            _ptr(k_per_seq, "k_per_seq", torch.int32, (B,), dev),
            _ptr(out, "out", p.torch_dtype, (B, p.num_q_heads, D), dev),
            _ptr(idx_out, "idx_out", torch.int32, (B, H, p.max_topk), dev, optional=True),
            _ptr(scores_out, "scores_out", torch.float32, (B, H, N), dev, optional=True))
    ws = _ws("decode", p, workspace, dev, stream)
    _check(lib().sikv_decode(ctypes.byref(p), *args, ws.ptr, ws.nbytes, _stream(stream, dev)), "sikv_decode")
    return ws


def sikv_quantize_values(p: Params, V, seq_lens, vq, workspace=None, stream=None):
    """2-bit value rows vq [B][Hkv][Nmax][48] (uint8) of V's rows [0, N_b)."""
    dev = V.device
    B, H, N, D = p.batch, p.num_kv_heads, p.max_seq_len, p.head_dim
    args = (_ptr(V, "V", p.torch_dtype, (B, H, N, D), dev), _ptr(seq_lens, "seq_lens", torch.int32, (B,), dev),
            _ptr(vq, "vq", torch.uint8, (B, H, N, VQ_ROW_BYTES), dev))
    ws = _ws("quantize_values", p, workspace, dev, stream)
    _check(lib().sikv_quantize_values(ctypes.byref(p), *args, ws.ptr, ws.nbytes, _stream(stream, dev)),
           "sikv_quantize_values")
    return ws


def sikv_sparse_attn_qv(p: Params, q, K, V, vq, codes, codebook, mu, idx, k_per_seq, seq_lens, out,
                        workspace=None, stream=None):
    """:func:`sikv_sparse_attn` with the selected tokens' values read from the 2-bit rows vq."""
    dev = q.device
    B, H, N, D = p.batch, p.num_kv_heads, p.max_seq_len, p.head_dim
    args = (_ptr(q, "q", p.torch_dtype, (B, p.num_q_heads, D), dev), _ptr(K, "K", p.torch_dtype, (B, H, N, D), dev),
            _ptr(V, "V", p.torch_dtype, (B, H, N, D), dev), _ptr(vq, "vq", torch.uint8, (B, H, N, VQ_ROW_BYTES), dev),
            _ptr(codes, "codes", torch.uint8, (B, H, N, D // 8), dev),
            _ptr(codebook, "codebook", torch.float32, (B, H, D // 4, 16, 4), dev),
            _ptr(mu, "mu", torch.float32, (B, H, D), dev),
            _ptr(idx, "idx", torch.int32, (B, H, p.max_topk), dev, optional=p.max_topk == 0),
            _ptr(k_per_seq, "k_per_seq", torch.int32, (B,), dev), _ptr(seq_lens, "seq_lens", torch.int32, (B,), dev),
            _ptr(out, "out", p.torch_dtype, (B, p.num_q_heads, D), dev))
    ws = _ws("sparse_attn", p, workspace, dev, stream)
    _check(lib().sikv_sparse_attn_qv(ctypes.byref(p), *args, ws.ptr, ws.nbytes, _stream(stream, dev)),
           "sikv_sparse_attn_qv")
    return ws


def sikv_decode_qv(p: Params, q, K, V, vq, codes, codebook, mu, seq_lens, k_per_seq, out, idx_out=None,
                   scores_out=None, workspace=None, stream=None):
    """:func:`sikv_decode` with the selected tokens' values read from the 2-bit rows vq."""
    dev = q.device
    B, H, N, D = p.batch, p.num_kv_heads, p.max_seq_len, p.head_dim
    args = (_ptr(q, "q", p.torch_dtype, (B, p.num_q_heads, D), dev), _ptr(K, "K", p.torch_dtype, (B, H, N, D), dev),
            _ptr(V, "V", p.torch_dtype, (B, H, N, D), dev), _ptr(vq, "vq", torch.uint8, (B, H, N, VQ_ROW_BYTES), dev),
            _ptr(codes, "codes", torch.uint8, (B, H, N, D // 8), dev),
            _ptr(codebook, "codebook", torch.float32, (B, H, D // 4, 16, 4), dev),
            _ptr(mu, "mu", torch.float32, (B, H, D), dev), _ptr(seq_lens, "seq_lens", torch.int32, (B,), dev),
            _ptr(k_per_seq, "k_per_seq", torch.int32, (B,), dev),
            _ptr(out, "out", p.torch_dtype, (B, p.num_q_heads, D), dev),
            _ptr(idx_out, "idx_out", torch.int32, (B, H, p.max_topk), dev, optional=True),
            _ptr(scores_out, "scores_out", torch.float32, (B, H, N), dev, optional=True))
    ws = _ws("decode", p, workspace, dev, stream)
    _check(lib().sikv_decode_qv(ctypes.byref(p), *args, ws.ptr, ws.nbytes, _stream(stream, dev)), "sikv_decode_qv")
    return ws


def default_scale(head_dim: int = 128) -> float:
    return 1.0 / math.sqrt(head_dim)


def _decode_device_args(p: Params, K, V, codes, codebook, mu, seq_lens, k_per_seq):
    dev = K.device
    B, H, N, D = p.batch, p.num_kv_heads, p.max_seq_len, p.head_dim
    return dev, (_ptr(K, "K", p.torch_dtype, (B, H, N, D), dev), _ptr(V, "V", p.torch_dtype, (B, H, N, D), dev),
                 _ptr(codes, "codes", torch.uint8, (B, H, N, D // 8), dev),
                 _ptr(codebook, "codebook", torch.float32, (B, H, D // 4, 16, 4), dev),
                 _ptr(mu, "mu", torch.float32, (B, H, D), dev), _ptr(seq_lens, "seq_lens", torch.int32, (B,), dev),
                 _ptr(k_per_seq, "k_per_seq", torch.int32, (B,), dev))


def sikv_decode_host(p: Params, q_host, K, V, codes, codebook, mu, seq_lens, k_per_seq, out_host,
                     workspace=None, stream=None):
    """One decode step with q and out in host memory (CPU tensors [B][Hq][D]).

    Returns after enqueueing the upload, the step and the download on
    ``stream``; synchronize before reading ``out_host``.
    """
    dev, dargs = _decode_device_args(p, K, V, codes, codebook, mu, seq_lens, k_per_seq)
    shape = (p.batch, p.num_q_heads, p.head_dim)
    q = _host_ptr(q_host, "q_host", p.torch_dtype, shape)
    o = _host_ptr(out_host, "out_host", p.torch_dtype, shape)
    ws = _ws("decode_host", p, workspace, dev, stream)
    _check(lib().sikv_decode_host(ctypes.byref(p), q, *dargs, o, ws.ptr, ws.nbytes, _stream(stream, dev)),
           "sikv_decode_host")
    return ws


class DecodeHostPlan:
    """A host-facing decode step prepared once for one cache
    (sikv_decode_host_plan_*).

    A serving loop that keeps queries and outputs on the host builds one plan
    per cache and calls it once per step with the step's host buffers (CPU
    tensors of shape [B][Hq][D] and the cache's dtype).  Construction captures
    the step as a CUDA graph on the plan's own workspace; each call points its
    query and output copies at the given buffers and launches it on the
    plan's stream (page-locked buffers aligned to 16 bytes; others take
    sikv_decode_host's staged path).  Synchronize before reading the output.
    """

    def __init__(self, p: Params, K, V, codes, codebook, mu, seq_lens, k_per_seq, workspace=None, stream=None):
        self.p = p
        dev, self._dargs = _decode_device_args(p, K, V, codes, codebook, mu, seq_lens, k_per_seq)
        self._keep = (K, V, codes, codebook, mu, seq_lens, k_per_seq)
        self.workspace = _ws("decode_host", p, workspace, dev, stream)
        self._shape = (p.batch, p.num_q_heads, p.head_dim)
        self._dtype = p.torch_dtype
        self._stream = _stream(stream, dev)
        L = lib()
        self._destroy = L.sikv_decode_host_plan_destroy
        self._run = L.sikv_decode_host_plan_run
        # the workspace was zeroed on the plan's stream, where every replay runs
        handle = ctypes.c_void_p()
        _check(L.sikv_decode_host_plan_create(ctypes.byref(p), *self._dargs, self.workspace.ptr,
                                              self.workspace.nbytes, ctypes.byref(handle)),
               "sikv_decode_host_plan_create")
        self._plan = handle

    def __call__(self, q_host, out_host):
        if q_host.is_cuda or out_host.is_cuda or q_host.dtype != self._dtype or out_host.dtype != self._dtype \
                or q_host.shape != self._shape or out_host.shape != self._shape \
                or not (q_host.is_contiguous() and out_host.is_contiguous()):
            _host_ptr(q_host, "q_host", self._dtype, self._shape)       # raises with the reason
            _host_ptr(out_host, "out_host", self._dtype, self._shape)
        st = self._run(self._plan, q_host.data_ptr(), out_host.data_ptr(), self._stream)
        if st != 0:
            raise SikvError(st, "sikv_decode_host_plan_run")

    def close(self):
        """Free the plan's graph (after its work has finished)."""
        if getattr(self, "_plan", None) is not None and self._plan.value:
            self._destroy(self._plan)
        self._plan = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ----------------------------------------------------------------------------
# comparison baselines (not the method)
# ----------------------------------------------------------------------------

def sikv_dense_score(p: Params, q, K, seq_lens, scores, workspace=None, stream=None):
    """Full-precision q_bar . K[t] for every non-sink token (-inf for sinks)."""
    dev = q.device
    B, H, N, D = p.batch, p.num_kv_heads, p.max_seq_len, p.head_dim
    args = (_ptr(q, "q", p.torch_dtype, (B, p.num_q_heads, D), dev), _ptr(K, "K", p.torch_dtype, (B, H, N, D), dev),
            _ptr(seq_lens, "seq_lens", torch.int32, (B,), dev), _ptr(scores, "scores", torch.float32, (B, H, N), dev))
    ws = workspace if workspace is not None else Workspace(256, dev, stream)
    _check(lib().sikv_dense_score(ctypes.byref(p), *args, ws.ptr, ws.nbytes, _stream(stream, dev)), "sikv_dense_score")
    return ws


def sikv_dense_attn(p: Params, q, K, V, seq_lens, out, workspace=None, stream=None):
    """Dense decode attention over every token of each sequence."""
    dev = q.device
    B, H, N, D = p.batch, p.num_kv_heads, p.max_seq_len, p.head_dim
    args = (_ptr(q, "q", p.torch_dtype, (B, p.num_q_heads, D), dev), _ptr(K, "K", p.torch_dtype, (B, H, N, D), dev),
            _ptr(V, "V", p.torch_dtype, (B, H, N, D), dev), _ptr(seq_lens, "seq_lens", torch.int32, (B,), dev),
            _ptr(out, "out", p.torch_dtype, (B, p.num_q_heads, D), dev))
    ws = _ws("dense_attn", p, workspace, dev, stream)
    _check(lib().sikv_dense_attn(ctypes.byref(p), *args, ws.ptr, ws.nbytes, _stream(stream, dev)), "sikv_dense_attn")
    return ws
