"""Self-Indexing KVCache decode hot path on B200 (sm_100a).

The work runs in ``libsikv.so`` (hand-written CUDA kernels behind the C ABI of
``include/sikv.h``); this package only marshals torch device tensors into it.

Method: "Self-Indexing KVCache: Predicting Sparse Attention from Compressed
Keys" (gist.science summary of paper 2603.14224), technical summary §2.1:
sign-based 1-bit VQ of the keys that doubles as the retrieval index,
compressed-domain LUT-GEMV top-k, and sparse attention over 64
full-precision sink tokens plus the selected tokens.
"""

from __future__ import annotations

import numpy as np
import torch

from ._binding import (EXPORTED, SIKV_DECODE_AUTO, SIKV_DECODE_CLUSTER, SIKV_DECODE_COMPOSED,  # noqa: F401
                       SIKV_DECODE_COOPERATIVE, SIKV_DEVERR_APPEND, SIKV_DEVERR_INDEX, SIKV_DEVERR_SEQ_LEN,  # noqa: F401
                       SIKV_DEVERR_TOPK, SIKV_DTYPE_BF16, SIKV_DTYPE_F32, DecodeHostPlan, Params, SikvError,
                       Workspace, default_scale, lib, library_path, make_params, sikv_append_codes, sikv_decode,
                       sikv_decode_host, sikv_dense_attn, sikv_dense_score, sikv_encode_keys, sikv_kmeans_codebook,
                       sikv_score, sikv_quantize_values, sikv_decode_qv, sikv_sparse_attn_qv, VQ_ROW_BYTES,
                       sikv_sparse_attn, sikv_topk, version, workspace_size)


def to_device(a: np.ndarray, dtype: str, device) -> torch.Tensor:
    """Upload host storage (float32, or bf16 bits as uint16) as a device tensor."""
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(device, non_blocking=False)


class SikvCache:
    """Compressed KV cache of one attention layer, resident on one GPU.

    Holds the full-precision K and V (sinks and values are read from them),
    the per-sequence lengths, and the encoded index: channel means, packed
    codes and the per-subspace codebook.  ``encode()`` runs the prefill
    encoder; ``decode(q, k_per_seq)`` runs one decode step.
    """

    def __init__(self, p: Params, K: torch.Tensor, V: torch.Tensor, seq_lens: torch.Tensor):
        self.p = p
        dev = K.device
        B, H, N, D = p.batch, p.num_kv_heads, p.max_seq_len, p.head_dim
        self.K, self.V, self.seq_lens = K, V, seq_lens
        self.mu = torch.empty((B, H, D), dtype=torch.float32, device=dev)
        self.codes = torch.empty((B, H, N, D // 8), dtype=torch.uint8, device=dev)
        self.codebook = torch.empty((B, H, D // 4, 16, 4), dtype=torch.float32, device=dev)
        self.counts = torch.empty((B, H, D // 4, 16), dtype=torch.int32, device=dev)
        self.ws_encode = Workspace(workspace_size("encode", p), dev)
        self.ws_decode = Workspace(workspace_size("decode", p), dev)
        self.vq = None            # 2-bit value rows, made by quantize_values()

    def encode(self, stream=None):
        sikv_encode_keys(self.p, self.K, self.seq_lens, self.mu, self.codes, self.codebook, self.counts,
                         workspace=self.ws_encode, stream=stream)

    def append(self, start: torch.Tensor, count: torch.Tensor, stream=None):
        """Code the keys of tokens [start[b], start[b] + count[b]) (already
        written into K and V) against the frozen prefill mean.  Raise
        ``seq_lens`` afterwards to make them visible to ``decode``."""
        sikv_append_codes(self.p, self.K, start, count, self.mu, self.codes, workspace=self.ws_encode,
                          stream=stream)

    def quantize_values(self, stream=None):
        """2-bit rows of V for the selected tokens' values (sinks keep V);
        ``decode_qv`` reads them."""
        if self.vq is None:
            p = self.p
            self.vq = torch.empty((p.batch, p.num_kv_heads, p.max_seq_len, VQ_ROW_BYTES), dtype=torch.uint8,
                                  device=self.K.device)
        sikv_quantize_values(self.p, self.V, self.seq_lens, self.vq, workspace=self.ws_encode, stream=stream)

    def decode_qv(self, q, k_per_seq, out=None, idx_out=None, scores_out=None, stream=None):
        """One decode step reading the selected tokens' values from the 2-bit rows."""
        if out is None:
            out = torch.empty_like(q)
        sikv_decode_qv(self.p, q, self.K, self.V, self.vq, self.codes, self.codebook, self.mu, self.seq_lens,
                       k_per_seq, out, idx_out=idx_out, scores_out=scores_out, workspace=self.ws_decode, stream=stream)
        return out

    def decode(self, q, k_per_seq, out=None, idx_out=None, scores_out=None, stream=None):
        if out is None:
            out = torch.empty_like(q)
        sikv_decode(self.p, q, self.K, self.V, self.codes, self.codebook, self.mu, self.seq_lens, k_per_seq,
                    out, idx_out=idx_out, scores_out=scores_out, workspace=self.ws_decode, stream=stream)
        return out

    def check(self):
        """Raise SikvError if a device-side check failed since the last call."""
        self.ws_encode.check()
        self.ws_decode.check()
