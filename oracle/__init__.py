"""Plain, slow CPU oracle of the Self-Indexing KVCache decode hot path.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import or run anything in
this package.  The product (the CUDA library and its Python binding) never
imports it and shares no code with it; the two meet only at the seeded inputs
of ``sikv_inputs``.

Source of every step: "Self-Indexing KVCache: Predicting Sparse Attention from
Compressed Keys" (summary page at gist.science, paper 2603.14224), cited below
as [SIKV §x] for section x of its technical summary:

* §2.1.1  sign-based 1-bit vector quantization: entropy-aware (channel mean)
          normalization, 4-dim sub-vectors mapped by their sign pattern to one
          of 16 clusters, one-pass (non-iterative) clustering into a codebook;
          the same code serves reconstruction and top-k retrieval;
* §2.1.2  compressed-domain top-k retrieval by LUT-GEMV: the query is split
          like the key, dotted with the 16 centroids of each subspace to form a
          lookup table, and a key's score is the sum of the table entries its
          codes index;
* §2.1.3  token-wise format and 64 full-precision sink tokens kept from prefill;
* §2.1.4  dequantization fused with the sparse attention pass.

Where the page is silent the plainest reading is taken; each one is tagged
[R#] and listed in the design notes of the repository:

R1  the mean is per (sequence, KV head, channel) over the prefill keys;
R2  sinks are tokens 0..S-1; they are excluded from the mean, the codebook and
    scoring, and are always attended with their stored K and V;
R3  the mean is the exact mean rounded once to fp32, and that fp32 value is
    what the sign decision compares against;
R4  bit i of a sub-vector's code is [k_{4s+i} >= mu_{4s+i}] (ties give 1),
    LSB first;
R5  sub-vectors are the contiguous dimensions [4s, 4s+4);
R6  two codes per byte, even subspace in the low nibble, one 16-byte row per
    token;
R7  a centroid is the arithmetic mean of the normalized sub-vectors (k - mu)
    of its cluster;
R8  an empty cluster has centroid 0;
R9  the query heads of a GQA group share one selection, scored with the sum
    of their queries;
R10 softmax scale 1/sqrt(D);
R11 k counts non-sink tokens only;
R12 top-k ties go to the lower token index;
R13 the selected set is returned in ascending token order;
R14 a selected key is reconstructed as mu + c[s][code_s];
R19 a token appended at decode time is coded against the prefill mean, which
    stays frozen;
R20 the codebook stays frozen too: appended tokens do not move the centroids.

The k-means codebook (a comparison baseline, not the method: the iterative
clustering that [SIKV §2.1.1]'s one-pass clustering replaces, timed against it
with 20 iterations in [SIKV §4]) adds:

R21 k-means clusters the same points as the one-pass codebook: the normalized
    sub-vectors x = fl32(k - mu) of the non-sink tokens, 16 clusters per
    subspace, Lloyd's iterations (assign every point to its nearest centroid,
    then move every centroid to the mean of its points);
R22 initialization picks 16 distinct non-sink tokens (drawn by the seeded
    input generator and passed in); centroid j of subspace s starts at token
    j's sub-vector s;
R23 the nearest centroid minimizes the squared distance
    ((d0*d0 + d1*d1) + d2*d2) + d3*d3 with d_i = x_i - c_i, every operation
    rounded to fp32 in that order (no fused multiply-add); ties go to the
    lower cluster index;
R24 a non-empty cluster's new centroid is the exact mean of its points,
    rounded once to fp32; an empty cluster keeps its centroid.  After the last
    iteration the codes are its assignment and the counts its cluster sizes.

The 2-bit value operating point (the pages say accuracy holds with 2-bit
quantization and that the memory saving matches 2-bit KIVI [SIKV §3, §4], but
give no scheme) adds:

R25 V is quantized per token in groups of 32 channels, asymmetrically: a group
    keeps its minimum m and step s = (max - min) / 3, a value its level
    q in {0, 1, 2, 3}, and reads back as m + q s (KIVI's per-token value
    quantization);
R26 m and s are stored in fp16 (round to nearest even) after s is formed in
    fp32 as fl32(fl32(max - min) / 3); the level is
    clamp(rint(fl32(fl32(v - m16) / s16)), 0, 3) in fp32 with ties to even,
    and 0 when s16 = 0; values must lie in the fp16 range;
R27 sinks keep their full-precision V; only selected tokens read quantized V;
R28 a token's quantized row is 48 bytes: 32 bytes of levels (dimension d in
    bits 2 (d mod 4) of byte d / 4), then (m16, s16) of groups 0..3.
"""

from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

SUB_DIM = 4          # [SIKV §2.1.1]: 4-dimensional sub-vectors
NUM_CLUSTERS = 16    # [SIKV §2.1.1]: sign pattern of 4 dims -> one of 16 clusters
DEFAULT_SINKS = 64   # [SIKV §2.1.3]: 64 full-precision sink tokens
KMEANS_ITERS = 20    # [SIKV §4]: the k-means the one-pass clustering is timed against
V_GROUP = 32         # R25: channels per quantization group of a value row
V_ROW_BYTES = 48     # R28: 32 bytes of 2-bit levels + 4 (m, s) fp16 pairs


# ----------------------------------------------------------------------------
# exact arithmetic helpers
# ----------------------------------------------------------------------------

def exact_sum(values) -> Fraction:
    """Exact sum of floats.

    ``math.fsum`` returns the correctly rounded sum; appending its negation and
    summing again yields the correctly rounded remainder, which is 0 exactly
    when nothing is left.  The remainder shrinks by at least 2**52 per round.
    """
    terms = [float(v) for v in values]
    total = Fraction(0)
    while True:
        s = math.fsum(terms)
        if s == 0.0:
            return total
        total += Fraction(s)
        terms.append(-s)


def round_to_f32(x: Fraction) -> np.float32:
    """Round an exact rational to the nearest fp32, ties to even."""
    c = np.float32(float(x))
    cands = [np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))]
    best, best_d = None, None
    for cand in cands:
        if not np.isfinite(cand):
            continue
        d = abs(Fraction(float(cand)) - x)
        if best is None or d < best_d or (d == best_d and int(np.float32(cand).view(np.uint32)) % 2 == 0):
            best, best_d = np.float32(cand), d
    return best


# ----------------------------------------------------------------------------
# prefill: encode the key cache  [SIKV §2.1.1, §2.1.3]
# ----------------------------------------------------------------------------

def channel_mean(K: np.ndarray, num_sinks: int = DEFAULT_SINKS) -> np.ndarray:
    """Entropy-aware normalization mean [SIKV §2.1.1] (R1, R2, R3).

    mu[c] = (1/n) * sum_{t=S}^{N-1} K[t, c], computed exactly and rounded once
    to fp32.  With no non-sink token (N <= S) the mean is 0.
    """
    K = np.asarray(K, dtype=np.float64)
    n_tok, d = K.shape
    rows = K[num_sinks:]
    n = rows.shape[0]
    mu = np.zeros(d, dtype=np.float32)
    if n == 0:
        return mu
    for c in range(d):
        mu[c] = round_to_f32(exact_sum(rows[:, c].tolist()) / n)
    return mu


def sign_codes(K: np.ndarray, mu: np.ndarray) -> np.ndarray:
    """Sign-pattern code of every 4-dim sub-vector [SIKV §2.1.1] (R4, R5).

    code[t, s] = sum_i [K[t, 4s+i] >= mu[4s+i]] * 2**i, one nibble per
    (token, subspace).  All tokens get a code, sinks included; sinks' codes are
    never used.
    """
    K = np.asarray(K, dtype=np.float64)
    mu = np.asarray(mu, dtype=np.float32).astype(np.float64)
    n_tok, d = K.shape
    p = d // SUB_DIM
    bits = (K >= mu[None, :]).astype(np.uint8).reshape(n_tok, p, SUB_DIM)
    code = np.zeros((n_tok, p), dtype=np.uint8)
    for i in range(SUB_DIM):
        code |= bits[:, :, i] << i
    return code


def pack_codes(code: np.ndarray) -> np.ndarray:
    """Token-wise packed layout [SIKV §2.1.3] (R6): byte m = code[2m] | code[2m+1] << 4."""
    code = np.asarray(code, dtype=np.uint8)
    if code.shape[1] % 2:
        raise ValueError("packing needs an even number of subspaces (D a multiple of 8)")
    return (code[:, 0::2] | (code[:, 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """Inverse of :func:`pack_codes`."""
    packed = np.asarray(packed, dtype=np.uint8)
    n, m = packed.shape
    code = np.zeros((n, 2 * m), dtype=np.uint8)
    code[:, 0::2] = packed & 0x0F
    code[:, 1::2] = packed >> 4
    return code


def append_codes(packed: np.ndarray, K: np.ndarray, mu: np.ndarray, start: int, count: int) -> np.ndarray:
    """Decode-time append (R19, R20): the code rows of tokens [start, start+count)
    become the packed sign codes of their keys against the frozen prefill mean
    [SIKV §2.1.1, §2.1.3]; every other row is kept.  Returns a new array.

    The pages give the encoding of a key but say nothing of keys that arrive
    after prefill; the plainest reading codes them like prefill keys with the
    statistics fixed at prefill.
    """
    out = np.array(packed, dtype=np.uint8, copy=True)
    if count > 0:
        out[start:start + count] = pack_codes(sign_codes(np.asarray(K)[start:start + count], mu))
    return out


def codebook(K: np.ndarray, mu: np.ndarray, code: np.ndarray, num_sinks: int = DEFAULT_SINKS):
    """One-pass sign-pattern clustering [SIKV §2.1.1] (R2, R7, R8).

    c[s][j] = mean over non-sink tokens t with code[t, s] == j of the
    normalized sub-vector K[t, 4s:4s+4] - mu[4s:4s+4]; 0 for an empty cluster.
    Returns (centroids float64 [P][16][4], counts int64 [P][16]).
    """
    K = np.asarray(K, dtype=np.float64)
    mu64 = np.asarray(mu, dtype=np.float32).astype(np.float64)
    n_tok, d = K.shape
    p = d // SUB_DIM
    cent = np.zeros((p, NUM_CLUSTERS, SUB_DIM))
    counts = np.zeros((p, NUM_CLUSTERS), dtype=np.int64)
    x = K[num_sinks:] - mu64[None, :]
    cs = code[num_sinks:]
    for s in range(p):
        xs = x[:, SUB_DIM * s:SUB_DIM * (s + 1)]
        for j in range(NUM_CLUSTERS):
            members = cs[:, s] == j
            cnt = int(members.sum())
            counts[s, j] = cnt
            if cnt:
                cent[s, j] = xs[members].mean(axis=0)
    return cent, counts


def encode_keys(K: np.ndarray, num_sinks: int = DEFAULT_SINKS):
    """Whole prefill encoder for one (sequence, KV head).

    Returns (mu fp32 [D], codes uint8 [N][P] one nibble per entry, centroids
    f64 [P][16][4], counts [P][16]); :func:`pack_codes` gives the stored rows.
    """
    mu = channel_mean(K, num_sinks)
    code = sign_codes(K, mu)
    cent, counts = codebook(K, mu, code, num_sinks)
    return mu, code, cent, counts


def reconstruct_keys(mu: np.ndarray, centroids: np.ndarray, code: np.ndarray) -> np.ndarray:
    """Dequantized keys k_hat[t] = mu + c[s][code[t, s]] per subspace (R14)."""
    mu64 = np.asarray(mu, dtype=np.float32).astype(np.float64)
    n_tok, p = code.shape
    k_hat = np.empty((n_tok, p * SUB_DIM))
    for s in range(p):
        k_hat[:, SUB_DIM * s:SUB_DIM * (s + 1)] = centroids[s][code[:, s]]
    return k_hat + mu64[None, :]


# ----------------------------------------------------------------------------
# decode: compressed-domain scoring  [SIKV §2.1.2]
# ----------------------------------------------------------------------------

def group_query(q_group: np.ndarray) -> np.ndarray:
    """Summed query of a GQA group (R9): q_bar = sum_h q_h."""
    return np.asarray(q_group, dtype=np.float64).sum(axis=0)


def lut(q_bar: np.ndarray, centroids: np.ndarray) -> np.ndarray:
    """Lookup table [SIKV §2.1.2]: LUT[s][j] = q_bar[4s:4s+4] . c[s][j]."""
    p = centroids.shape[0]
    qs = np.asarray(q_bar, dtype=np.float64).reshape(p, SUB_DIM)
    return np.einsum("si,sji->sj", qs, centroids)


def scores(q_group: np.ndarray, mu: np.ndarray, centroids: np.ndarray, code: np.ndarray,
           num_sinks: int = DEFAULT_SINKS):
    """LUT-GEMV scores of every token [SIKV §2.1.2] (R2, R9).

    score[t] = sum_s LUT[s][code[t, s]] + q_bar . mu for t >= S, -inf for sinks.
    Also returns the condition scale sum_s |LUT[s][code[t, s]]| + |q_bar . mu|
    that bounds the rounding error of any evaluation order of that sum.
    """
    q_bar = group_query(q_group)
    table = lut(q_bar, centroids)
    n_tok, p = code.shape
    picked = table[np.arange(p)[None, :], code.astype(np.int64)]        # [N][P]
    qmu = float(np.dot(q_bar, np.asarray(mu, dtype=np.float32).astype(np.float64)))
    sc = picked.sum(axis=1) + qmu
    scale = np.abs(picked).sum(axis=1) + abs(qmu)
    sc[:min(num_sinks, n_tok)] = -np.inf
    return sc, scale


def topk(score: np.ndarray, k: int, num_sinks: int = DEFAULT_SINKS) -> np.ndarray:
    """Top-k over the non-sink tokens (R11, R12, R13).

    Orders tokens t in [S, N) by (-score[t], t) and keeps the first k; returns
    them in ascending token order.  -0.0 and +0.0 compare equal.
    """
    score = np.asarray(score, dtype=np.float64)
    n_tok = score.shape[0]
    cand = np.arange(num_sinks, n_tok)
    if k < 0 or k > cand.size:
        raise ValueError(f"k={k} outside [0, {cand.size}]")
    order = np.lexsort((cand, -score[cand]))
    return np.sort(cand[order[:k]]).astype(np.int64)


# ----------------------------------------------------------------------------
# decode: sparse attention over sinks + selected tokens  [SIKV §2.1.3, §2.1.4]
# ----------------------------------------------------------------------------

def sparse_attention(q_group: np.ndarray, K: np.ndarray, V: np.ndarray, mu: np.ndarray,
                     centroids: np.ndarray, code: np.ndarray, idx: np.ndarray,
                     num_sinks: int = DEFAULT_SINKS, scale: float | None = None) -> np.ndarray:
    """Attention of each query head over T = {0..S-1} (full precision) and idx.

    logit_t = scale * q_h . K[t] for a sink, scale * q_h . (mu + c[code_t]) for
    a selected token (R14); out_h = sum_t softmax(logit)_t V[t] (R10).
    Returns float64 [G][D].
    """
    q = np.asarray(q_group, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    g, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    n_tok = K.shape[0]
    sinks = np.arange(min(num_sinks, n_tok))
    idx = np.asarray(idx, dtype=np.int64)
    keys = np.concatenate([K[sinks], reconstruct_keys(mu, centroids, code[idx])], axis=0)
    vals = np.concatenate([V[sinks], V[idx]], axis=0)
    if keys.shape[0] == 0:
        return np.zeros((g, d))
    logits = scale * (q @ keys.T)                                    # [G][T]
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    p /= p.sum(axis=1, keepdims=True)
    return p @ vals


def dense_scores(q_group: np.ndarray, K: np.ndarray, num_sinks: int = DEFAULT_SINKS) -> np.ndarray:
    """Comparison baseline, not the method: the full-precision score q_bar . K[t]
    of every non-sink token (R9), -inf for sinks.  It is the dot product the
    compressed-domain score of [SIKV §2.1.2] stands in for.  Returns float64 [N].
    """
    q_bar = group_query(q_group)
    K = np.asarray(K, dtype=np.float64)
    out = K @ q_bar
    out[:min(num_sinks, K.shape[0])] = -np.inf
    return out


def dense_attention(q_group: np.ndarray, K: np.ndarray, V: np.ndarray, n_tok: int | None = None,
                    scale: float | None = None) -> np.ndarray:
    """Comparison baseline, not the method: softmax attention of each query
    head over every token [0, n_tok) with its stored key and value (R10).  It
    is the dense decode attention that [SIKV §2.1.4]'s sparse pass replaces.
    Returns float64 [G][D] (zeros for an empty sequence).
    """
    q = np.asarray(q_group, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    n = K.shape[0] if n_tok is None else n_tok
    g, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if n == 0:
        return np.zeros((g, d))
    logits = scale * (q @ K[:n].T)
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    p /= p.sum(axis=1, keepdims=True)
    return p @ V[:n]


# ----------------------------------------------------------------------------
# comparison baseline: k-means codebook  [SIKV §2.1.1, §4]  (R21-R24)
# ----------------------------------------------------------------------------

def kmeans_points(K: np.ndarray, mu: np.ndarray, num_sinks: int = DEFAULT_SINKS) -> np.ndarray:
    """The points k-means clusters (R21): x[t, s] = fl32(K[t, 4s:4s+4] - mu[4s:4s+4])
    for the non-sink tokens, float32 [N - S][P][4].  Stored keys are exact in fp32.
    """
    K32 = np.asarray(K, dtype=np.float64).astype(np.float32)
    mu32 = np.asarray(mu, dtype=np.float32)
    n_tok, d = K32.shape
    x = K32[num_sinks:] - mu32[None, :]                 # one fp32 subtraction each
    return x.reshape(max(n_tok - num_sinks, 0), d // SUB_DIM, SUB_DIM)


def kmeans_assign(x: np.ndarray, cent: np.ndarray) -> np.ndarray:
    """Nearest centroid of every point (R23).  x float32 [n][P][4], cent float32
    [P][16][4]; returns uint8 [n][P].  numpy rounds each float32 operation on its
    own, and argmin returns the first of equal minima (the lower index).
    """
    out = np.zeros(x.shape[:2], dtype=np.uint8)
    for t0 in range(0, x.shape[0], 4096):
        diff = x[t0:t0 + 4096, :, None, :] - cent[None, :, :, :]          # [n][P][16][4]
        sq = diff * diff
        dist = ((sq[..., 0] + sq[..., 1]) + sq[..., 2]) + sq[..., 3]
        out[t0:t0 + 4096] = np.argmin(dist, axis=2)
    return out


def kmeans_update(x: np.ndarray, assign: np.ndarray, cent: np.ndarray):
    """Move every non-empty centroid to the exact mean of its points, rounded
    once to fp32; empty clusters keep theirs (R24).  Returns (centroids float32
    [P][16][4], counts int64 [P][16]).
    """
    p = x.shape[1]
    new = np.array(cent, dtype=np.float32, copy=True)
    counts = np.zeros((p, NUM_CLUSTERS), dtype=np.int64)
    for s in range(p):
        for j in range(NUM_CLUSTERS):
            members = x[assign[:, s] == j, s, :]
            counts[s, j] = members.shape[0]
            if members.shape[0]:
                for i in range(SUB_DIM):
                    new[s, j, i] = round_to_f32(exact_sum(members[:, i].tolist()) / members.shape[0])
    return new, counts


def kmeans_codebook(K: np.ndarray, mu: np.ndarray, init_idx, iters: int = KMEANS_ITERS,
                    num_sinks: int = DEFAULT_SINKS):
    """K-means codebook of one (sequence, KV head), the iterative baseline of
    [SIKV §2.1.1] (R21-R24): ``iters`` Lloyd's iterations from the centroids at
    the 16 tokens ``init_idx``.

    Returns (codes uint8 [N][P] one nibble per entry, rows t < S zero;
    centroids float32 [P][16][4]; counts int64 [P][16]).  With no non-sink
    token every centroid and count is 0.
    """
    if iters < 1:
        raise ValueError("k-means needs at least one iteration")
    n_tok, d = np.asarray(K).shape
    p = d // SUB_DIM
    code = np.zeros((n_tok, p), dtype=np.uint8)
    x = kmeans_points(K, mu, num_sinks)
    if x.shape[0] == 0:
        return code, np.zeros((p, NUM_CLUSTERS, SUB_DIM), dtype=np.float32), np.zeros((p, NUM_CLUSTERS), np.int64)
    idx = np.asarray(init_idx, dtype=np.int64)
    if idx.shape != (NUM_CLUSTERS,) or np.any(idx < num_sinks) or np.any(idx >= n_tok):
        raise ValueError("init_idx must hold 16 non-sink token positions")
    cent = np.ascontiguousarray(x[idx - num_sinks].transpose(1, 0, 2))   # [P][16][4]
    for _ in range(iters):
        assign = kmeans_assign(x, cent)
        cent, counts = kmeans_update(x, assign, cent)
    code[num_sinks:] = assign
    return code, cent, counts


# ----------------------------------------------------------------------------
# 2-bit values  [SIKV §3, §4]  (R25-R28)
# ----------------------------------------------------------------------------

def quantize_values(V: np.ndarray) -> np.ndarray:
    """Per-token 2-bit quantization of value rows (R25, R26, R28).

    V holds stored values (exact in fp32), [N][D] with D = 128.  Returns the
    48-byte rows, uint8 [N][48].
    """
    V32 = np.asarray(V, dtype=np.float64).astype(np.float32)
    n, d = V32.shape
    ng = d // V_GROUP
    G = V32.reshape(n, ng, V_GROUP)
    lo, hi = G.min(axis=2), G.max(axis=2)
    step32 = (hi - lo) / np.float32(3)                     # two fp32 operations
    m16, s16 = lo.astype(np.float16), step32.astype(np.float16)
    m32, s32 = m16.astype(np.float32)[..., None], s16.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (G - m32) / s32                                # fp32 subtraction, then fp32 division
    level = np.where(s32 > 0, np.clip(np.rint(t), 0, 3), 0).astype(np.uint8).reshape(n, d // 4, 4)
    out = np.zeros((n, V_ROW_BYTES), dtype=np.uint8)
    out[:, :d // 4] = level[..., 0] | (level[..., 1] << 2) | (level[..., 2] << 4) | (level[..., 3] << 6)
    out[:, d // 4:] = np.stack([m16, s16], axis=2).reshape(n, 2 * ng).view(np.uint8)
    return out


def dequantize_values(packed: np.ndarray, d: int = 128) -> np.ndarray:
    """The values the quantized rows stand for: m + q s, float64 [N][D] (R25)."""
    packed = np.asarray(packed, dtype=np.uint8)
    n = packed.shape[0]
    ng = d // V_GROUP
    b = packed[:, :d // 4]
    level = np.stack([(b >> (2 * i)) & 3 for i in range(4)], axis=2).reshape(n, ng, V_GROUP).astype(np.float64)
    ms = np.ascontiguousarray(packed[:, d // 4:d // 4 + 4 * ng]).view(np.float16).reshape(n, ng, 2).astype(np.float64)
    return (ms[..., 0:1] + level * ms[..., 1:2]).reshape(n, d)


def sparse_attention_qv(q_group, K, V, packed, mu, centroids, code, idx, num_sinks=DEFAULT_SINKS, scale=None):
    """Sparse attention with 2-bit values for the selected tokens and
    full-precision values for the sinks (R27); otherwise
    :func:`sparse_attention`."""
    Vmix = np.array(V, dtype=np.float64, copy=True)
    s = min(num_sinks, Vmix.shape[0])
    Vmix[s:] = dequantize_values(np.asarray(packed)[s:Vmix.shape[0]], Vmix.shape[1])
    return sparse_attention(q_group, K, Vmix, mu, centroids, code, idx, num_sinks, scale)


def decode_step_qv(q_group, K, V, packed, mu, centroids, code, k, num_sinks=DEFAULT_SINKS, scale=None):
    """:func:`decode_step` with 2-bit values for the selected tokens (R27)."""
    sc, cond = scores(q_group, mu, centroids, code, num_sinks)
    idx = topk(sc, k, num_sinks)
    out = sparse_attention_qv(q_group, K, V, packed, mu, centroids, code, idx, num_sinks, scale)
    return out, idx, sc, cond


def decode_step(q_group, K, V, mu, centroids, code, k, num_sinks=DEFAULT_SINKS, scale=None):
    """One decode step of one (sequence, KV head): score, select, attend.

    Returns (out float64 [G][D], idx ascending, scores, condition scale).
    """
    sc, cond = scores(q_group, mu, centroids, code, num_sinks)
    idx = topk(sc, k, num_sinks)
    out = sparse_attention(q_group, K, V, mu, centroids, code, idx, num_sinks, scale)
    return out, idx, sc, cond
