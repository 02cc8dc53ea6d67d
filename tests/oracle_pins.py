"""Pins of the CPU oracle to facts outside itself.

Each ``check_*`` takes the oracle module (or a mutated copy of it) and raises
AssertionError when the oracle disagrees with something the pages or the
mathematics fix: a hand-worked example from ``tests/golden``, a closed form,
an invariant, a brute-force enumeration or a library routine.  The pin tests
call them on the real oracle; the mutation tests call them on deliberately
broken copies to show that each plausible mistake is caught by at least one.

Page cited: "Self-Indexing KVCache: Predicting Sparse Attention from
Compressed Keys" (gist.science summary of paper 2603.14224), technical summary
§2.1 items 1-4.
"""

from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np

import sikv_inputs as gen

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# exact mean (§2.1 item 1, entropy-aware normalization)
# --------------------------------------------------------------------------

def check_exact_sum(o):
    assert o.exact_sum([1e16, 1.0, -1e16]) == 1
    assert o.exact_sum([2.0 ** 60, 2.0 ** -60, -(2.0 ** 60)]) == Fraction(1, 2 ** 60)
    rng = np.random.default_rng(11)
    for _ in range(20):
        v = rng.standard_normal(50) * np.exp2(rng.integers(-40, 40, size=50))
        assert o.exact_sum(v) == sum(Fraction(float(x)) for x in v)


def check_round_to_f32(o):
    one = Fraction(1)
    ulp = Fraction(1, 2 ** 23)
    # exact midpoints round to the even neighbour
    assert o.round_to_f32(one + ulp / 2) == np.float32(1.0)
    assert o.round_to_f32(one + 3 * ulp / 2) == np.float32(1.0 + 2.0 ** -22)
    # just above a midpoint rounds up even where a double rounding would not
    assert o.round_to_f32(one + ulp / 2 + Fraction(1, 2 ** 80)) == np.float32(1.0 + 2.0 ** -23)
    rng = np.random.default_rng(12)
    for x in rng.standard_normal(200) * 1e3:
        assert o.round_to_f32(Fraction(float(x))) == np.float32(x)


def check_channel_mean(o):
    rng = np.random.default_rng(13)
    for n, s in ((5, 0), (37, 3), (200, 64)):
        K = rng.standard_normal((n, 8)) * np.exp2(rng.integers(-30, 30, size=(n, 8)))
        K = K.astype(np.float32).astype(np.float64)
        mu = o.channel_mean(K, s)
        rows = K[s:]
        for c in range(8):
            want = sum(Fraction(float(x)) for x in rows[:, c]) / rows.shape[0]
            # brute-force correct rounding: nearest fp32 by enumeration of neighbours
            cand = np.float32(float(want))
            nb = [np.nextafter(cand, np.float32(-np.inf)), cand, np.nextafter(cand, np.float32(np.inf))]
            dist = [abs(Fraction(float(x)) - want) for x in nb]
            best = min(dist)
            ok = [np.float32(x) for x, dd in zip(nb, dist) if dd == best]
            assert mu[c] in ok, (n, s, c, mu[c], ok)
        # sinks never enter the mean
        K2 = K.copy()
        K2[:s] = 1e30
        assert np.array_equal(o.channel_mean(K2, s), mu)
    # cancellation that plain fp64 summation gets wrong
    col = np.array([2.0 ** 60, 3.0, -(2.0 ** 60), 0.0])
    K = np.stack([col] * 4, axis=1)
    assert np.all(o.channel_mean(K, 0) == np.float32(0.75))
    # nothing to average
    assert np.all(o.channel_mean(np.ones((3, 4)), 64) == 0)


# --------------------------------------------------------------------------
# sign codes and packing (§2.1 items 1 and 3)
# --------------------------------------------------------------------------

def check_sign_codes_golden(o):
    g = _load("sign_codes_d8.json")
    K = np.asarray(g["keys"], dtype=np.float32).astype(np.float64)
    mu = np.asarray(g["mu"], dtype=np.float32)
    code = o.sign_codes(K, mu)
    assert code.tolist() == g["codes"], code.tolist()
    assert o.pack_codes(code).tolist() == g["packed"]


def check_codes_by_construction(o):
    rng = np.random.default_rng(14)
    n, d = 64, 32
    want = rng.integers(0, 16, size=(n, d // 4))
    mu = rng.standard_normal(d).astype(np.float32)
    K = np.empty((n, d))
    for t in range(n):
        for s in range(d // 4):
            for i in range(4):
                bit = (int(want[t, s]) >> i) & 1
                mag = float(rng.uniform(0.01, 3.0))
                K[t, 4 * s + i] = float(mu[4 * s + i]) + (mag if bit else -mag)
    code = o.sign_codes(K.astype(np.float32).astype(np.float64), mu)
    assert np.array_equal(code, want)
    packed = o.pack_codes(code)
    for t in range(n):
        for m in range(d // 8):
            assert packed[t, m] == int(want[t, 2 * m]) + 16 * int(want[t, 2 * m + 1])
    assert np.array_equal(o.unpack_codes(packed), want)


# --------------------------------------------------------------------------
# codebook (§2.1 item 1: one-pass sign-pattern clustering)
# --------------------------------------------------------------------------

def check_codebook_golden(o):
    g = _load("codebook_d4.json")
    for case in g["cases"]:
        K = np.asarray(case["keys"], dtype=np.float64)
        s = case["num_sinks"]
        mu = o.channel_mean(K, s)
        assert mu.tolist() == case["mu"], (case["name"], mu)
        code = o.sign_codes(K, mu)
        assert code.tolist() == case["codes"], (case["name"], code.tolist())
        cent, counts = o.codebook(K, mu, code, s)
        want = np.zeros((1, 16, 4))
        for j, v in case["centroids_nonzero"].items():
            want[0, int(j)] = v
        wc = np.zeros((1, 16), dtype=np.int64)
        for j, v in case["counts_nonzero"].items():
            wc[0, int(j)] = v
        assert np.array_equal(cent, want), (case["name"], cent)
        assert np.array_equal(counts, wc)


def check_codebook_invariants(o):
    w = gen.small(0, n=1500)
    hi = gen.head_inputs(w, 0, 0)
    K = gen.storage_to_f64(hi.keys, w.dtype)
    mu, code, cent, counts = o.encode_keys(K, w.num_sinks)
    n = K.shape[0] - w.num_sinks
    assert np.all(counts.sum(axis=1) == n)
    for s in range(cent.shape[0]):
        for j in range(16):
            if counts[s, j] == 0:
                assert np.all(cent[s, j] == 0)
                continue
            for i in range(4):
                # members all satisfy k >= mu exactly when bit i is set
                if (j >> i) & 1:
                    assert cent[s, j, i] >= 0
                else:
                    assert cent[s, j, i] < 0
    # count-weighted centroids add up to the total normalized mass
    x = K[w.num_sinks:] - mu.astype(np.float64)[None, :]
    tot = (counts[:, :, None] * cent).sum(axis=1).reshape(-1)
    assert np.allclose(tot, x.sum(axis=0), rtol=1e-9, atol=1e-6)
    # cluster membership recounted by brute force
    for s in (0, 7, 31):
        for j in (0, 5, 15):
            assert counts[s, j] == int(np.sum(code[w.num_sinks:, s] == j))


def _distinct_pattern_keys(num_sinks: int, d: int = 8, seed: int = 15):
    """16 non-sink keys whose sub-vectors take each sign pattern once.

    Magnitudes are +-a_i per dimension, so the channel mean is the centre c
    exactly and every cluster holds one token: reconstruction is exact.
    """
    rng = np.random.default_rng(seed)
    c = rng.integers(-8, 8, size=d).astype(np.float64)
    a = rng.integers(1, 5, size=d).astype(np.float64)
    perms = [rng.permutation(16) for _ in range(d // 4)]
    rows = []
    for t in range(16):
        row = np.empty(d)
        for s in range(d // 4):
            j = perms[s][t]
            for i in range(4):
                row[4 * s + i] = c[4 * s + i] + (a[4 * s + i] if (j >> i) & 1 else -a[4 * s + i])
        rows.append(row)
    sinks = rng.standard_normal((num_sinks, d)) * 3
    return np.concatenate([sinks, np.asarray(rows)], axis=0), c


def check_one_member_clusters_reconstruct(o):
    for s in (0, 3):
        K, c = _distinct_pattern_keys(s)
        mu, code, cent, counts = o.encode_keys(K, s)
        assert np.array_equal(mu, c.astype(np.float32))
        assert np.all(counts == 1)
        k_hat = o.reconstruct_keys(mu, cent, code)
        assert np.array_equal(k_hat[s:], K[s:])


# --------------------------------------------------------------------------
# LUT-GEMV scores (§2.1 item 2)
# --------------------------------------------------------------------------

def check_scores_golden(o):
    case = _load("codebook_d4.json")["cases"][0]
    K = np.asarray(case["keys"], dtype=np.float64)
    s = case["num_sinks"]
    mu, code, cent, _ = o.encode_keys(K, s)
    q = np.asarray(case["queries"])
    q_bar = o.group_query(q)
    assert float(np.dot(q_bar, mu.astype(np.float64))) == case["q_bar_dot_mu"]
    table = o.lut(q_bar, cent)
    want = np.zeros(16)
    for j, v in case["lut_nonzero"].items():
        want[int(j)] = v
    assert np.array_equal(table[0], want), table
    sc, cond = o.scores(q, mu, cent, code, s)
    exp = [(-np.inf if v is None else v) for v in case["scores"]]
    assert sc.tolist() == exp, sc


def check_lut_identity(o):
    """sum_s LUT[s][code_s] + q_bar.mu = q_bar . k_hat  (identity behind §2.1 item 2)."""
    w = gen.small(1, n=900, batch=1, num_q_heads=4, num_kv_heads=1)
    hi = gen.head_inputs(w, 0, 0)
    K = gen.storage_to_f64(hi.keys, w.dtype)
    q = gen.storage_to_f64(hi.queries[0], w.dtype)
    mu, code, cent, _ = o.encode_keys(K, w.num_sinks)
    sc, cond = o.scores(q, mu, cent, code, w.num_sinks)
    # independent formulation: dequantize each key coordinate, then a plain dot
    k_hat = np.empty_like(K)
    for t in range(K.shape[0]):
        for dim in range(K.shape[1]):
            k_hat[t, dim] = float(mu[dim]) + cent[dim // 4, code[t, dim // 4], dim % 4]
    direct = k_hat @ q.sum(axis=0)
    sl = slice(w.num_sinks, None)
    assert np.all(np.abs(sc[sl] - direct[sl]) <= 1e-12 * cond[sl])
    assert np.all(np.isneginf(sc[:w.num_sinks]))
    # GQA: the group score is the sum of the single-head scores
    per_head = sum(o.scores(q[h:h + 1], mu, cent, code, w.num_sinks)[0][sl] for h in range(q.shape[0]))
    assert np.allclose(per_head, sc[sl], rtol=0, atol=1e-10 * float(cond.max()))


# --------------------------------------------------------------------------
# top-k (selection of the k highest compressed-domain scores)
# --------------------------------------------------------------------------

def _is_topk_by_definition(score, chosen, k, s):
    n = len(score)
    chosen = set(int(t) for t in chosen)
    if len(chosen) != k or any(t < s or t >= n for t in chosen):
        return False

    def before(a, b):
        return score[a] > score[b] or (score[a] == score[b] and a < b)

    for t in chosen:
        for u in range(s, n):
            if u not in chosen and not before(t, u):
                return False
    return True


def check_topk(o):
    case = _load("codebook_d4.json")["cases"][0]
    sc = np.array([(-np.inf if v is None else v) for v in case["scores"]])
    for k, want in case["topk"].items():
        assert o.topk(sc, int(k), case["num_sinks"]).tolist() == want
    rng = np.random.default_rng(16)
    for trial in range(60):
        n = int(rng.integers(1, 24))
        s = int(rng.integers(0, min(n, 5) + 1))
        score = rng.integers(-3, 4, size=n).astype(np.float64)   # many exact ties
        score[rng.random(n) < 0.2] = -0.0
        k = int(rng.integers(0, n - s + 1))
        got = o.topk(score, k, s)
        assert list(got) == sorted(got)
        assert _is_topk_by_definition(score, got, k, s), (score, s, k, got)


# --------------------------------------------------------------------------
# sparse attention (§2.1 items 3 and 4)
# --------------------------------------------------------------------------

def check_attention_golden(o):
    case = _load("codebook_d4.json")["cases"][0]
    K = np.asarray(case["keys"], dtype=np.float64)
    V = np.asarray(case["values"], dtype=np.float64)
    s = case["num_sinks"]
    mu, code, cent, _ = o.encode_keys(K, s)
    q = np.asarray(case["queries"])
    out = o.sparse_attention(q, K, V, mu, cent, code, np.array([1, 2]), s)
    assert np.allclose(out, case["attention_k2"]["out"], rtol=0, atol=1e-15), out
    e = math.e
    assert np.allclose(out[0], np.array([1, e, 1, 0]) / (2 + e), rtol=0, atol=1e-15)


def check_attention_full_selection_is_dense(o):
    """k = N - S with exact reconstruction equals dense softmax attention over K itself."""
    import torch

    for s in (0, 2):
        K, _ = _distinct_pattern_keys(s, seed=17)
        rng = np.random.default_rng(18)
        V = rng.standard_normal(K.shape)
        q = rng.standard_normal((3, K.shape[1]))
        mu, code, cent, _ = o.encode_keys(K, s)
        idx = np.arange(s, K.shape[0])
        out = o.sparse_attention(q, K, V, mu, cent, code, idx, s)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[None, :, None, :], torch.from_numpy(K)[None, None].expand(1, 3, -1, -1),
            torch.from_numpy(V)[None, None].expand(1, 3, -1, -1))[0, :, 0].numpy()
        assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)


def check_attention_invariants(o):
    w = gen.small(0, n=400)
    hi = gen.head_inputs(w, 0, 0)
    K = gen.storage_to_f64(hi.keys, w.dtype)
    V = gen.storage_to_f64(hi.values, w.dtype)
    mu, code, cent, _ = o.encode_keys(K, w.num_sinks)
    # no sinks, one selected token: the output is that token's value row
    out = o.sparse_attention(np.ones((1, 128)), K, V, mu, cent, code, np.array([123]), 0)
    assert np.allclose(out[0], V[123], rtol=0, atol=1e-12)
    # a zero query averages the value rows of sinks + selected uniformly
    idx = np.array([70, 80, 399])
    out = o.sparse_attention(np.zeros((2, 128)), K, V, mu, cent, code, idx, w.num_sinks)
    rows = np.concatenate([V[:w.num_sinks], V[idx]])
    assert np.allclose(out, rows.mean(axis=0)[None, :].repeat(2, 0), rtol=0, atol=1e-12)
    # selection order does not matter
    a = o.sparse_attention(np.ones((1, 128)), K, V, mu, cent, code, idx, w.num_sinks)
    b = o.sparse_attention(np.ones((1, 128)), K, V, mu, cent, code, idx[::-1], w.num_sinks)
    assert np.allclose(a, b, rtol=0, atol=1e-12)


def check_needle_recall(o):
    """Planted needle keys are recalled by the compressed-domain selection."""
    w = gen.config(0)
    hi = gen.head_inputs(w, 0, 0)
    K = gen.storage_to_f64(hi.keys, w.dtype)
    q = gen.storage_to_f64(hi.queries[0], w.dtype)
    mu, code, cent, _ = o.encode_keys(K, w.num_sinks)
    sc, _ = o.scores(q, mu, cent, code, w.num_sinks)
    idx = o.topk(sc, w.topk[0], w.num_sinks)
    assert set(hi.needle_pos.tolist()) <= set(idx.tolist())



# --------------------------------------------------------------------------
# one decode step: score, select, attend (§2.1 items 2-4), composed
# --------------------------------------------------------------------------

def check_decode_step_golden(o):
    """The composed step on the hand-worked D = 4 case with one sink.

    k = 2 selects {1, 2} and reproduces the worked attention output; k = 3
    selects {1, 2, 4}; a softmax scale of 1 instead of 1/sqrt(D) doubles the
    logits.  Closed forms, worked by hand from the fixture's keys (token t's
    reconstructed key is 2 e_{t-1} for t = 1..4, the sink's key is 0):
      scale 1/2, k = 3: head 0 logits (0, 1, 0, 0) over tokens (0, 1, 2, 4)
        -> [2, e + 1, 2, 1] / (3 + e); head 1 logits (0, 0, 1, 1)
        -> [1 + e, 1 + e, 2 e, e] / (2 + 2 e);
      scale 1, k = 2: head 0 -> [1, e^2, 1, 0] / (2 + e^2),
        head 1 -> [1, 1, e^2, 0] / (2 + e^2)."""
    case = _load("codebook_d4.json")["cases"][0]
    K = np.asarray(case["keys"], dtype=np.float64)
    V = np.asarray(case["values"], dtype=np.float64)
    q = np.asarray(case["queries"], dtype=np.float64)
    s = case["num_sinks"]
    mu, code, cent, _ = o.encode_keys(K, s)
    out, idx, sc, _ = o.decode_step(q, K, V, mu, cent, code, 2, s)
    assert list(idx) == case["topk"]["2"]
    assert np.isneginf(sc[0]) and np.allclose(sc[1:], case["scores"][1:], rtol=0, atol=1e-15)
    assert np.allclose(out, case["attention_k2"]["out"], rtol=0, atol=1e-15), out
    e = math.e
    out3, idx3, _, _ = o.decode_step(q, K, V, mu, cent, code, 3, s)
    assert list(idx3) == case["topk"]["3"]
    want3 = np.array([[2, e + 1, 2, 1], [1 + e, 1 + e, 2 * e, e]]) / np.array([[3 + e], [2 + 2 * e]])
    assert np.allclose(out3, want3, rtol=0, atol=1e-15), out3
    out_s1, _, _, _ = o.decode_step(q, K, V, mu, cent, code, 2, s, scale=1.0)
    e2 = math.exp(2.0)
    want_s1 = np.array([[1, e2, 1, 0], [1, 1, e2, 0]]) / (2 + e2)
    assert np.allclose(out_s1, want_s1, rtol=0, atol=1e-15), out_s1


def _embed_d4_case(o, d=128):
    """The D = 4 fixture embedded in D = 128: the extra key channels are 0
    (their codes are all 15 and their centroids 0, so scores and logits are
    unchanged) and the value rows get an exactly representable 2-bit grid."""
    case = _load("codebook_d4.json")["cases"][0]
    K4 = np.asarray(case["keys"], dtype=np.float64)
    n = K4.shape[0]
    K = np.zeros((n, d))
    K[:, :4] = K4
    q = np.zeros((2, d))
    q[:, :4] = np.asarray(case["queries"], dtype=np.float64)
    rng = np.random.default_rng(44)
    grid = rng.integers(0, 4, (n, d)).astype(np.float64)
    grid[:, ::32] = 0.0
    grid[:, 1::32] = 3.0
    V = 0.5 + 0.25 * grid
    return case, K, V, q


def check_decode_step_qv(o):
    """The 2-bit step: with values on the exact 2-bit grid it equals the
    full-precision step (selection included) for any k, sink count and
    scale; with off-grid values the selection is unchanged and the output
    moves by at most the largest read-back error of a selected row."""
    case, K, V, q = _embed_d4_case(o)
    s = case["num_sinks"]
    mu, code, cent, _ = o.encode_keys(K, s)
    packed = o.quantize_values(V)
    for k, scale in ((2, None), (3, None), (2, 1.0), (4, 0.25)):
        a, ia, _, _ = o.decode_step(q, K, V, mu, cent, code, k, s, scale)
        b, ib, _, _ = o.decode_step_qv(q, K, V, packed, mu, cent, code, k, s, scale)
        assert list(ia) == list(ib) == sorted(case["topk"][str(k)])
        assert np.allclose(a, b, rtol=0, atol=1e-15)
    rng = np.random.default_rng(45)
    Vr = rng.standard_normal(V.shape).astype(np.float32).astype(np.float64)
    pr = o.quantize_values(Vr)
    a, ia, _, _ = o.decode_step(q, K, Vr, mu, cent, code, 3, s, 1.0)
    b, ib, _, _ = o.decode_step_qv(q, K, Vr, pr, mu, cent, code, 3, s, 1.0)
    worst = np.abs(o.dequantize_values(pr) - Vr)[ia].max()
    assert list(ia) == list(ib) and np.all(np.abs(a - b) <= worst + 1e-12)
    assert not np.allclose(a, b, rtol=0, atol=1e-9)
    # with nothing selected only the full-precision sink is attended
    c, _, _, _ = o.decode_step_qv(q, K, Vr, pr, mu, cent, code, 0, s)
    assert np.allclose(c, Vr[0][None, :].repeat(2, 0), rtol=0, atol=1e-15)

# --------------------------------------------------------------------------
# decode-time append (R19, R20: frozen prefill mean and codebook)
# --------------------------------------------------------------------------

def check_append_by_construction(o):
    """Appended rows carry the sign patterns their keys were built with,
    relative to the prefill mean; the other rows are untouched.  Heavy
    appended keys would drag a re-estimated mean far enough to flip the
    small-margin bits, so a mean that moves with the appends is caught."""
    rng = np.random.default_rng(19)
    d, s, n0, n_pat, n_heavy, n_tail = 16, 8, 80, 6, 6, 4
    K0 = rng.standard_normal((n0, d)).astype(np.float32).astype(np.float64)
    mu = o.channel_mean(K0, s)
    want = rng.integers(0, 16, size=(n_pat, d // 4))
    Kp = np.empty((n_pat, d))
    for t in range(n_pat):
        for sub in range(d // 4):
            for i in range(4):
                bit = (int(want[t, sub]) >> i) & 1
                mag = float(rng.uniform(0.01, 0.05))
                Kp[t, 4 * sub + i] = float(mu[4 * sub + i]) + (mag if bit else -mag)
    Kh = np.asarray(mu, dtype=np.float64)[None, :] + 50.0 * np.ones((n_heavy, d))
    Kt = rng.standard_normal((n_tail, d))
    K = np.concatenate([K0, Kp, Kh, Kt]).astype(np.float32).astype(np.float64)
    before = np.zeros((K.shape[0], d // 8), dtype=np.uint8)
    before[:n0] = o.pack_codes(o.sign_codes(K0, mu))
    before[n0 + n_pat + n_heavy:] = 0xA5
    got = o.append_codes(before, K, mu, n0, n_pat + n_heavy)
    assert np.array_equal(got[:n0], before[:n0])
    assert np.array_equal(got[n0 + n_pat + n_heavy:], before[n0 + n_pat + n_heavy:])
    assert np.array_equal(o.unpack_codes(got[n0:n0 + n_pat]), want)
    assert np.all(got[n0 + n_pat:n0 + n_pat + n_heavy] == 0xFF)
    assert np.array_equal(o.append_codes(before, K, mu, n0, 0), before)


def check_append_golden(o):
    """Appending the hand-worked D=8 vectors reproduces their fixture codes."""
    g = _load("sign_codes_d8.json")
    K = np.asarray(g["keys"], dtype=np.float32).astype(np.float64)
    mu = np.asarray(g["mu"], dtype=np.float32)
    n = K.shape[0]
    cache = np.full((n + 2, 1), 0x5A, dtype=np.uint8)
    Kc = np.concatenate([K, np.zeros((2, K.shape[1]))])
    got = o.append_codes(cache, Kc, mu, 0, n)
    assert got[:n].tolist() == g["packed"]
    assert got[n:].tolist() == [[0x5A], [0x5A]]


# --------------------------------------------------------------------------
# comparison baselines (dense scoring and dense attention, not the method)
# --------------------------------------------------------------------------

def check_dense_scores_equal_lut_scores_when_exact(o):
    """With one token per cluster the reconstruction is exact, so the
    compressed-domain score equals the full dot product q_bar . k."""
    s = 4
    K, _ = _distinct_pattern_keys(s, seed=21)
    rng = np.random.default_rng(22)
    q = rng.standard_normal((3, K.shape[1]))
    mu, code, cent, _ = o.encode_keys(K, s)
    lut_sc, _ = o.scores(q, mu, cent, code, s)
    dense = o.dense_scores(q, K, s)
    assert np.all(np.isneginf(dense[:s]))
    assert np.allclose(dense[s:], lut_sc[s:], rtol=1e-12, atol=1e-12)
    assert np.allclose(dense[s:], K[s:] @ q.sum(axis=0), rtol=0, atol=1e-12)


def check_dense_attention(o):
    import torch

    rng = np.random.default_rng(23)
    K = rng.standard_normal((300, 16))
    V = rng.standard_normal((300, 16))
    q = rng.standard_normal((4, 16))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], torch.from_numpy(K)[None, None].expand(1, 4, -1, -1),
        torch.from_numpy(V)[None, None].expand(1, 4, -1, -1))[0, :, 0].numpy()
    assert np.allclose(o.dense_attention(q, K, V), ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(o.dense_attention(q, K, V, 1)[0], V[0], rtol=0, atol=1e-12)       # one token
    assert np.allclose(o.dense_attention(np.zeros((2, 16)), K, V, 57), V[:57].mean(axis=0)[None].repeat(2, 0),
                       rtol=0, atol=1e-12)                                               # zero query: mean
    assert np.all(o.dense_attention(q, K, V, 0) == 0)




# --------------------------------------------------------------------------
# k-means codebook baseline (§2.1 item 1: the iterative clustering that the
# one-pass sign-pattern clustering replaces; §4: timed with 20 iterations)
# --------------------------------------------------------------------------

def _corner(j):
    return [1.0 if (j >> i) & 1 else -1.0 for i in range(4)]


def check_kmeans_golden(o):
    g = _load("kmeans_d8.json")
    s = g["num_sinks"]
    mu = np.array(g["mu"], dtype=np.float32)
    x = np.array(g["x"], dtype=np.float64).reshape(len(g["x"]), 8)
    K = x + mu.astype(np.float64)[None, :]
    want_cent = np.array([[_corner(j) for j in range(16)] for _ in range(2)], dtype=np.float32)
    for sub, cs in g["centroids_not_on_corner"].items():
        for j, c in cs.items():
            want_cent[int(sub), int(j)] = c
    for iters in g["iters"]:
        code, cent, counts = o.kmeans_codebook(K, mu, g["init_idx"], iters, s)
        assert np.array_equal(code, np.array(g["codes"], dtype=np.uint8)), iters
        assert np.array_equal(counts, np.array(g["counts"])), iters
        assert cent.dtype == np.float32 and np.array_equal(cent, want_cent), iters


def check_kmeans_update_exact(o):
    """A centroid is the exact mean rounded once: 2**30 + 2**-30 - 2**30 loses
    its middle term in any fp64 running sum."""
    x = np.zeros((3, 1, 4), dtype=np.float32)
    x[:, 0, 0] = [2.0 ** 30, 2.0 ** -30, -(2.0 ** 30)]
    x[:, 0, 1] = [1.0, 2.0, 4.0]
    x[:, 0, 2] = [0.1, 0.2, 0.3]
    cent0 = np.arange(64, dtype=np.float32).reshape(1, 16, 4)
    cent, counts = o.kmeans_update(x, np.zeros((3, 1), dtype=np.uint8), cent0)
    assert counts.tolist() == [[3] + [0] * 15]
    assert cent[0, 0, 0] == np.float32(float(Fraction(1, 3 * 2 ** 30)))
    assert cent[0, 0, 1] == np.float32(7.0 / 3.0)
    exact = sum(Fraction(float(v)) for v in x[:, 0, 2]) / 3
    assert abs(Fraction(float(cent[0, 0, 2])) - exact) <= Fraction(float(np.spacing(np.float32(0.2)))) / 2
    assert cent[0, 0, 3] == 0.0
    assert np.array_equal(cent[0, 1:], cent0[0, 1:])               # empty clusters keep theirs


def _kmeans_data(seed=31, n=400, s=3):
    rng = np.random.default_rng(seed)
    K = (rng.standard_normal((n + s, 8)) * 1.5 + rng.standard_normal(8)).astype(np.float32).astype(np.float64)
    mu = rng.standard_normal(8).astype(np.float32)
    init = rng.choice(np.arange(s, n + s), size=16, replace=False)
    return K, mu, init, s


def check_kmeans_matches_sklearn(o):
    """Lloyd's iterations from the same start agree with scikit-learn's
    KMeans (lloyd, fp64, no early stop) on points with no empty cluster."""
    from sklearn.cluster import KMeans

    K, mu, init, s = _kmeans_data()
    x = (K.astype(np.float32)[s:] - mu[None, :]).astype(np.float64)
    for iters in (1, 3):
        code, cent, counts = o.kmeans_codebook(K, mu, init, iters, s)
        assert np.all(counts > 0)
        for sub in range(2):
            pts = x[:, 4 * sub:4 * sub + 4]
            km = KMeans(n_clusters=16, init=pts[init - s], n_init=1, max_iter=iters, tol=0.0,
                        algorithm="lloyd").fit(pts)
            assert np.allclose(cent[sub], km.cluster_centers_, rtol=0, atol=1e-5), (iters, sub)


def check_kmeans_lloyd_invariants(o):
    """Cluster sizes add up to n, every centroid is the mean of its points, the
    codes of sinks are 0, and the within-cluster sum of squares never grows
    from one iteration to the next."""
    K, mu, init, s = _kmeans_data(seed=37)
    x = (K.astype(np.float32)[s:] - mu[None, :]).astype(np.float64)
    prev = None
    for iters in range(1, 7):
        code, cent, counts = o.kmeans_codebook(K, mu, init, iters, s)
        assert np.all(code[:s] == 0) and np.all(counts.sum(axis=1) == x.shape[0])
        sse = 0.0
        for sub in range(2):
            pts = x[:, 4 * sub:4 * sub + 4]
            lab = code[s:, sub]
            assert np.array_equal(np.bincount(lab, minlength=16), counts[sub])
            for j in range(16):
                if counts[sub, j]:
                    assert np.allclose(cent[sub, j], pts[lab == j].mean(axis=0), rtol=1e-6, atol=1e-6)
            sse += float(((pts - cent[sub][lab].astype(np.float64)) ** 2).sum())
        assert prev is None or sse <= prev * (1 + 1e-6), (iters, sse, prev)
        prev = sse



# --------------------------------------------------------------------------
# 2-bit values (§3 and §4: accuracy kept with 2-bit quantization, the memory
# saving of 2-bit KIVI; the scheme is a reading of this repository)
# --------------------------------------------------------------------------

def _golden_value_row():
    g = _load("values_2bit_d128.json")
    row = np.zeros(128, dtype=np.float32)
    row[0:32] = np.tile(np.float32(g["row"]["group0"]), 8)
    row[32:64] = g["row"]["group1"][0]
    row[64:96] = np.tile(np.float32([-1.0, -1.0 / 3.0, 1.0 / 3.0, 1.0]), 8)
    row[96:128] = np.tile(np.float32(g["row"]["group3"]), 4)
    return g, row.astype(np.float64)


def check_values_golden(o):
    g, row = _golden_value_row()
    packed = o.quantize_values(row[None])
    assert packed.dtype == np.uint8 and packed.shape == (1, 48)
    assert packed[0].tolist() == g["packed"]
    back = o.dequantize_values(packed)[0]
    rb = g["read_back"]
    assert back[0:32].tolist() == list(map(float, rb["group0"])) * 8
    assert back[32:64].tolist() == rb["group1"] * 32
    assert back[64:96].tolist() == rb["group2"] * 8
    assert back[96:128].tolist() == list(map(float, rb["group3"])) * 4


def check_values_error_bound(o):
    """Every value reads back within half a step of itself (plus the fp16
    rounding of the group's minimum and step); a group's minimum reads back as
    its fp16 minimum; values on an exact fp16 grid read back exactly."""
    rng = np.random.default_rng(41)
    V = (rng.standard_normal((300, 128)) * rng.uniform(0.1, 10.0, (300, 1))).astype(np.float32).astype(np.float64)
    back = o.dequantize_values(o.quantize_values(V))
    G = V.reshape(300, 4, 32)
    lo, hi = G.min(axis=2), G.max(axis=2)
    m16 = lo.astype(np.float16).astype(np.float64)
    s = (hi - lo) / 3.0
    s16 = s.astype(np.float16).astype(np.float64)
    bound = s16 / 2 + np.abs(lo - m16) + 3 * np.abs(s - s16) + 1e-6 * np.abs(G).max(axis=2)
    err = np.abs(back.reshape(300, 4, 32) - G).max(axis=2)
    assert np.all(err <= bound)
    amin = G.argmin(axis=2)
    assert np.array_equal(np.take_along_axis(back.reshape(300, 4, 32), amin[..., None], 2)[..., 0], m16)
    grid = rng.integers(0, 4, (50, 128)).astype(np.float64)
    grid[:, ::32] = 0.0
    grid[:, 1::32] = 3.0                                    # every group spans the four levels
    Vg = -2.5 + 0.75 * grid
    assert np.array_equal(o.dequantize_values(o.quantize_values(Vg)), Vg)


def check_values_attention(o):
    """Sinks keep full-precision values: with nothing selected the 2-bit
    attention equals the full-precision one for any values; with values on
    an exact grid it equals it for any selection; otherwise the outputs differ
    by at most the largest read-back error (softmax weights form a convex
    combination)."""
    rng = np.random.default_rng(43)
    s, n, d = 4, 60, 128
    K = rng.standard_normal((n, d))
    V = (rng.standard_normal((n, d)) * 3).astype(np.float32).astype(np.float64)
    q = rng.standard_normal((2, d))
    mu, code, cent, _ = o.encode_keys(K, s)
    packed = o.quantize_values(V)
    none = np.zeros(0, dtype=np.int64)
    assert np.allclose(o.sparse_attention_qv(q, K, V, packed, mu, cent, code, none, s),
                       o.sparse_attention(q, K, V, mu, cent, code, none, s), rtol=0, atol=1e-12)
    idx = np.arange(s, n, 3)
    full = o.sparse_attention(q, K, V, mu, cent, code, idx, s)
    qv = o.sparse_attention_qv(q, K, V, packed, mu, cent, code, idx, s)
    worst = np.abs(o.dequantize_values(packed) - V)[idx].max()
    assert np.all(np.abs(qv - full) <= worst + 1e-12) and not np.allclose(qv, full, rtol=0, atol=1e-9)
    grid = rng.integers(0, 4, (n, d)).astype(np.float64)
    grid[:, ::32] = 0.0
    grid[:, 1::32] = 3.0
    Vg = 1.25 + 0.5 * grid
    assert np.allclose(o.sparse_attention_qv(q, K, Vg, o.quantize_values(Vg), mu, cent, code, idx, s),
                       o.sparse_attention(q, K, Vg, mu, cent, code, idx, s), rtol=0, atol=1e-12)

ALL_CHECKS = [
    check_exact_sum, check_round_to_f32, check_channel_mean, check_sign_codes_golden,
    check_codes_by_construction, check_codebook_golden, check_codebook_invariants,
    check_one_member_clusters_reconstruct, check_scores_golden, check_lut_identity,
    check_topk, check_attention_golden, check_attention_full_selection_is_dense,
    check_attention_invariants, check_needle_recall, check_decode_step_golden, check_decode_step_qv, check_append_by_construction, check_append_golden,
    check_dense_scores_equal_lut_scores_when_exact, check_dense_attention,
    check_kmeans_golden, check_kmeans_update_exact, check_kmeans_matches_sklearn,
    check_kmeans_lloyd_invariants, check_values_golden, check_values_error_bound, check_values_attention,
]
