"""The CPU oracle against hand-worked examples, closed forms and invariants."""

import builtins
import copy
import types

import numpy as np
import pytest

import oracle
from tests import oracle_pins as pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(oracle)


def _mutant(**overrides):
    m = types.ModuleType("oracle_mutant")
    m.__dict__.update({k: v for k, v in vars(oracle).items() if not k.startswith("__")})
    m.__dict__["__builtins__"] = builtins          # the rebound functions look builtins up here
    m.__dict__.update(overrides)
    # rebind module-level helpers so composite functions use the mutated pieces
    for name, fn in list(vars(oracle).items()):
        if isinstance(fn, types.FunctionType) and name not in overrides:
            m.__dict__[name] = types.FunctionType(fn.__code__, m.__dict__, fn.__name__,
                                                  fn.__defaults__, fn.__closure__)
    return m


def _mut_codes_strict(K, mu):
    K = np.asarray(K, dtype=np.float64)
    mu = np.asarray(mu, dtype=np.float32).astype(np.float64)
    bits = (K > mu[None, :]).astype(np.uint8).reshape(K.shape[0], -1, 4)
    return (bits[..., 0] | bits[..., 1] << 1 | bits[..., 2] << 2 | bits[..., 3] << 3).astype(np.uint8)


def _mut_codes_msb_first(K, mu):
    K = np.asarray(K, dtype=np.float64)
    mu = np.asarray(mu, dtype=np.float32).astype(np.float64)
    bits = (K >= mu[None, :]).astype(np.uint8).reshape(K.shape[0], -1, 4)
    return (bits[..., 3] | bits[..., 2] << 1 | bits[..., 1] << 2 | bits[..., 0] << 3).astype(np.uint8)


def _mut_pack_swapped(code):
    code = np.asarray(code, dtype=np.uint8)
    return (code[:, 1::2] | (code[:, 0::2] << 4)).astype(np.uint8)


def _mut_mean_with_sinks(K, num_sinks=64):
    return oracle.channel_mean(K, 0)


def _mut_mean_fp64(K, num_sinks=64):
    K = np.asarray(K, dtype=np.float64)
    r = K[num_sinks:]
    if r.shape[0] == 0:
        return np.zeros(K.shape[1], dtype=np.float32)
    return (r.sum(axis=0) / r.shape[0]).astype(np.float32)


def _mut_lut_transposed(q_bar, centroids):
    p = centroids.shape[0]
    qs = np.asarray(q_bar, dtype=np.float64).reshape(p, 4)
    return np.einsum("si,sji->sj", qs[::-1], centroids)


def _mut_topk_ties_high(score, k, num_sinks=64):
    score = np.asarray(score, dtype=np.float64)
    cand = np.arange(num_sinks, score.shape[0])
    order = np.lexsort((-cand, -score[cand]))
    return np.sort(cand[order[:k]])


def _mut_no_sink_keys(q_group, K, V, mu, centroids, code, idx, num_sinks=64, scale=None):
    return oracle.sparse_attention(q_group, K, V, mu, centroids, code, idx, 0, scale)


def _mut_scores_no_qmu(q_group, mu, centroids, code, num_sinks=64):
    sc, cond = oracle.scores(q_group, np.zeros_like(mu), centroids, code, num_sinks)
    return sc, cond


def _mut_append_reestimates_mean(packed, K, mu, start, count):
    mu2 = oracle.channel_mean(np.asarray(K)[:start + count], 8)
    return oracle.append_codes(packed, K, mu2, start, count)


def _mut_append_one_row_too_many(packed, K, mu, start, count):
    return oracle.append_codes(packed, K, mu, start, count + 1) if start + count < np.asarray(K).shape[0] \
        else oracle.append_codes(packed, K, mu, start, count)


def _mut_kmeans_ties_high(x, cent):
    diff = x[:, :, None, :] - cent[None, :, :, :]
    sq = diff * diff
    dist = ((sq[..., 0] + sq[..., 1]) + sq[..., 2]) + sq[..., 3]
    return (15 - np.argmin(dist[:, :, ::-1], axis=2)).astype(np.uint8)


def _mut_kmeans_l1(x, cent):
    dist = np.abs(x[:, :, None, :] - cent[None, :, :, :]).sum(axis=3)
    return np.argmin(dist, axis=2).astype(np.uint8)


def _mut_kmeans_empty_zero(x, assign, cent):
    new, counts = oracle.kmeans_update(x, assign, cent)
    new[counts == 0] = 0.0
    return new, counts


def _mut_kmeans_fp64_mean(x, assign, cent):
    new = np.array(cent, dtype=np.float32, copy=True)
    counts = np.zeros((x.shape[1], 16), dtype=np.int64)
    for s in range(x.shape[1]):
        for j in range(16):
            m = x[assign[:, s] == j, s, :].astype(np.float64)
            counts[s, j] = m.shape[0]
            if m.shape[0]:
                new[s, j] = m.mean(axis=0).astype(np.float32)
    return new, counts


def _mut_kmeans_no_mu(K, mu, num_sinks=64):
    return oracle.kmeans_points(K, np.zeros_like(np.asarray(mu, dtype=np.float32)), num_sinks)


def _mut_kmeans_with_sinks(K, mu, init_idx, iters=20, num_sinks=64):
    code, cent, counts = oracle.kmeans_codebook(K, mu, init_idx, iters, 0)
    code[:num_sinks] = 0
    return code, cent, counts


def _mut_kmeans_one_short(K, mu, init_idx, iters=20, num_sinks=64):
    return oracle.kmeans_codebook(K, mu, init_idx, max(iters - 1, 1), num_sinks)


def _mut_values(level_fn=None, step_div=3.0, group=32, msb_first=False):
    def quantize(V):
        V32 = np.asarray(V, dtype=np.float64).astype(np.float32)
        n, d = V32.shape
        G = V32.reshape(n, d // group, group)
        lo, hi = G.min(axis=2), G.max(axis=2)
        m16, s16 = lo.astype(np.float16), ((hi - lo) / np.float32(step_div)).astype(np.float16)
        m32, s32 = m16.astype(np.float32)[..., None], s16.astype(np.float32)[..., None]
        with np.errstate(divide="ignore", invalid="ignore"):
            t = (G - m32) / s32
        r = level_fn(t) if level_fn else np.rint(t)
        lv = np.where(s32 > 0, np.clip(r, 0, 3), 0).astype(np.uint8).reshape(n, d // 4, 4)
        out = np.zeros((n, 48), dtype=np.uint8)
        sh = [6, 4, 2, 0] if msb_first else [0, 2, 4, 6]
        out[:, :d // 4] = (lv[..., 0] << sh[0]) | (lv[..., 1] << sh[1]) | (lv[..., 2] << sh[2]) | (lv[..., 3] << sh[3])
        prm = np.stack([m16, s16], axis=2).reshape(n, -1)[:, :8]
        out[:, d // 4:] = prm.view(np.uint8)
        return out
    return quantize


def _mut_values_sinks_quantized(q_group, K, V, packed, mu, centroids, code, idx, num_sinks=64, scale=None):
    Vq = oracle.dequantize_values(np.asarray(packed)[:np.asarray(V).shape[0]], np.asarray(V).shape[1])
    return oracle.sparse_attention(q_group, K, Vq, mu, centroids, code, idx, num_sinks, scale)



def _mut_decode_drops_sinks(q_group, K, V, mu, centroids, code, k, num_sinks=64, scale=None):
    sc, cond = oracle.scores(q_group, mu, centroids, code, num_sinks)
    idx = oracle.topk(sc, k, num_sinks)
    return oracle.sparse_attention(q_group, K, V, mu, centroids, code, idx, scale=scale), idx, sc, cond


def _mut_decode_drops_scale(q_group, K, V, mu, centroids, code, k, num_sinks=64, scale=None):
    return oracle.decode_step(q_group, K, V, mu, centroids, code, k, num_sinks)


def _mut_decode_qv_drops_sinks(q_group, K, V, packed, mu, centroids, code, k, num_sinks=64, scale=None):
    sc, cond = oracle.scores(q_group, mu, centroids, code, num_sinks)
    idx = oracle.topk(sc, k, num_sinks)
    out = oracle.sparse_attention_qv(q_group, K, V, packed, mu, centroids, code, idx, scale=scale)
    return out, idx, sc, cond


def _mut_decode_qv_drops_scale(q_group, K, V, packed, mu, centroids, code, k, num_sinks=64, scale=None):
    return oracle.decode_step_qv(q_group, K, V, packed, mu, centroids, code, k, num_sinks)

MUTATIONS = {
    "strict-greater": dict(sign_codes=_mut_codes_strict),
    "msb-first-bits": dict(sign_codes=_mut_codes_msb_first),
    "swapped-nibbles": dict(pack_codes=_mut_pack_swapped),
    "mean-includes-sinks": dict(channel_mean=_mut_mean_with_sinks),
    "mean-plain-fp64": dict(channel_mean=_mut_mean_fp64),
    "lut-wrong-subvector": dict(lut=_mut_lut_transposed),
    "ties-to-higher-index": dict(topk=_mut_topk_ties_high),
    "sinks-dropped": dict(sparse_attention=_mut_no_sink_keys),
    "dropped-q-dot-mu": dict(scores=_mut_scores_no_qmu),
    "append-reestimates-mean": dict(append_codes=_mut_append_reestimates_mean),
    "append-one-row-too-many": dict(append_codes=_mut_append_one_row_too_many),
    "kmeans-ties-to-higher-index": dict(kmeans_assign=_mut_kmeans_ties_high),
    "kmeans-l1-distance": dict(kmeans_assign=_mut_kmeans_l1),
    "kmeans-empty-cluster-to-zero": dict(kmeans_update=_mut_kmeans_empty_zero),
    "kmeans-plain-fp64-mean": dict(kmeans_update=_mut_kmeans_fp64_mean),
    "kmeans-no-mean-normalization": dict(kmeans_points=_mut_kmeans_no_mu),
    "kmeans-clusters-sinks": dict(kmeans_codebook=_mut_kmeans_with_sinks),
    "kmeans-one-iteration-short": dict(kmeans_codebook=_mut_kmeans_one_short),
    "values-round-half-up": dict(quantize_values=_mut_values(level_fn=lambda t: np.floor(t + np.float32(0.5)))),
    "values-step-over-4": dict(quantize_values=_mut_values(step_div=4.0)),
    "values-levels-msb-first": dict(quantize_values=_mut_values(msb_first=True)),
    "values-groups-of-16": dict(quantize_values=_mut_values(group=16)),
    "values-sinks-quantized": dict(sparse_attention_qv=_mut_values_sinks_quantized),
    "decode-drops-num-sinks": dict(decode_step=_mut_decode_drops_sinks),
    "decode-drops-scale": dict(decode_step=_mut_decode_drops_scale),
    "decode-qv-drops-num-sinks": dict(decode_step_qv=_mut_decode_qv_drops_sinks),
    "decode-qv-drops-scale": dict(decode_step_qv=_mut_decode_qv_drops_scale),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name):
    """A plausible mistake planted in the oracle fails at least one pin."""
    m = _mutant(**MUTATIONS[name])
    failures = []
    for check in pins.ALL_CHECKS:
        try:
            check(m)
        except AssertionError:
            failures.append(check.__name__)
    assert failures, f"mutation {name} passed every pin"
