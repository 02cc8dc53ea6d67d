"""The CPU oracle against hand-worked examples, closed forms and invariants."""

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
