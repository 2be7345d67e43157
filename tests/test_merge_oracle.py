"""The key-head merge oracle against its pins, and planted mistakes that the pins must catch (no GPU)."""
import importlib.util
import os

import numpy as np
import pytest

from oracle import merge_oracle
from tests import merge_pins

ORACLE_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "merge_oracle.py")


@pytest.mark.parametrize("pin", merge_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_merge_oracle_pin(pin):
    pin(merge_oracle)


def _fresh(tag):
    spec = importlib.util.spec_from_file_location(f"_merge_mutant_{tag}", ORACLE_PATH)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _m_one_sided_s(o):  # S_b left out of the pseudoinverse
    def merged_projection(Q, W, a, b, h_q, h_k):
        Sa, Sb = o.gram_s(Q, a, h_q, h_k), o.gram_s(Q, b, h_q, h_k)
        return (W[a] @ Sa + W[b] @ Sb) @ np.linalg.pinv(Sa, hermitian=True)
    o.merged_projection = merged_projection


def _m_plain_mean(o):  # the mean of the two projections instead of eq. 15
    o.merged_projection = lambda Q, W, a, b, h_q, h_k: (np.asarray(W[a]) + np.asarray(W[b])) / 2


def _m_interleaved_groups(o):
    o.key_head_of = lambda j, h_q, h_k: j % h_k


def _m_loss_one_head(o):  # eq. 13 without b's query heads
    orig = o.pair_loss

    def pair_loss(X, Q, W, a, b, M, h_q, h_k):
        return orig(X, Q, W, a, a, M, h_q, h_k) / 2
    o.pair_loss = pair_loss


def _m_max_matching(o):
    def min_weight_matching(w):
        best, best_total = None, None
        for m in o.perfect_matchings(range(w.shape[0])):
            total = sum(float(w[a, b]) for a, b in m)
            if best_total is None or total > best_total:
                best, best_total = m, total
        return best, best_total
    o.min_weight_matching = min_weight_matching


def _m_gram_transposed(o):  # Q^j Q^j^T contracted the wrong way (trace-preserving but wrong)
    def gram_s(Q, r, h_q, h_k):
        Q = np.asarray(Q, dtype=np.float64)
        d = Q.shape[2]
        S = np.zeros((d, d))
        for j in o.query_heads_of(r, h_q, h_k):
            S += np.diag(np.sum(Q[:, j, :] ** 2, axis=0))
        return S
    o.gram_s = gram_s


MUTANTS = [_m_one_sided_s, _m_plain_mean, _m_interleaved_groups, _m_loss_one_head, _m_max_matching,
           _m_gram_transposed]


@pytest.mark.parametrize("mutate", MUTANTS, ids=lambda f: f.__name__[3:])
def test_planted_mistake_is_caught(mutate):
    o = _fresh(mutate.__name__)
    mutate(o)
    failed = []
    for pin in merge_pins.ALL_PINS:
        try:
            pin(o)
        except Exception as e:  # noqa: BLE001 - any failure counts as caught
            failed.append((pin.__name__, type(e).__name__))
    assert failed, f"no pin caught {mutate.__name__}"
