"""Plant plausible mistakes in copies of the oracle; each must fail at least one pin.

The mistakes are planted in a private copy of the oracle module on the CPU;
the real oracle is untouched.
"""
import importlib.util
import os

import numpy as np
import pytest

from tests import oracle_pins

ORACLE_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "saga_oracle.py")


def _fresh_oracle(tag):
    spec = importlib.util.spec_from_file_location(f"_oracle_mutant_{tag}", ORACLE_PATH)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _m_key_head_mod(o):
    o.key_head = lambda j, h_q, h_k: np.asarray(j) % h_k


def _m_value_head_interleaved(o):
    o.value_head = lambda j, h_q, h_v: np.asarray(j) % h_v


def _m_no_scale(o):
    orig = o.scores

    def scores(q, k, L):
        return (orig(q, k, L).astype(np.float64) * np.sqrt(q.shape[-1])).astype(np.float32)
    o.scores = scores


def _m_negated_scores(o):
    orig = o.scores
    o.scores = lambda q, k, L: -orig(q, k, L)


def _m_nth_off_by_one(o):
    def nth_largest(row, n):
        row = np.asarray(row, np.float32)
        if n >= row.shape[0]:
            return o.NEG_INF
        return np.float32(np.sort(row)[::-1][min(n, row.shape[0] - 1)])
    o.nth_largest = nth_largest


def _m_strict_compare(o):
    o.select = lambda A, tau: A > tau[..., None]


def _m_refresh_every_step(o):
    o.is_refresh_step = lambda t, R: True


def _m_refresh_wrong_phase(o):
    o.is_refresh_step = lambda t, R: t % R == R - 1


def _m_unnormalised(o):
    orig = o.sparse_attention

    def sparse_attention(A, keep, v, L):
        out = orig(A, keep, v, L)
        return out * np.maximum(1, keep.sum(-1))[..., None] ** 0.5
    o.sparse_attention = sparse_attention


def _m_append_off_by_one(o):
    def kv_append(k, v, kn, vn, pos):
        k[:, :, pos + 1] = kn
        v[:, :, pos + 1] = vn
    o.kv_append = kv_append


def _m_dense_threshold_min(o):
    # N == L read as "the N-th largest is the minimum" instead of "no threshold"
    def nth_largest(row, n):
        row = np.asarray(row, np.float32)
        if n > row.shape[0]:
            return o.NEG_INF
        return np.float32(np.sort(row)[::-1][n - 1])
    o.nth_largest = nth_largest


def _m_refresh_threshold_short_row(o):
    # the stand-alone refresh reads one token too few (the new token left out)
    o.refresh_threshold = lambda q, k, L, n: o.threshold(o.scores(q, k, L - 1), n)


def _m_grow_drops_rows(o):
    # growth reallocates the caches without carrying the cached rows over
    def _grow(self):
        if self.length < self.k.shape[2]:
            return
        pad = max(64, self.k.shape[2] // 4)
        self.k = np.zeros((*self.k.shape[:2], self.k.shape[2] + pad, self.k.shape[3]), np.float32)
        self.v = np.zeros((*self.v.shape[:2], self.v.shape[2] + pad, self.v.shape[3]), np.float32)
    o.OracleLayer._grow = _grow


MUTANTS = [_m_key_head_mod, _m_value_head_interleaved, _m_no_scale, _m_negated_scores, _m_nth_off_by_one,
           _m_strict_compare, _m_refresh_every_step, _m_refresh_wrong_phase, _m_unnormalised, _m_append_off_by_one,
           _m_dense_threshold_min, _m_refresh_threshold_short_row, _m_grow_drops_rows]


@pytest.mark.parametrize("mutate", MUTANTS, ids=lambda f: f.__name__[3:])
def test_planted_mistake_is_caught(mutate):
    o = _fresh_oracle(mutate.__name__)
    mutate(o)
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(o)
        except Exception as e:  # noqa: BLE001 - any failure counts as caught
            failed.append((pin.__name__, type(e).__name__))
    assert failed, f"no pin caught {mutate.__name__}"
