"""The QKV projection oracle against independent checks (no GPU).

* torch.nn.functional.linear in float64 with the three projections kept as
  separate weight matrices (a library routine on a different layout: it pins
  the packing, the head split and the order Q, K, V);
* a hand-made case: identity-like weights copy chosen input coordinates to
  known heads and dimensions;
* the append: only row pos of every head changes, to the rounded projection;
* rounding: the outputs are bf16 values, within 2^-8 relative (half a bf16 ulp) of the exact
  products;
plus planted mistakes (K and V swapped, heads interleaved, append at the
wrong row) that the checks catch.
"""
import importlib.util
import os

import numpy as np
import pytest
import torch

from oracle import qkv_oracle

ORACLE_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "qkv_oracle.py")


def _weights(rng, h_q, h_k, h_v, d, D):
    WQ = rng.standard_normal((D, h_q * d))
    WK = rng.standard_normal((D, h_k * d))
    WV = rng.standard_normal((D, h_v * d))
    return WQ, WK, WV, np.concatenate([WQ.T, WK.T, WV.T], axis=0)


def check_linear(o):
    rng = np.random.default_rng(41)
    for (B, h_q, h_k, h_v, d, D) in ((1, 8, 1, 8, 4, 16), (3, 12, 1, 4, 8, 24), (2, 8, 4, 2, 4, 12)):
        x = rng.standard_normal((B, D))
        WQ, WK, WV, W = _weights(rng, h_q, h_k, h_v, d, D)
        q, k, v = o.project(x, W, h_q, h_k, h_v, d)
        xt = torch.as_tensor(x)
        for got, Wm, h in ((q, WQ, h_q), (k, WK, h_k), (v, WV, h_v)):
            ref = torch.nn.functional.linear(xt, torch.as_tensor(Wm.T)).numpy().reshape(B, h, d)
            np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def check_hand_made(o):
    # D = 6, d = 2, h_q = 1, h_k = 1, h_v = 1: q = (x0, x1), k = (x2, x3), v = (2 x4, -x5)
    W = np.zeros((6, 6))
    W[0, 0] = W[1, 1] = W[2, 2] = W[3, 3] = 1.0
    W[4, 4] = 2.0
    W[5, 5] = -1.0
    x = np.array([[1.5, -2.0, 3.0, 0.25, 1.0, 4.0]])
    q, k, v = o.project(x, W, 1, 1, 1, 2)
    assert q.tolist() == [[[1.5, -2.0]]] and k.tolist() == [[[3.0, 0.25]]] and v.tolist() == [[[2.0, -4.0]]]


def check_append_and_rounding(o):
    rng = np.random.default_rng(42)
    B, h_q, h_k, h_v, d, D, l_cap, pos = 2, 8, 2, 4, 4, 20, 9, 6
    x = rng.standard_normal((B, D))
    _, _, _, W = _weights(rng, h_q, h_k, h_v, d, D)
    kc0, vc0 = rng.standard_normal((B, h_k, l_cap, d)), rng.standard_normal((B, h_v, l_cap, d))
    q, kc, vc = o.project_and_append(x, W, kc0, vc0, pos, h_q, h_k, h_v, d)
    qe, ke, ve = o.project(x, W, h_q, h_k, h_v, d)
    other = [r for r in range(l_cap) if r != pos]
    np.testing.assert_array_equal(kc[:, :, other], kc0[:, :, other])
    np.testing.assert_array_equal(vc[:, :, other], vc0[:, :, other])
    for got, exact in ((q, qe), (kc[:, :, pos], ke), (vc[:, :, pos], ve)):
        assert np.array_equal(torch.as_tensor(got).to(torch.bfloat16).double().numpy(), got)  # bf16 values
        assert np.all(np.abs(got - exact) <= np.abs(exact) * 2.0 ** -8 * (1 + 2.0 ** -15))


CHECKS = [check_linear, check_hand_made, check_append_and_rounding]


@pytest.mark.parametrize("check", CHECKS, ids=lambda f: f.__name__)
def test_qkv_oracle(check):
    check(qkv_oracle)


def _fresh(tag):
    spec = importlib.util.spec_from_file_location(f"_qkv_mutant_{tag}", ORACLE_PATH)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _m_swap_kv(o):
    orig = o.project

    def project(x, w, h_q, h_k, h_v, d):
        q, k, v = orig(x, w, h_q, h_k, h_v, d)
        if h_k == h_v:
            return q, v, k
        B = q.shape[0]
        y = np.concatenate([q.reshape(B, -1), v.reshape(B, -1), k.reshape(B, -1)], axis=1)
        return y[:, :h_q * d].reshape(B, h_q, d), y[:, h_q * d:(h_q + h_k) * d].reshape(B, h_k, d), \
            y[:, (h_q + h_k) * d:].reshape(B, h_v, d)
    o.project = project


def _m_interleaved_heads(o):
    orig = o.project

    def project(x, w, h_q, h_k, h_v, d):
        q, k, v = orig(x, w, h_q, h_k, h_v, d)
        return q.reshape(q.shape[0], d, h_q).transpose(0, 2, 1), k, v
    o.project = project


def _m_append_wrong_row(o):
    orig = o.project_and_append

    def project_and_append(x, w, kc, vc, pos, h_q, h_k, h_v, d):
        return orig(x, w, kc, vc, pos - 1, h_q, h_k, h_v, d)
    o.project_and_append = project_and_append


@pytest.mark.parametrize("mutate", [_m_swap_kv, _m_interleaved_heads, _m_append_wrong_row],
                         ids=lambda f: f.__name__[3:])
def test_planted_mistake_is_caught(mutate):
    o = _fresh(mutate.__name__)
    mutate(o)
    failed = 0
    for check in CHECKS:
        try:
            check(o)
        except Exception:  # noqa: BLE001
            failed += 1
    assert failed, mutate.__name__
