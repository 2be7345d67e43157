"""Checks that tie the CPU oracle to something other than itself.

Each pin takes the oracle module as an argument so that the mutation tests
can run the same checks against copies of the oracle with a planted mistake.
A pin raises AssertionError (or any exception) when the oracle is wrong.

What pins what:
* scores, scale, head maps, append, softmax and value sum: the dense case
  (N >= L) must equal torch's scaled_dot_product_attention in float64, a
  library routine, with K and V heads expanded by repeat_interleave (the
  contiguous grouping), the appended token included;
* threshold + comparison: brute-force top-N by np.argsort on tiny rows, and
  the count |S| = N at every step when the threshold is refreshed every step
  on tie-free data;
* tie rule: every score equal to the threshold is kept;
* stale-threshold reuse: a two-step example worked out by hand (closed form);
* the stand-alone refresh threshold: brute-force exact scores (math.fsum) and a Python sort, with
  ties; it also equals what a refresh step stores;
* capacity growth: a layer that outgrows its initial capacity matches one created large enough;
* softmax / value sum: constant value rows give that constant; each output
  coordinate lies between the kept rows' extremes; a single kept token gives
  its value row; an empty selection gives zero;
* byte model: the explainer's vector-read table.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _bf16(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def _rand(rng, shape):
    return _bf16(rng.standard_normal(shape))


def _sdpa(q, K, V, h_q):
    """torch SDPA (float64, CPU) for one query token; K/V heads expanded by repeat_interleave."""
    B, h_k, L, d = K.shape
    h_v = V.shape[1]
    Kt = torch.as_tensor(K, dtype=torch.float64).repeat_interleave(h_q // h_k, dim=1)
    Vt = torch.as_tensor(V, dtype=torch.float64).repeat_interleave(h_q // h_v, dim=1)
    qt = torch.as_tensor(q, dtype=torch.float64)[:, :, None, :]
    return torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt)[:, :, 0, :].numpy()


def pin_dense_matches_sdpa(o, h_q=8, h_k=2, h_v=4, d=64, l_kv=37, B=2, seed=0):
    """N >= L: the step is plain attention over all cached tokens (eqs. 2-4)."""
    rng = np.random.default_rng(seed)
    k0, v0 = _rand(rng, (B, h_k, l_kv, d)), _rand(rng, (B, h_v, l_kv, d))
    layer = o.OracleLayer(k0, v0, h_q, n_top=10 ** 9, refresh=3)
    Kall, Vall = k0, v0
    for _ in range(3):
        q = _rand(rng, (B, h_q, d))
        kn, vn = _rand(rng, (B, h_k, d)), _rand(rng, (B, h_v, d))
        res = layer.step(q, kn, vn)
        Kall = np.concatenate([Kall, kn[:, :, None]], axis=2)
        Vall = np.concatenate([Vall, vn[:, :, None]], axis=2)
        ref = _sdpa(q, Kall, Vall, h_q)
        assert res["keep"].all()
        np.testing.assert_allclose(res["out"], ref, rtol=0, atol=2e-6)


def pin_dense_cases(o):
    pin_dense_matches_sdpa(o, h_q=8, h_k=8, h_v=8, d=64, seed=1)     # MHA
    pin_dense_matches_sdpa(o, h_q=8, h_k=2, h_v=2, d=64, seed=2)     # GQA
    pin_dense_matches_sdpa(o, h_q=12, h_k=1, h_v=4, d=128, seed=3)   # SAGA, fewer key heads
    pin_dense_matches_sdpa(o, h_q=8, h_k=4, h_v=2, d=32, seed=4)     # more key than value heads


def pin_bruteforce_topn(o, trials=20):
    """Threshold refreshed every step: the kept set is exactly the N largest scores."""
    rng = np.random.default_rng(10)
    for trial in range(trials):
        B, h_q, h_k, h_v, d = 1, 4, 2, 4, 16
        l_kv = int(rng.integers(4, 60))
        n = int(rng.integers(1, l_kv))
        layer = o.OracleLayer(_rand(rng, (B, h_k, l_kv, d)), _rand(rng, (B, h_v, l_kv, d)), h_q, n, 1)
        for _ in range(3):
            res = layer.step(_rand(rng, (B, h_q, d)), _rand(rng, (B, h_k, d)), _rand(rng, (B, h_v, d)))
            A = res["scores"]
            for j in range(h_q):
                if len(np.unique(A[0, j])) != A.shape[2]:
                    continue  # ties: covered by pin_ties
                top = set(np.argsort(-A[0, j].astype(np.float64), kind="stable")[:n].tolist())
                assert set(np.nonzero(res["keep"][0, j])[0].tolist()) == top


def pin_exact_count(o):
    """R = 1 on tie-free data selects exactly N tokens per row at every step."""
    rng = np.random.default_rng(11)
    B, h_q, h_k, h_v, d, l_kv, n = 2, 8, 1, 8, 64, 300, 17
    layer = o.OracleLayer(_rand(rng, (B, h_k, l_kv, d)), _rand(rng, (B, h_v, l_kv, d)), h_q, n, 1)
    for _ in range(4):
        res = layer.step(_rand(rng, (B, h_q, d)), _rand(rng, (B, h_k, d)), _rand(rng, (B, h_v, d)))
        for b in range(B):
            for j in range(h_q):
                if len(np.unique(res["scores"][b, j])) == res["L"]:
                    assert res["keep"][b, j].sum() == n


def pin_ties(o):
    """The threshold is the N-th largest with multiplicity and all ties at it are kept."""
    # d = 4, scale 1/2; q = e0 so the score of a key is its first coordinate / 2
    k_first = np.array([6, 4, 4, 4, 2, 0], dtype=np.float32)
    k0 = np.zeros((1, 1, 6, 4), np.float32)
    k0[0, 0, :, 0] = k_first
    v0 = np.eye(6, 4, dtype=np.float32)[None, None]
    layer = o.OracleLayer(k0[:, :, :5], v0[:, :, :5], 1, n_top=2, refresh=1)
    res = layer.step(np.array([[[1, 0, 0, 0]]], np.float32), k0[:, :, 5], v0[:, :, 5])
    assert res["tau"][0, 0] == 2.0
    assert res["keep"][0, 0].tolist() == [True, True, True, True, False, False]
    # N = 4 ends the tied group, N = 5 falls below it; N >= L = 6 leaves no N-th largest to exclude anything
    for n, tau, cnt in ((4, 2.0, 4), (5, 1.0, 5), (6, -np.inf, 6), (7, -np.inf, 6)):
        layer = o.OracleLayer(k0[:, :, :5], v0[:, :, :5], 1, n_top=n, refresh=1)
        res = layer.step(np.array([[[1, 0, 0, 0]]], np.float32), k0[:, :, 5], v0[:, :, 5])
        assert res["tau"][0, 0] == tau and res["keep"][0, 0].sum() == cnt


def pin_stale_two_step(o):
    """A threshold from a refresh step is reused unchanged on the next (R = 2).

    d = 4 (scale 1/2), h_q = 2, h_k = 1, h_v = 2, N = 2.  Worked by hand:
      step 0 (refresh): head 0 scores [1,0,1,0] -> tau 1, keep {0,2};
                        head 1 scores [0,1,1,0] -> tau 1, keep {1,2}.
      step 1 (stale):   head 0 scores [2,0,2,0,1] >= 1 -> keep {0,2,4},
                        weights (e, e, 1)/(2e+1);
                        head 1 scores [0,0,0,1,0] >= 1 -> keep {3}.
    A fresh threshold at step 1 would keep {0,2} and {0..4} instead.
    """
    k0 = np.array([[[[2, 0, 0, 0], [0, 2, 0, 0], [2, 2, 0, 0]]]], np.float32)
    v0 = np.zeros((1, 2, 3, 4), np.float32)
    v0[0, 0] = [[1, 0, 0, 0], [0, 1, 0, 0], [0, 0, 1, 0]]
    v0[0, 1] = [[0, 1, 0, 0], [0, 0, 1, 0], [0, 0, 0, 1]]
    layer = o.OracleLayer(k0, v0, 2, n_top=2, refresh=2)
    r0 = layer.step(np.array([[[1, 0, 0, 0], [0, 1, 0, 0]]], np.float32),
                    np.array([[[0, 0, 0, 2]]], np.float32),
                    np.array([[[0, 0, 0, 1], [1, 0, 0, 0]]], np.float32))
    assert r0["refreshed"] and r0["tau"].tolist() == [[1.0, 1.0]]
    assert np.nonzero(r0["keep"][0, 0])[0].tolist() == [0, 2]
    assert np.nonzero(r0["keep"][0, 1])[0].tolist() == [1, 2]
    np.testing.assert_allclose(r0["out"][0], [[0.5, 0, 0.5, 0], [0, 0, 0.5, 0.5]], atol=1e-15)
    r1 = layer.step(np.array([[[2, 0, 0, 0], [0, 0, 0, 1]]], np.float32),
                    np.array([[[1, 0, 0, 0]]], np.float32),
                    np.array([[[0, 2, 0, 0], [0, 0, 2, 0]]], np.float32))
    assert not r1["refreshed"] and r1["tau"].tolist() == [[1.0, 1.0]]
    assert np.nonzero(r1["keep"][0, 0])[0].tolist() == [0, 2, 4]
    assert np.nonzero(r1["keep"][0, 1])[0].tolist() == [3]
    e = math.e
    np.testing.assert_allclose(r1["out"][0, 0], np.array([e, 2, e, 0]) / (2 * e + 1), atol=1e-14)
    np.testing.assert_allclose(r1["out"][0, 1], [1, 0, 0, 0], atol=1e-15)


def pin_softmax_invariants(o):
    """Constant value rows give the constant (weights sum to 1); outputs stay in the kept rows' range."""
    rng = np.random.default_rng(12)
    B, h_q, h_k, h_v, d, l_kv = 1, 6, 2, 3, 32, 200
    k0 = _rand(rng, (B, h_k, l_kv, d))
    v_const = np.full((B, h_v, l_kv, d), 0.75, np.float32)
    layer = o.OracleLayer(k0, v_const, h_q, 20, 4)
    for _ in range(5):
        res = layer.step(_rand(rng, (B, h_q, d)), _rand(rng, (B, h_k, d)), np.full((B, h_v, d), 0.75, np.float32))
        np.testing.assert_allclose(res["out"], 0.75, atol=1e-12)
    v0 = _rand(rng, (B, h_v, l_kv, d))
    layer = o.OracleLayer(k0, v0, h_q, 20, 4)
    for _ in range(5):
        res = layer.step(_rand(rng, (B, h_q, d)), _rand(rng, (B, h_k, d)), _rand(rng, (B, h_v, d)))
        for j in range(h_q):
            idx = np.nonzero(res["keep"][0, j])[0]
            rows = layer.v[0, (j * h_v) // h_q, idx]
            assert (res["out"][0, j] <= rows.max(0) + 1e-12).all()
            assert (res["out"][0, j] >= rows.min(0) - 1e-12).all()


def pin_single_and_empty(o):
    """N = 1 keeps one token (output = its value row); a stale threshold above every score keeps none (output 0)."""
    rng = np.random.default_rng(13)
    B, h_q, h_k, h_v, d, l_kv = 1, 2, 1, 2, 16, 40
    k0, v0 = _rand(rng, (B, h_k, l_kv, d)), _rand(rng, (B, h_v, l_kv, d))
    layer = o.OracleLayer(k0, v0, h_q, 1, 2)
    q = _rand(rng, (B, h_q, d))
    res = layer.step(q, _rand(rng, (B, h_k, d)), _rand(rng, (B, h_v, d)))
    for j in range(h_q):
        i = int(np.argmax(res["scores"][0, j]))
        assert np.nonzero(res["keep"][0, j])[0].tolist() == [i]
        np.testing.assert_array_equal(res["out"][0, j], layer.v[0, (j * h_v) // h_q, i].astype(np.float64))
    # next step: a zero query scores every token 0, below the stale (positive) threshold
    assert (res["tau"] > 0).all()
    res = layer.step(np.zeros_like(q), np.zeros((B, h_k, d), np.float32), _rand(rng, (B, h_v, d)))
    assert not res["keep"].any()
    assert (res["out"] == 0).all()


def pin_refresh_threshold_bruteforce(o):
    """The stand-alone refresh threshold is the N-th largest (with multiplicity) of the row's scores.

    Scores by brute force on a hand-made cache: K heads expanded to the query heads with
    repeat_interleave (the contiguous grouping), every dot product summed exactly with math.fsum
    (bf16 products are exact in float64; d = 16 makes the 1/sqrt(d) scale 0.25, exact too), rounded
    once to fp32, then sorted with Python's sort.  Integer-valued keys make ties at the threshold.
    The same threshold must also be what a refresh step of OracleLayer stores for the same inputs.
    """
    rng = np.random.default_rng(14)
    B, h_q, h_k, h_v, d, l_kv = 2, 6, 2, 3, 16, 23
    for trial in range(6):
        k0 = _bf16(np.round(rng.standard_normal((B, h_k, l_kv, d)) * 2) if trial % 2 else rng.standard_normal((B, h_k, l_kv, d)))
        v0 = _rand(rng, (B, h_v, l_kv, d))
        q = _bf16(np.round(rng.standard_normal((B, h_q, d)) * 2) if trial % 2 else rng.standard_normal((B, h_q, d)))
        kn, vn = _rand(rng, (B, h_k, d)), _rand(rng, (B, h_v, d))
        K = np.concatenate([k0, kn[:, :, None]], axis=2)
        L = l_kv + 1
        Kq = torch.as_tensor(K, dtype=torch.float64).repeat_interleave(h_q // h_k, dim=1).numpy()
        for n in (1, 3, 7, L - 1, L, L + 4):
            got = o.refresh_threshold(q, K, L, n)
            for b in range(B):
                for j in range(h_q):
                    row = [float(np.float32(math.fsum(float(q[b, j, c]) * float(Kq[b, j, i, c]) for c in range(d)) * 0.25))
                           for i in range(L)]
                    expect = sorted(row, reverse=True)[n - 1] if n < L else -math.inf
                    assert float(got[b, j]) == expect, (trial, n, b, j, float(got[b, j]), expect)
            layer = o.OracleLayer(k0, v0, h_q, n, 5)
            res = layer.step(q, kn, vn)
            assert res["refreshed"]
            np.testing.assert_array_equal(res["tau"], got)


def pin_capacity_growth(o):
    """A layer created with the default capacity grows past it and gives, step for step, the same
    thresholds, selections and outputs as one created large enough from the start."""
    rng = np.random.default_rng(15)
    B, h_q, h_k, h_v, d, l_kv, steps = 1, 4, 1, 2, 8, 12, 150
    k0, v0 = _rand(rng, (B, h_k, l_kv, d)), _rand(rng, (B, h_v, l_kv, d))
    grown = o.OracleLayer(k0, v0, h_q, 5, 7)
    big = o.OracleLayer(k0, v0, h_q, 5, 7, l_cap=l_kv + steps)
    for _ in range(steps):
        q, kn, vn = _rand(rng, (B, h_q, d)), _rand(rng, (B, h_k, d)), _rand(rng, (B, h_v, d))
        a, b = grown.step(q, kn, vn), big.step(q, kn, vn)
        for key in ("tau", "keep", "scores", "out"):
            np.testing.assert_array_equal(a[key], b[key])
    assert grown.length == l_kv + steps


def pin_vector_reads(o):
    with open(os.path.join(GOLDEN, "vector_reads_llama_128k.json")) as f:
        g = json.load(f)
    s = g["setup"]
    for row in g["rows"]:
        n = s["L"] if row["dense"] else s["n_top"]
        keys, values = o.vector_reads(s["h_q"], row["h_k"], row["h_v"], s["L"], n, s["batch"])
        assert (keys, values, keys + values) == (row["keys"], row["values"], row["total"])


ALL_PINS = [pin_dense_cases, pin_bruteforce_topn, pin_exact_count, pin_ties, pin_stale_two_step,
            pin_softmax_invariants, pin_single_and_empty, pin_refresh_threshold_bruteforce, pin_capacity_growth,
            pin_vector_reads]
