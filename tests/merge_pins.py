"""Checks that tie the key-head merge oracle to something other than itself.

Each pin takes the oracle module as an argument (the mutation tests run the
same pins against copies with a planted mistake) and raises on a mismatch.

* Lemma 4.1 (eq. 15) against brute force: eq. 13 is a sum of squares of
  linear functions of M, so its minimiser also comes from np.linalg.lstsq on
  the vectorised system (every logit of every query head of both key heads);
* closed forms: merging a head with itself gives M = W and zero loss; with
  S_a = S_b = c I the merge is the mean (W_a + W_b) / 2 and the loss is
  c / 2 * ||X (W_a - W_b)||_F^2;
* a rank-deficient S (queries in a subspace): the pseudoinverse form reaches
  the same minimum value as least squares;
* the loss written through the Gram matrices, tr(D S D^T X^T X) summed over
  both heads with D = M - W_r, equals the definition for any M;
* Theorem 4.2: the enumerated matching against a bitmask dynamic program (a
  different algorithm) on random weights, and hand-made weights with a
  known unique optimum.
"""
from __future__ import annotations

import itertools

import numpy as np


def _case(rng, T=12, D=5, d=3, h_q=4, h_k=2):
    X = rng.standard_normal((T, D))
    Q = rng.standard_normal((T, h_q, d))
    W = rng.standard_normal((h_k, D, d))
    return X, Q, W, h_q, h_k


def _lstsq_merge(X, Q, W, a, b, h_q, h_k):
    """argmin_M of eq. 13 by least squares over vec(M): logits Q^j M^T X^T are linear in M."""
    D, d = W[a].shape
    rows, rhs = [], []
    for r in (a, b):
        for j in range(h_q):
            if (j * h_k) // h_q != r:
                continue
            Qj = Q[:, j, :]
            target = Qj @ (X @ W[r]).T  # [T, T]
            # logit[t, s] = sum_{k, c} Qj[t, c] * X[s, k] * M[k, c]
            A = np.einsum("tc,sk->tskc", Qj, X).reshape(-1, D * d)
            rows.append(A)
            rhs.append(target.reshape(-1))
    sol, *_ = np.linalg.lstsq(np.concatenate(rows), np.concatenate(rhs), rcond=None)
    return sol.reshape(D, d)


def pin_merge_matches_least_squares(o):
    rng = np.random.default_rng(31)
    for trial in range(4):
        X, Q, W, h_q, h_k = _case(rng, T=10 + trial, D=4 + trial % 2, d=3, h_q=4, h_k=2)
        M = o.merged_projection(Q, W, 0, 1, h_q, h_k)
        ref = _lstsq_merge(X, Q, W, 0, 1, h_q, h_k)
        np.testing.assert_allclose(M, ref, rtol=0, atol=1e-8)
        assert o.pair_loss(X, Q, W, 0, 1, M, h_q, h_k) <= o.pair_loss(X, Q, W, 0, 1, ref, h_q, h_k) + 1e-8


def pin_merge_identical_heads(o):
    rng = np.random.default_rng(32)
    X, Q, W, h_q, h_k = _case(rng)
    W = np.stack([W[0], W[0]])
    M = o.merged_projection(Q, W, 0, 1, h_q, h_k)
    np.testing.assert_allclose(M, W[0], rtol=0, atol=1e-10)
    assert abs(o.pair_loss(X, Q, W, 0, 1, M, h_q, h_k)) < 1e-18 * (1 + np.sum(X * X)) + 1e-20


def pin_merge_scaled_identity(o):
    """S_a = S_b = c I: every query head of a group is sqrt(c / g) [I_d; 0]."""
    rng = np.random.default_rng(33)
    T, D, d, h_q, h_k, c = 9, 4, 3, 4, 2, 2.5
    g = h_q // h_k
    Qj = np.zeros((T, d))
    Qj[:d, :d] = np.eye(d) * np.sqrt(c / g)
    Q = np.repeat(Qj[:, None, :], h_q, axis=1)
    X = rng.standard_normal((T, D))
    W = rng.standard_normal((h_k, D, d))
    M = o.merged_projection(Q, W, 0, 1, h_q, h_k)
    np.testing.assert_allclose(M, (W[0] + W[1]) / 2, rtol=0, atol=1e-12)
    expect = c / 2 * float(np.sum((X @ (W[0] - W[1])) ** 2))
    np.testing.assert_allclose(o.pair_loss(X, Q, W, 0, 1, M, h_q, h_k), expect, rtol=1e-12)


def pin_merge_rank_deficient(o):
    """Queries confined to a 2-dimensional subspace of d = 4: S is singular; the pseudoinverse merge still
    reaches the least-squares minimum of eq. 13."""
    rng = np.random.default_rng(34)
    T, D, d, h_q, h_k = 10, 5, 4, 4, 2
    basis = rng.standard_normal((2, d))
    Q = rng.standard_normal((T, h_q, 2)) @ basis
    X = rng.standard_normal((T, D))
    W = rng.standard_normal((h_k, D, d))
    M = o.merged_projection(Q, W, 0, 1, h_q, h_k)
    ref = _lstsq_merge(X, Q, W, 0, 1, h_q, h_k)
    la, lb = o.pair_loss(X, Q, W, 0, 1, M, h_q, h_k), o.pair_loss(X, Q, W, 0, 1, ref, h_q, h_k)
    np.testing.assert_allclose(la, lb, rtol=1e-9, atol=1e-9)


def pin_loss_through_grams(o):
    rng = np.random.default_rng(35)
    X, Q, W, h_q, h_k = _case(rng, T=11, D=6, d=4, h_q=6, h_k=3)
    G = X.T @ X
    for a, b in itertools.combinations(range(h_k), 2):
        M = rng.standard_normal(W[0].shape)
        expect = 0.0
        for r in (a, b):
            S = sum(Q[:, j, :].T @ Q[:, j, :] for j in range(h_q) if (j * h_k) // h_q == r)
            Dm = M - W[r]
            expect += float(np.trace(Dm @ S @ Dm.T @ G))
        np.testing.assert_allclose(o.pair_loss(X, Q, W, a, b, M, h_q, h_k), expect, rtol=1e-10)


def _dp_matching(w):
    """Minimum-weight perfect matching by dynamic programming over subsets (lowest node paired first)."""
    n = w.shape[0]
    best = {0: 0.0}
    for mask in range(1, 1 << n):
        if bin(mask).count("1") % 2:
            continue
        a = (mask & -mask).bit_length() - 1
        rest = mask & ~(1 << a)
        v = None
        for b in range(a + 1, n):
            if rest >> b & 1:
                c = best[rest & ~(1 << b)] + w[a, b]
                v = c if v is None or c < v else v
        best[mask] = v
    return best[(1 << n) - 1]


def pin_matching(o):
    rng = np.random.default_rng(36)
    for n in (2, 4, 6, 8):
        for _ in range(5):
            A = rng.random((n, n))
            w = A + A.T
            pairs, total = o.min_weight_matching(w)
            assert sorted(x for p in pairs for x in p) == list(range(n))
            np.testing.assert_allclose(total, _dp_matching(w), rtol=1e-12)
    # a known unique optimum: (0, 3), (1, 5), (2, 4) cost 0, every other edge 1
    w = np.ones((6, 6))
    for a, b in ((0, 3), (1, 5), (2, 4)):
        w[a, b] = w[b, a] = 0.0
    pairs, total = o.min_weight_matching(w)
    assert sorted(tuple(sorted(p)) for p in pairs) == [(0, 3), (1, 5), (2, 4)] and total == 0.0


def pin_whole_merge(o):
    """key_head_merge: its weights are the pair losses at their merged projections, its pairing the optimum
    of those weights, its merged projections those of the chosen pairs."""
    rng = np.random.default_rng(37)
    X, Q, W, h_q, h_k = _case(rng, T=14, D=5, d=3, h_q=8, h_k=4)
    res = o.key_head_merge(X, Q, W, h_q)
    for a, b in itertools.combinations(range(h_k), 2):
        ref = _lstsq_merge(X, Q, W, a, b, h_q, h_k)
        np.testing.assert_allclose(res["weights"][a, b], o.pair_loss(X, Q, W, a, b, ref, h_q, h_k), rtol=1e-8)
    np.testing.assert_allclose(res["total"], _dp_matching(res["weights"]), rtol=1e-12)
    for (a, b), M in zip(res["pairs"], res["merged"]):
        assert res["pairing"][a] == b and res["pairing"][b] == a
        np.testing.assert_allclose(M, _lstsq_merge(X, Q, W, a, b, h_q, h_k), rtol=0, atol=1e-8)


ALL_PINS = [pin_merge_matches_least_squares, pin_merge_identical_heads, pin_merge_scaled_identity,
            pin_merge_rank_deficient, pin_loss_through_grams, pin_matching, pin_whole_merge]
