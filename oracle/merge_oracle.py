"""CPU oracle for the closed-form GQA-to-SAGA key-head merge.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import this module; the CUDA path never
calls it and shares no code with it.

What it restates (summary page "More Value per Key: Asymmetric Sparse
Attention for Faster LLM Decoding", Methodology > GQA-to-SAGA Conversion >
Stage 1: Closed-Form Initialization), in numpy float64:

* the pairwise loss of merging teacher key heads a and b into one key
  projection M (eq. 13): for every query head j of a, the squared Frobenius
  norm of Q^j (X M)^T - Q^j (X W_K^a)^T, plus the same over the query heads
  of b with W_K^b;
* the closed-form minimiser (Lemma 4.1, eq. 15):
  M(a, b) = (W_K^a S_a + W_K^b S_b) (S_a + S_b)^+, S_r = sum over the query
  heads j of r of Q^j^T Q^j, ^+ the Moore-Penrose pseudoinverse;
* the pairing of the teacher's key heads (Theorem 4.2, objective eq. 14): a
  minimum-weight perfect matching of the complete graph whose edge weights
  are w(a, b) = L_ab(M(a, b)), found by enumerating every perfect matching.

Shapes (this build's reading of the page's notation): X is [T, D] (the
calibration tokens' hidden states), W_K^r is [D, d] so that X W_K^r are the
keys of head r, Q^j is [T, d] (the queries of head j on the same tokens).
Query head j belongs to teacher key head floor(j * h_k / h_q) (contiguous
groups, as in GQA).  The student has h_k / 2 key heads (pairs, m = 2).
"""
from __future__ import annotations

import itertools

import numpy as np


def key_head_of(j, h_q, h_k):
    """Teacher key head of query head j (contiguous groups)."""
    return (j * h_k) // h_q


def query_heads_of(r, h_q, h_k):
    return [j for j in range(h_q) if key_head_of(j, h_q, h_k) == r]


def gram_s(Q, r, h_q, h_k):
    """S_r = sum over the query heads j of key head r of Q^j^T Q^j (Lemma 4.1).  Q: [T, h_q, d]."""
    Q = np.asarray(Q, dtype=np.float64)
    d = Q.shape[2]
    S = np.zeros((d, d))
    for j in query_heads_of(r, h_q, h_k):
        S += Q[:, j, :].T @ Q[:, j, :]
    return S


def pair_loss(X, Q, W, a, b, M, h_q, h_k):
    """Eq. 13: L_ab(M), written out from the definition (logits of every query head of a and of b)."""
    X = np.asarray(X, dtype=np.float64)
    Q = np.asarray(Q, dtype=np.float64)
    KM = X @ np.asarray(M, dtype=np.float64)  # keys under the merged projection, [T, d]
    total = 0.0
    for r in (a, b):
        Kr = X @ np.asarray(W[r], dtype=np.float64)
        for j in query_heads_of(r, h_q, h_k):
            diff = Q[:, j, :] @ KM.T - Q[:, j, :] @ Kr.T
            total += float(np.sum(diff * diff))
    return total


def merged_projection(Q, W, a, b, h_q, h_k):
    """Eq. 15: M(a, b) = (W_K^a S_a + W_K^b S_b)(S_a + S_b)^+, the pseudoinverse by numpy (hermitian)."""
    Sa, Sb = gram_s(Q, a, h_q, h_k), gram_s(Q, b, h_q, h_k)
    Wa, Wb = np.asarray(W[a], np.float64), np.asarray(W[b], np.float64)
    return (Wa @ Sa + Wb @ Sb) @ np.linalg.pinv(Sa + Sb, hermitian=True)


def perfect_matchings(nodes):
    """Every perfect matching of the complete graph on `nodes` (an even number), as lists of pairs."""
    nodes = list(nodes)
    if not nodes:
        yield []
        return
    a = nodes[0]
    for i in range(1, len(nodes)):
        b = nodes[i]
        rest = nodes[1:i] + nodes[i + 1:]
        for m in perfect_matchings(rest):
            yield [(a, b)] + m


def min_weight_matching(w):
    """Theorem 4.2: the perfect matching of minimum total weight over every perfect matching (ties: the one
    enumerated first).  w: symmetric [n, n].  Returns (pairs, total)."""
    n = w.shape[0]
    best, best_total = None, None
    for m in perfect_matchings(range(n)):
        total = sum(float(w[a, b]) for a, b in m)
        if best_total is None or total < best_total:
            best, best_total = m, total
    return best, best_total


def key_head_merge(X, Q, W, h_q):
    """The whole Stage-1 initialisation: every pair's merged projection and loss, the optimal pairing, and
    the merged projections of the chosen pairs.  W: [h_k, D, d].  Returns dict(weights [h_k, h_k] (diagonal
    0), pairing [h_k] (partner of each head), pairs (a < b, ascending a), merged [h_k / 2, D, d], total)."""
    h_k = len(W)
    w = np.zeros((h_k, h_k))
    M = {}
    for a, b in itertools.combinations(range(h_k), 2):
        M[(a, b)] = merged_projection(Q, W, a, b, h_q, h_k)
        w[a, b] = w[b, a] = pair_loss(X, Q, W, a, b, M[(a, b)], h_q, h_k)
    pairs, total = min_weight_matching(w)
    pairs = sorted((min(p), max(p)) for p in pairs)
    pairing = np.zeros(h_k, dtype=np.int64)
    for a, b in pairs:
        pairing[a], pairing[b] = b, a
    merged = np.stack([M[p] for p in pairs])
    return {"weights": w, "pairing": pairing, "pairs": pairs, "merged": merged, "total": total, "all_merged": M}
