"""CPU oracle for the SAGA + Atop-N single-token decode-attention step.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import this module.  The product path (the
CUDA library and its binding) never calls it, and it shares no code with it.

It is a plain, slow restatement of what the paper "More Value per Key:
Asymmetric Sparse Attention for Faster LLM Decoding" says one decode step
computes, written in numpy:

* KV cache append (the "KV cache" entry of the explainer's jargon list).
* scores A = q K^T / sqrt(d)                         (eq. 2)
* the Atop-N threshold: the N-th largest score of the row, refreshed exactly
  once every R decode steps and reused in between     (Atop-N, steps 1-2)
* selection i = { positions whose score is >= the threshold } (Atop-N step 1,
  the per-element comparison that stands in for TopN of eq. 6)
* O = softmax(A[i]) V[i]                              (eq. 7)
* separate key and value head counts h_k != h_v      (SAGA architecture)

Precision.  The decision "is this token kept?" is taken in fp32 on both the
GPU and here: A is the exact dot product of the bf16 inputs (formed in
float64, where every bf16 x bf16 product is exact) scaled by 1/sqrt(d) in
float64 and rounded once to fp32.  The threshold is an element of that fp32
row and the comparison is an fp32 comparison.  Softmax and the value sum are
float64.

Readings where the pages are silent (each also listed in the design notes):
* query head j uses key head floor(j*h_k/h_q) and value head floor(j*h_v/h_q)
  (contiguous groups, as in GQA; SAGA only decouples the two counts);
* one threshold per (batch, query head) row;
* the threshold is the N-th largest score counted with multiplicity, and every
  score >= it is kept, so ties at the threshold are all kept; when N >= L
  there is no N-th largest to exclude anything and the threshold is -inf;
* refresh steps are t = 0, R, 2R, ... and use the threshold computed from
  their own scores; later steps compare against that stale threshold,
  including the tokens appended since;
* the new token is appended before attending, so step t attends to
  L = l_kv + t + 1 tokens;
* an empty selection gives O = 0.
"""
from __future__ import annotations

import numpy as np

NEG_INF = np.float32(-np.inf)


def key_head(j, h_q, h_k):
    """Key head read by query head j (contiguous GQA-style groups)."""
    return (np.asarray(j) * h_k) // h_q


def value_head(j, h_q, h_v):
    """Value head read by query head j; independent of the key head count (SAGA)."""
    return (np.asarray(j) * h_v) // h_q


def kv_append(k_cache, v_cache, k_new, v_new, pos):
    """Store the new token's key and value rows at position pos of every head."""
    k_cache[:, :, pos, :] = k_new
    v_cache[:, :, pos, :] = v_new


def scores(q, k_cache, L):
    """Eq. 2: A[b, j, i] = q[b, j] . K[b, key_head(j), i] / sqrt(d), for i < L.

    q: [B, h_q, d], k_cache: [B, h_k, >=L, d] (bf16-exact values in any float
    dtype).  Returns fp32 [B, h_q, L].
    """
    B, h_q, d = q.shape
    h_k = k_cache.shape[1]
    K = np.asarray(k_cache[:, :, :L, :], dtype=np.float64)
    q64 = np.asarray(q, dtype=np.float64)
    out = np.empty((B, h_q, L), dtype=np.float32)
    inv_sqrt_d = 1.0 / np.sqrt(np.float64(d))
    for b in range(B):
        for j in range(h_q):
            dots = K[b, key_head(j, h_q, h_k)] @ q64[b, j]
            out[b, j] = (dots * inv_sqrt_d).astype(np.float32)
    return out


def nth_largest(row, n):
    """The N-th largest value of a row, counted with multiplicity; -inf if N >= len(row)."""
    row = np.asarray(row, dtype=np.float32)
    if n >= row.shape[0]:
        return NEG_INF
    descending = np.sort(row)[::-1]
    return np.float32(descending[n - 1])


def threshold(A, n):
    """Atop-N step 1: per-row threshold [B, h_q] from fp32 scores [B, h_q, L]."""
    B, h_q, _ = A.shape
    tau = np.empty((B, h_q), dtype=np.float32)
    for b in range(B):
        for j in range(h_q):
            tau[b, j] = nth_largest(A[b, j], n)
    return tau


def select(A, tau):
    """Per-element comparison against the row's threshold (fp32): keep A >= tau."""
    return A >= tau[..., None]


def sparse_attention(A, keep, v_cache, L):
    """Eq. 7: O[b, j] = softmax(A[b, j, i]) V[b, value_head(j), i] over the kept i.

    Softmax subtracts the row's kept maximum first (the same function).  Float64.
    Returns [B, h_q, d] float64; rows with nothing kept are zero.
    """
    B, h_q, _ = A.shape
    h_v, d = v_cache.shape[1], v_cache.shape[3]
    out = np.zeros((B, h_q, d), dtype=np.float64)
    for b in range(B):
        for j in range(h_q):
            idx = np.nonzero(keep[b, j])[0]
            if idx.size == 0:
                continue
            a = A[b, j, idx].astype(np.float64)
            e = np.exp(a - a.max())
            p = e / e.sum()
            Vrows = np.asarray(v_cache[b, value_head(j, h_q, h_v), idx, :], dtype=np.float64)
            out[b, j] = p @ Vrows
    return out


def is_refresh_step(t, R):
    """Atop-N step 2: the exact threshold is recomputed once every R steps (t = 0, R, 2R, ...)."""
    return t % R == 0


class OracleLayer:
    """One attention layer's decode state: its caches, its thresholds, its length.

    k0: [B, h_k, l_kv, d], v0: [B, h_v, l_kv, d] (float arrays holding bf16
    values).  Capacity grows one row per step.
    """

    def __init__(self, k0, v0, h_q, n_top, refresh, l_cap=None):
        B, h_k, l_kv, d = k0.shape
        h_v = v0.shape[1]
        cap = l_cap if l_cap is not None else l_kv + 64
        self.k = np.zeros((B, h_k, cap, d), dtype=np.float32)
        self.v = np.zeros((B, h_v, cap, d), dtype=np.float32)
        self.k[:, :, :l_kv] = k0
        self.v[:, :, :l_kv] = v0
        self.length = l_kv
        self.h_q, self.n_top, self.refresh = h_q, n_top, refresh
        self.tau = None
        self.t = 0

    def _grow(self):
        if self.length < self.k.shape[2]:
            return
        pad = max(64, self.k.shape[2] // 4)
        self.k = np.concatenate([self.k, np.zeros_like(self.k[:, :, :pad])], axis=2)
        self.v = np.concatenate([self.v, np.zeros_like(self.v[:, :, :pad])], axis=2)

    def step(self, q, k_new, v_new):
        """One decode step: append, score, (refresh), compare, attend."""
        self._grow()
        kv_append(self.k, self.v, k_new, v_new, self.length)
        self.length += 1
        L = self.length
        A = scores(q, self.k, L)
        refreshed = is_refresh_step(self.t, self.refresh)
        if refreshed:
            self.tau = threshold(A, self.n_top)
        keep = select(A, self.tau)
        out = sparse_attention(A, keep, self.v, L)
        self.t += 1
        return {"out": out, "tau": self.tau.copy(), "keep": keep, "scores": A, "L": L, "refreshed": refreshed}


def refresh_threshold(q, k_cache, L, n_top):
    """The exact threshold a refresh step computes from the current scores."""
    return threshold(scores(q, k_cache, L), n_top)


def vector_reads(h_q, h_k, h_v, L, n_top, batch=1):
    """Key and value vectors one decode step reads per layer (the explainer's count).

    Every cached key of every key head is read; each query head reads N value
    vectors, or every value vector once when N covers the context.
    """
    keys = batch * h_k * L
    values = batch * min(h_q * n_top, h_v * L)
    return keys, values
