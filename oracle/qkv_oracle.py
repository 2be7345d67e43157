"""CPU oracle for the decode step's query/key/value projection with SAGA head counts.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import this module; the CUDA path never
calls it and shares no code with it.

It restates eq. 1 of the summary page ("More Value per Key: Asymmetric
Sparse Attention for Faster LLM Decoding", Attention Mechanism
Formalization): Q = X W_Q, K = X W_K, V = X W_V, for the one new token of a
decode step, with h_q query heads, h_k key heads and h_v value heads of
dimension d (SAGA decouples h_k from h_v: a smaller key projection, Methodology
> SAGA Architecture).  The new key and value rows go to the KV cache at
position pos (the KV cache of the explainer's jargon list).

Packing (this build's reading: the pages give no layout): the three
projections are stacked row-wise as one bf16 matrix w_qkv [(h_q + h_k + h_v)
* d, D] whose row n holds the weights of output column n: rows [0, h_q d)
are W_Q's columns (query head n // d, dimension n % d), then h_k d rows of
W_K, then h_v d rows of W_V.  Products are formed in float64 and the results
rounded once to bf16 (round to nearest even).
"""
from __future__ import annotations

import numpy as np
import torch


def to_bf16(a):
    """float64 -> bf16 (round to nearest even), returned as float64 values."""
    return torch.as_tensor(np.asarray(a, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def project(x, w_qkv, h_q, h_k, h_v, d):
    """Eq. 1 for one decode token per batch row.  x: [B, D]; w_qkv: [(h_q + h_k + h_v) d, D].
    Returns float64 (q [B, h_q, d], k_new [B, h_k, d], v_new [B, h_v, d]) before rounding."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_qkv, dtype=np.float64)
    y = x @ w.T  # [B, (h_q + h_k + h_v) d]
    B = x.shape[0]
    q = y[:, :h_q * d].reshape(B, h_q, d)
    k = y[:, h_q * d:(h_q + h_k) * d].reshape(B, h_k, d)
    v = y[:, (h_q + h_k) * d:].reshape(B, h_v, d)
    return q, k, v


def project_and_append(x, w_qkv, k_cache, v_cache, pos, h_q, h_k, h_v, d):
    """The bf16 query and the caches with the new key/value rows written at pos (copies; inputs untouched)."""
    q, k, v = project(x, w_qkv, h_q, h_k, h_v, d)
    kc, vc = np.array(k_cache, dtype=np.float64), np.array(v_cache, dtype=np.float64)
    kc[:, :, pos, :] = to_bf16(k)
    vc[:, :, pos, :] = to_bf16(v)
    return to_bf16(q), kc, vc
