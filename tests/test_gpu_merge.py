"""The closed-form GQA-to-SAGA key-head merge on the GPU against the fp64 oracle (needs a B200).

Inputs are bf16 X and Q (the oracle reads the same rounded values) and fp32 W_K.  Each teacher head has a
planted partner (W_K of the partner = W_K of the head + a small perturbation), with partners chosen so the
optimal pairing is not the adjacent one and is well separated from the others; sizes are not multiples of
the GEMM tiles.  Tolerances come from the GPU's fp32 Gram sums (relative error about sqrt(K) * 2^-24,
K up to a few thousand) amplified by the condition number of S_a + S_b (about 2 for these queries):
1e-4 of the largest entry on the merged projections.  A pair loss is quadratic in M(a, b) - W_K^r, so its
error follows the error of M, which scales with |W|, not with the loss: each loss is held to 1e-3 of
itself plus 1e-4 of the largest pair loss.
"""
import numpy as np
import pytest
import torch

from long_context_decoding_saga_b200 import saga
from oracle import merge_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_decoding_saga_b200 import build
    build.build()
    saga.load()


def _case(T, D, d, h_q, h_k, partners, seed, eps=0.05):
    g = torch.Generator().manual_seed(seed)
    X = torch.randn((T, D), generator=g).to(torch.bfloat16)
    Q = torch.randn((T, h_q, d), generator=g).to(torch.bfloat16)
    W = torch.randn((h_k, D, d), generator=g) * D ** -0.5
    for a, b in partners:
        W[b] = W[a] + eps * torch.randn((D, d), generator=g) * D ** -0.5
    return X, Q, W


CASES = [
    dict(T=300, D=200, d=64, h_q=8, h_k=4, partners=[(0, 2), (1, 3)], seed=1),
    dict(T=1000, D=333, d=128, h_q=16, h_k=8, partners=[(0, 5), (1, 7), (2, 4), (3, 6)], seed=2),
    dict(T=777, D=256, d=64, h_q=32, h_k=8, partners=[(0, 3), (1, 2), (4, 7), (5, 6)], seed=3),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"T{c['T']}_D{c['D']}_d{c['d']}_hk{c['h_k']}")
def test_merge_matches_oracle(case):
    X, Q, W = _case(**case)
    h_k, h_q = case["h_k"], case["h_q"]
    loss, pairing, merged, ws = saga.key_head_merge(X.cuda(), Q.cuda(), W.cuda(), h_k)
    torch.cuda.synchronize()
    assert saga.saga_get_status(ws) == 0
    ref = merge_oracle.key_head_merge(X.float().numpy(), Q.float().numpy(), W.numpy(), h_q)
    loss, pairing, merged = loss.cpu().numpy().astype(np.float64), pairing.cpu().numpy(), merged.cpu().numpy()
    assert np.array_equal(pairing, ref["pairing"])
    assert sorted((min(a, b), max(a, b)) for a, b in case["partners"]) == ref["pairs"]
    assert np.all(np.diag(loss) == 0) and np.array_equal(loss, loss.T)
    tol = 1e-4 * np.max(ref["weights"]) + 1e-3 * ref["weights"]
    assert np.all(np.abs(loss - ref["weights"]) <= tol)
    for m, mr in zip(merged, ref["merged"]):
        assert np.max(np.abs(m - mr)) <= 1e-4 * np.max(np.abs(mr))
    # every pair's loss: the planted partners are the cheapest merges by a wide margin
    for a, b in ref["pairs"]:
        others = [loss[a, c] for c in range(h_k) if c not in (a, b)]
        assert loss[a, b] < 0.2 * min(others)


def test_merge_of_identical_heads_is_that_head():
    """W_K^a = W_K^b: M(a, b) = W_K^a and L_ab = 0 (Lemma 4.1), up to the fp32 rounding of the Grams."""
    X, Q, W = _case(T=256, D=128, d=64, h_q=4, h_k=2, partners=[], seed=4)
    W[1] = W[0]
    loss, pairing, merged, _ = saga.key_head_merge(X.cuda(), Q.cuda(), W.cuda(), 2)
    torch.cuda.synchronize()
    assert pairing.cpu().tolist() == [1, 0]
    np.testing.assert_allclose(merged[0].cpu().numpy(), W[0].numpy(), rtol=0, atol=1e-5 * float(W[0].abs().max()))
    scale = float((X.float() @ W[0]).square().sum() * Q.float().square().sum() / X.shape[0])
    assert abs(float(loss[0, 1])) <= 1e-9 * scale
