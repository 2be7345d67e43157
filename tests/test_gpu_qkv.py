"""The decode-step QKV projection (eq. 1 with SAGA head counts) on the GPU against the fp64 oracle.

Inputs: x ~ N(0, 1) and weights ~ N(0, 1/D), both rounded to bf16 on the CPU (the oracle reads the same
bf16 values, so every product x_k w_kn is exact in fp32 and only the summation order differs).  Batch 1
runs on CUDA cores: every lane a sequential run of D / 32 products, then a 5-level shuffle tree, at most
D / 32 + 5 roundings of half an ulp.  Batch 2 .. 16 runs on the tensor cores: one accumulation per
16-element MMA step (the tensor core may truncate rather than round: a full ulp each), then at most 8
split partials added in order.  Both stay within e = (D / 8 + 64) 2^-24 sum_k |x_k w_kn| of
the exact value; the one rounding to bf16 adds at most 2^-8 of the value
(half a bf16 ulp).  The test bound is |out - exact| <= 2^-8 (|exact| + e) + e, element by element.  Rows of
the caches other than pos must be bit-identical to what was there, and a second call on the same
workspace must reproduce the first bit for bit (the split partials are added in a fixed order).
Cases that need a split of the hidden dimension run the cluster reduction; the 8-wide hidden runs one split.
"""
import numpy as np
import pytest
import torch

from long_context_decoding_saga_b200 import saga
from oracle import qkv_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_decoding_saga_b200 import build
    build.build()
    saga.load()


def _inputs(B, D, h_q, h_k, h_v, d, l_cap, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((B, D), generator=g).to(torch.bfloat16)
    w = (torch.randn(((h_q + h_k + h_v) * d, D), generator=g) * D ** -0.5).to(torch.bfloat16)
    kc = torch.randn((B, h_k, l_cap, d), generator=g).to(torch.bfloat16)
    vc = torch.randn((B, h_v, l_cap, d), generator=g).to(torch.bfloat16)
    return x, w, kc, vc


def _bound(x, w, exact, B, D):
    e = (D / 8 + 64) * 2.0 ** -24 * (np.abs(x) @ np.abs(w).T)  # [B, n_cols]
    return 2.0 ** -8 * (np.abs(exact) + e) + e


def _run(B, D, h_q, h_k, h_v, d, l_cap, pos, seed, dev_len=None):
    x, w, kc0, vc0 = _inputs(B, D, h_q, h_k, h_v, d, l_cap, seed)
    shape = saga.SagaShape(B, h_q, h_k, h_v, d, l_cap)
    xg, wg, kcg, vcg = x.cuda(), w.cuda(), kc0.cuda(), vc0.cuda()
    q = torch.full((B, h_q, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    sl = None if dev_len is None else torch.tensor([dev_len], dtype=torch.int32, device="cuda")
    ws = saga.saga_qkv_project(shape, xg, wg, q, kcg, vcg, pos, seq_len_dev=sl)
    torch.cuda.synchronize()
    first = (q.clone(), kcg.clone(), vcg.clone())
    saga.saga_qkv_project(shape, xg, wg, q, kcg, vcg, pos, workspace=ws, seq_len_dev=sl)
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(first, (q, kcg, vcg))), "second call differs"
    assert saga.saga_get_status(ws) == 0
    return x, w, kc0, vc0, q.cpu(), kcg.cpu(), vcg.cpu()


def _check(B, D, h_q, h_k, h_v, d, l_cap, pos, seed, dev_len=None, expect_pos=None):
    x, w, kc0, vc0, q, kc, vc = _run(B, D, h_q, h_k, h_v, d, l_cap, pos, seed, dev_len)
    p = pos if expect_pos is None else expect_pos
    xf, wf = x.double().numpy(), w.double().numpy()
    qe, ke, ve = qkv_oracle.project(xf, wf, h_q, h_k, h_v, d)
    bound = _bound(xf, wf, np.concatenate([qe.reshape(B, -1), ke.reshape(B, -1), ve.reshape(B, -1)], axis=1), B, D)
    nq, nk = h_q * d, h_k * d
    got = np.concatenate([q.double().numpy().reshape(B, -1), kc[:, :, p].double().numpy().reshape(B, -1),
                          vc[:, :, p].double().numpy().reshape(B, -1)], axis=1)
    exact = np.concatenate([qe.reshape(B, -1), ke.reshape(B, -1), ve.reshape(B, -1)], axis=1)
    err = np.abs(got - exact)
    assert np.all(np.isfinite(got))
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), f"column {worst[1]} (q<{nq}, k<{nq + nk}) row {worst[0]}: err {err[worst]} > {bound[worst]}"
    # the oracle's own rounded answer, for the bulk of the outputs (differences only where the exact value sits
    # within the summation error of a rounding boundary)
    ref_q, ref_k, ref_v = qkv_oracle.project_and_append(xf, wf, kc0.double().numpy(), vc0.double().numpy(), p,
                                                       h_q, h_k, h_v, d)
    same = np.mean(got == np.concatenate([ref_q.reshape(B, -1), ref_k[:, :, p].reshape(B, -1),
                                          ref_v[:, :, p].reshape(B, -1)], axis=1))
    assert same > 0.98, same
    other = [r for r in range(l_cap) if r != p]
    assert torch.equal(kc[:, :, other], kc0[:, :, other]) and torch.equal(vc[:, :, other], vc0[:, :, other])


# (B, D, h_q, h_k, h_v, d, l_cap, pos): the two SAGA models' projection shapes at batch 1 and 16, ragged
# batches, hidden sizes that leave a ragged last chunk or k-block (1000, 2056, 4104) or a single 8-element
# piece, output widths that end in a partial 128-column tile (448, 2816), splits longer than the weight
# ring (4096: 8 k-blocks per split), a projection of 148 tiles whose splits stage 32 k-blocks of x each,
# and the first and last cache rows.
CASES = [
    (1, 2048, 32, 2, 8, 64, 40, 17),      # Llama-3.2-1B SAGA projection
    (16, 2048, 32, 2, 8, 64, 9, 8),
    (1, 1536, 12, 1, 4, 128, 33, 0),      # Qwen2.5-1.5B SAGA projection
    (16, 1536, 12, 1, 4, 128, 5, 4),
    (3, 1000, 8, 8, 8, 64, 7, 3),         # plain MHA head counts, ragged batch and hidden
    (5, 2056, 16, 2, 4, 128, 6, 5),
    (2, 8, 4, 1, 2, 64, 3, 1),
    (1, 8, 4, 1, 2, 64, 3, 2),
    (9, 4096, 8, 1, 8, 128, 4, 2),
    (1, 4104, 8, 1, 8, 128, 4, 1),
    (4, 4096, 128, 4, 16, 128, 2, 1),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}_D{}_hq{}_hk{}_hv{}_d{}".format(*c[:6]))
def test_qkv_matches_oracle(case):
    _check(*case, seed=sum(case))


def test_qkv_position_from_device():
    # seq_len on the device overrides the host pos: the new row goes to seq_len - 1
    _check(2, 512, 8, 2, 4, 64, 12, pos=0, seed=5, dev_len=10, expect_pos=9)
    # out-of-range lengths clamp into the cache, as the attention kernels do
    _check(2, 512, 8, 2, 4, 64, 12, pos=3, seed=6, dev_len=0, expect_pos=0)
    _check(2, 512, 8, 2, 4, 64, 12, pos=3, seed=7, dev_len=99, expect_pos=11)


def test_qkv_workspace_too_small():
    shape = saga.SagaShape(4, 8, 1, 8, 64, 4)
    x = torch.zeros((4, 2048), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((17 * 64, 2048), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((4, 8, 64), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((4, 1, 4, 64), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros((4, 8, 4, 64), dtype=torch.bfloat16, device="cuda")
    need = saga.saga_qkv_workspace_bytes(shape, 2048)
    ws = torch.zeros(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(saga.SagaError) as e:
        saga.saga_qkv_project(shape, x, w, q, kc, vc, 0, workspace=ws)
    assert e.value.code == saga.SAGA_ERR_WORKSPACE


def test_qkv_rejects_bad_arguments():
    shape = saga.SagaShape(17, 8, 1, 8, 64, 4)
    x = torch.zeros((17, 64), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((17 * 64, 64), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((17, 8, 64), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((17, 1, 4, 64), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros((17, 8, 4, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(saga.SagaError) as e:
        saga.saga_qkv_project(shape, x, w, q, kc, vc, 0)
    assert e.value.code == saga.SAGA_ERR_UNSUPPORTED
    shape = saga.SagaShape(1, 8, 1, 8, 64, 4)
    with pytest.raises(saga.SagaError) as e:
        saga.saga_qkv_project(shape, x[:1], w, q[:1], kc[:1], vc[:1], 4)
    assert e.value.code == saga.SAGA_ERR_ARG


@pytest.mark.parametrize("B", [1, 4])
def test_qkv_graph_replay_with_device_length(B):
    """Captured once in a CUDA graph with the position read from a device length; replayed at two
    lengths, each replay writes its own cache row and leaves the other rows alone."""
    h_q, h_k, h_v, d, D, l_cap = 12, 1, 4, 128, 1536, 16
    x, w, kc0, vc0 = _inputs(B, D, h_q, h_k, h_v, d, l_cap, seed=123 + B)
    shape = saga.SagaShape(B, h_q, h_k, h_v, d, l_cap)
    xg, wg, kcg, vcg = x.cuda(), w.cuda(), kc0.cuda(), vc0.cuda()
    q = torch.zeros((B, h_q, d), dtype=torch.bfloat16, device="cuda")
    sl = torch.tensor([5], dtype=torch.int32, device="cuda")
    ws = saga.alloc_qkv_workspace(shape, D)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        saga.saga_qkv_project(shape, xg, wg, q, kcg, vcg, 4, workspace=ws, seq_len_dev=sl, stream=stream)
    stream.synchronize()
    kcg.copy_(kc0.cuda())
    vcg.copy_(vc0.cuda())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        saga.saga_qkv_project(shape, xg, wg, q, kcg, vcg, 4, workspace=ws, seq_len_dev=sl, stream=stream)
    xf, wf = x.double().numpy(), w.double().numpy()
    qe, ke, ve = qkv_oracle.project(xf, wf, h_q, h_k, h_v, d)
    bound_k = _bound(xf, wf[h_q * d:(h_q + h_k) * d], ke.reshape(B, -1), B, D)
    for length in (9, 14):
        sl.fill_(length)
        graph.replay()
        torch.cuda.synchronize()
        row = kcg[:, :, length - 1].cpu().double().numpy().reshape(B, -1)
        assert np.all(np.abs(row - ke.reshape(B, -1)) <= bound_k), length
    untouched = [r for r in range(l_cap) if r not in (8, 13)]
    assert torch.equal(kcg.cpu()[:, :, untouched], kc0[:, :, untouched])
    assert torch.equal(vcg.cpu()[:, :, untouched], vc0[:, :, untouched])
    assert saga.saga_get_status(ws) == 0
    del graph
