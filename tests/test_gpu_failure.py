"""Failure detection on the GPU without a fault (needs a B200).

Every wait inside the kernels is bounded; when one gives up, the kernel
unwinds (in-flight copies drained, TMEM freed), sets SAGA_STATUS_TIMEOUT in
the status word and returns, so the context stays usable.  The test hook
saga_test_expire_next_wait makes the next reuse step's keep kernel wait on a
barrier that nothing arrives at, with a 2 ms limit: the wait runs out for
certain, nothing hangs or faults.  The test then checks that the flag is
set, that the same step redone on a fresh workspace matches the oracle, and
that argument errors of the allocation-free entry point enqueue nothing
that could set its status.
"""
import numpy as np
import pytest
import torch

from long_context_decoding_saga_b200 import saga, workload
from oracle import saga_oracle
from tests import gpu_harness

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_decoding_saga_b200 import build
    build.build()
    saga.load()


def test_expired_wait_flags_timeout_and_the_context_stays_usable():
    wl = workload.Workload("expire", 1, 12, 1, 4, 128, 3000, 1, 2, 50, 4, 0.02, "planted_mean", 5)
    inp = workload.make_layer(wl, 0, device="cuda", steps=2)
    l_cap = wl.l_kv + 2
    shape = saga.SagaShape.of(1, 12, 1, 4, 128, l_cap)
    caches = workload.alloc_caches(wl, l_cap, inp, "cuda")
    kc, vc = caches["k_cache"], caches["v_cache"]
    tau = torch.zeros((1, 12), device="cuda")
    out = torch.zeros((1, 12, 128), device="cuda")
    cnt = torch.zeros((1, 12), dtype=torch.int32, device="cuda")
    idx = torch.zeros((1, 12, l_cap), dtype=torch.int32, device="cuda")
    orc = saga_oracle.OracleLayer(inp["K0"].float().cpu().numpy(), inp["V0"].float().cpu().numpy(), 12, wl.n_top,
                                  wl.refresh, l_cap=l_cap)
    ws = saga.alloc_workspace(shape)

    def step(t, workspace):
        saga.saga_decode_step(shape, inp["q"][t], inp["k_new"][t], inp["v_new"][t], kc, vc, wl.l_kv + t + 1,
                              wl.n_top, wl.refresh, t, tau, out, workspace, sel_count=cnt, sel_idx=idx)

    step(0, ws)  # refresh step, normal
    torch.cuda.synchronize()
    assert saga.saga_get_status(ws) == 0
    res0 = orc.step(inp["q"][0].float().cpu().numpy(), inp["k_new"][0].float().cpu().numpy(),
                    inp["v_new"][0].float().cpu().numpy())
    gpu_harness.compare_step(res0, out[0].cpu().numpy(), tau[0].cpu().numpy(), cnt.cpu().numpy(),
                             idx.cpu().numpy(), 0)

    saga.saga_test_expire_next_wait(2_000_000)  # 2 ms
    step(1, ws)  # reuse step: its keep kernel's wait runs out
    torch.cuda.synchronize()  # returns: the kernel unwound instead of hanging
    assert saga.saga_get_status(ws) & saga.SAGA_STATUS_TIMEOUT

    # the same step on a fresh workspace (the fused append rewrites the same row) matches the oracle
    ws2 = saga.alloc_workspace(shape)
    step(1, ws2)
    torch.cuda.synchronize()
    assert saga.saga_get_status(ws2) == 0
    res1 = orc.step(inp["q"][1].float().cpu().numpy(), inp["k_new"][1].float().cpu().numpy(),
                    inp["v_new"][1].float().cpu().numpy())
    rep = gpu_harness.compare_step(res1, out[0].cpu().numpy(), tau[0].cpu().numpy(), cnt.cpu().numpy(),
                                   idx.cpu().numpy(), 1)
    assert not rep.refreshed and rep.kept_max > 0


def test_noalloc_argument_errors_enqueue_nothing():
    """A bad argument is refused before the allocation-free entry point clears or uses its scratch."""
    shape = saga.SagaShape.of(1, 8, 1, 8, 64, 256)
    z = lambda *s, dt=torch.bfloat16: torch.zeros(s, dtype=dt, device="cuda")  # noqa: E731
    q, kc, vc = z(1, 8, 64), z(1, 1, 256, 64), z(1, 8, 256, 64)
    tau, out = z(1, 8, dt=torch.float32), z(1, 8, 64, dt=torch.float32)
    # a length beyond the capacity, read on the device, sets the clamp flag of this call
    lens = torch.tensor([100000], dtype=torch.int32, device="cuda")
    saga.saga_decode_attn_noalloc(shape, q, kc, vc, 10, 4, 2, 0, tau, out, seq_len_dev=lens)
    assert saga.saga_noalloc_get_status() & saga.SAGA_STATUS_LEN_CLAMPED
    for bad in (dict(n_top=0), dict(seq_len=0), dict(refresh_interval=0)):
        kw = dict(seq_len=10, n_top=4, refresh_interval=2)
        kw.update(bad)
        with pytest.raises(saga.SagaError) as e:
            saga.saga_decode_attn_noalloc(shape, q, kc, vc, kw["seq_len"], kw["n_top"], kw["refresh_interval"], 0,
                                          tau, out)
        assert e.value.code == saga.SAGA_ERR_ARG
        # nothing was enqueued: the previous call's flag is still there (no clear ran)
        assert saga.saga_noalloc_get_status() & saga.SAGA_STATUS_LEN_CLAMPED
    saga.saga_decode_attn_noalloc(shape, q, kc, vc, 10, 4, 2, 0, tau, out)
    assert saga.saga_noalloc_get_status() == 0
    assert np.all(out.cpu().numpy() == 0)  # zero caches and queries: every score 0, uniform weights over zero rows
