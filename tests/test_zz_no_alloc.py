"""The allocation-free decode entry point against the workspace entry point.

saga_decode_attn_noalloc exists for callers that cannot allocate device
memory around a decode call: their device memory belongs to another
allocator (a serving engine that reserves HBM up front), or allocating is
not allowed at that point.  It uses a fixed scratch array built into the
library instead of a caller workspace.  This test runs the same two decode
steps (a threshold refresh, then a reuse step) through both entry points on
identical caches and compares the results bit for bit (both entry points run
the same deterministic kernels with the same launch sizes), reads the status
word of the allocation-free calls, and checks that a shape too large for the
built-in scratch is refused before anything is enqueued.
"""
import ctypes

import numpy as np
import pytest
import torch

from long_context_decoding_saga_b200 import saga, workload

pytestmark = pytest.mark.gpu

@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_decoding_saga_b200 import build
    build.build()
    saga.load()


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    wl = workload.Workload("noalloc", 1, 12, 1, 4, 128, 3000, 1, 2, 48, 2, 0.02, "planted_mean", 77)
    inp = workload.make_layer(wl, 0, steps=2)
    l_cap = wl.l_kv + 2
    shape = saga.SagaShape.of(1, 12, 1, 4, 128, l_cap)
    lib = saga.load()
    assert saga.saga_workspace_bytes(shape) <= lib.saga_noalloc_scratch_bytes()
    caches = [workload.alloc_caches(wl, l_cap, inp, "cuda") for _ in range(2)]
    ws = saga.alloc_workspace(shape)
    tau = [torch.zeros((1, 12), device="cuda") for _ in range(2)]
    out = [torch.zeros((1, 12, 128), device="cuda") for _ in range(2)]
    cnt = [torch.zeros((1, 12), dtype=torch.int32, device="cuda") for _ in range(2)]
    idx = [torch.zeros((1, 12, l_cap), dtype=torch.int32, device="cuda") for _ in range(2)]
    for t in range(2):
        q = inp["q"][t].cuda()
        kn, vn = inp["k_new"][t].cuda(), inp["v_new"][t].cuda()
        L = wl.l_kv + t + 1
        for c in caches:
            saga.saga_kv_append(shape, c["k_cache"], c["v_cache"], kn, vn, L - 1)
        saga.saga_decode_attn(shape, q, caches[0]["k_cache"], caches[0]["v_cache"], L, wl.n_top, wl.refresh, t,
                              tau[0], out[0], ws, sel_count=cnt[0], sel_idx=idx[0])
        saga.saga_decode_attn_noalloc(shape, q, caches[1]["k_cache"], caches[1]["v_cache"], L, wl.n_top, wl.refresh,
                                      t, tau[1], out[1], sel_count=cnt[1], sel_idx=idx[1])
        torch.cuda.synchronize()
        assert torch.equal(out[0], out[1]), f"call {t}: outputs differ by {(out[0] - out[1]).abs().max().item()}"
        assert torch.equal(tau[0], tau[1])
        assert torch.equal(cnt[0], cnt[1])
        n = cnt[0].cpu().numpy()
        a, b = idx[0].cpu().numpy(), idx[1].cpu().numpy()
        for j in range(12):
            assert np.array_equal(a[0, j, :n[0, j]], b[0, j, :n[0, j]])
        assert (n > 0).all()
        assert saga.saga_noalloc_get_status() == 0, f"call {t}: status word set"


def test_noalloc_refuses_shapes_beyond_its_scratch():
    lib = saga.load()
    big = saga.SagaShape.of(4, 32, 8, 8, 64, 131072)
    assert saga.saga_workspace_bytes(big) > lib.saga_noalloc_scratch_bytes()
    fake = ctypes.c_void_p(0x100000)  # never dereferenced: the size check refuses first
    rc = lib.saga_decode_attn_noalloc(ctypes.byref(big), fake, fake, fake, 100, None, 8, 4, 0, fake, fake, 0, None,
                                      None, None)
    assert rc == saga.SAGA_ERR_WORKSPACE
    assert b"scratch" in lib.saga_noalloc_last_error()
