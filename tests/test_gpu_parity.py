"""Parity of the CUDA decode path with the CPU oracle (needs a B200)."""
import numpy as np
import pytest
import torch

from long_context_decoding_saga_b200 import saga, workload
from oracle import saga_oracle
from tests import gpu_harness

pytestmark = pytest.mark.gpu

W = workload.Workload


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_decoding_saga_b200 import build
    build.build()
    saga.load()


def small(name, **kw):
    base = dict(name=name, batch=1, h_q=8, h_k=1, h_v=8, d=64, l_kv=1000, layers=1, steps=12, n_top=40, refresh=4,
                planted=0.02, q_mode="planted_mean", seed=7)
    base.update(kw)
    return W(**base)


# Shapes spanning groups of 1 to 64 query heads per key head (groups of up to 4 also take the score dump's
# top-byte counts on refresh steps), d = 64 and 128, value heads above / equal to / below the key heads,
# batch > 1, ragged lengths (not multiples of 32 or 128).
CASES = [
    small("g8_d64", h_q=8, h_k=1, h_v=8, d=64, l_kv=1000),
    small("g12_d128_hv4", h_q=12, h_k=1, h_v=4, d=128, l_kv=2085, n_top=50),
    small("g16_d64_b2", batch=2, h_q=32, h_k=2, h_v=8, d=64, l_kv=1531, n_top=64),
    small("g32_d64", h_q=32, h_k=1, h_v=8, d=64, l_kv=777, n_top=33),
    small("g64_d64", h_q=64, h_k=1, h_v=16, d=64, l_kv=650, n_top=20),
    small("g4_d64_gqa", h_q=32, h_k=8, h_v=8, d=64, l_kv=1100, n_top=30),
    small("g2_d128_hv_lt_hk", h_q=8, h_k=4, h_v=2, d=128, l_kv=903, n_top=25),
    small("g1_mha_d128", h_q=4, h_k=4, h_v=4, d=128, l_kv=300, n_top=9, batch=3),
    small("g16_d128_r1", h_q=16, h_k=1, h_v=2, d=128, l_kv=1290, n_top=100, refresh=1, steps=5),
    small("g8_n1", h_q=8, h_k=1, h_v=8, d=64, l_kv=500, n_top=1, refresh=3),
    small("tiny_l", h_q=8, h_k=2, h_v=4, d=64, l_kv=5, n_top=3, refresh=2, steps=6, q_mode="gaussian", planted=0.0),
    small("n_gt_l", h_q=8, h_k=1, h_v=8, d=64, l_kv=40, n_top=60, refresh=2, steps=30),
    small("dense_g4", h_q=16, h_k=4, h_v=4, d=64, l_kv=1500, n_top=workload.DENSE, refresh=1 << 30,
          q_mode="gaussian", planted=0.0, steps=4),
    small("dense_g12_d128", h_q=12, h_k=1, h_v=4, d=128, l_kv=700, n_top=workload.DENSE, refresh=1 << 30,
          q_mode="gaussian", planted=0.0, steps=3),
    # dense kernel (value tiles by TMA): d = 128 with value heads shared by key heads, batch 2, ragged length
    small("dense_hv_lt_hk_d128", batch=2, h_q=8, h_k=4, h_v=2, d=128, l_kv=1333, n_top=workload.DENSE,
          refresh=1 << 30, q_mode="gaussian", planted=0.0, steps=3),
    small("dense_g16_d64", h_q=32, h_k=2, h_v=2, d=64, l_kv=2500, n_top=workload.DENSE, refresh=1 << 30,
          q_mode="gaussian", planted=0.0, steps=3),
]


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_decode_matches_oracle(wl):
    reports, _ = gpu_harness.run_parity(wl, wl.steps)
    assert len(reports) == wl.steps
    assert reports[0].refreshed


def test_tiny_config_full():
    """The tiny configuration, all 32 steps: 1 layer, l_kv=1024, h_q=8, h_k=1, h_v=8, N=64, R=8."""
    reports, _ = gpu_harness.run_parity(workload.TINY, workload.TINY.steps)
    assert sum(r.refreshed for r in reports) == 4


def test_graph_replay_matches_oracle():
    wl = small("graphs", h_q=12, h_k=1, h_v=4, d=128, l_kv=3001, n_top=70, refresh=3, steps=8)
    reports, _ = gpu_harness.run_parity(wl, wl.steps, graphs=True)
    assert len(reports) == wl.steps


def test_bf16_output_is_rounded_fp32_output():
    wl = small("bf16", h_q=12, h_k=1, h_v=4, d=128, l_kv=1200, n_top=40, steps=3)
    _, s32 = gpu_harness.run_parity(wl, wl.steps)
    _, s16 = gpu_harness.run_parity(wl, wl.steps, out_dtype=torch.bfloat16)
    assert torch.equal(s32.out.to(torch.bfloat16), s16.out)


def test_runs_are_bitwise_deterministic():
    wl = small("det", h_q=32, h_k=2, h_v=8, d=64, l_kv=4000, n_top=64, steps=5)
    _, a = gpu_harness.run_parity(wl, wl.steps)
    _, b = gpu_harness.run_parity(wl, wl.steps)
    assert torch.equal(a.out, b.out) and torch.equal(a.tau, b.tau) and torch.equal(a.sel_idx, b.sel_idx)


def test_kv_append_bit_exact():
    shape = saga.SagaShape.of(2, 8, 2, 4, 128, 64)
    g = torch.Generator(device="cuda").manual_seed(3)
    kc = torch.randn((2, 2, 64, 128), device="cuda", generator=g).to(torch.bfloat16)
    vc = torch.randn((2, 4, 64, 128), device="cuda", generator=g).to(torch.bfloat16)
    kn = torch.randn((2, 2, 128), device="cuda", generator=g).to(torch.bfloat16)
    vn = torch.randn((2, 4, 128), device="cuda", generator=g).to(torch.bfloat16)
    ref_k, ref_v = kc.clone(), vc.clone()
    ref_k[:, :, 17] = kn
    ref_v[:, :, 17] = vn
    saga.saga_kv_append(shape, kc, vc, kn, vn, 17)
    torch.cuda.synchronize()
    assert torch.equal(kc, ref_k) and torch.equal(vc, ref_v)


def _select_rows():
    rng = np.random.default_rng(5)
    rows = []
    for n in (1, 2, 3, 5, 31, 32, 33, 1000, 4097, 65536 + 7):
        rows.append(rng.standard_normal(n).astype(np.float32))
    rows.append(np.round(rng.standard_normal(3000) * 4).astype(np.float32))   # heavy ties
    rows.append(np.full(777, 1.25, np.float32))                              # all equal
    z = rng.standard_normal(500).astype(np.float32)
    z[::3] = 0.0
    z[1::7] = -0.0
    rows.append(z)                                                           # signed zeros
    rows.append((rng.standard_normal(20000) * 1e-30).astype(np.float32))   # tiny magnitudes
    rows.append(np.concatenate([rng.standard_normal(40000), 1e30 * rng.standard_normal(50)]).astype(np.float32))
    return rows


def test_radix_select_matches_oracle_nth_largest():
    rows = _select_rows()
    ws = torch.zeros(saga.load().atopn_select_workspace_bytes(1), dtype=torch.uint8, device="cuda")
    for row in rows:
        L = row.size
        stride = (L + 3) // 4 * 4
        buf = np.zeros((1, stride), np.float32)
        buf[0, :L] = row
        dev = torch.from_numpy(buf).cuda()
        for n in sorted({1, 2, max(1, L // 3), max(1, L - 1), L, L + 5}):
            tau = torch.zeros(1, device="cuda")
            saga.atopn_select_threshold(dev, L, n, tau, ws)
            torch.cuda.synchronize()
            expect = saga_oracle.nth_largest(row, n)
            got = float(tau.item())
            assert (got == expect) or (np.isneginf(got) and np.isneginf(expect)), (L, n, got, expect)


def test_refresh_threshold_entry_point():
    wl = small("refresh_ep", h_q=12, h_k=1, h_v=4, d=128, l_kv=5000, n_top=77)
    inp = workload.make_layer(wl, 0, steps=1)
    shape = saga.SagaShape.of(1, 12, 1, 4, 128, 5000)
    kc = inp["K0"].cuda().contiguous()
    q = inp["q"][0].cuda().contiguous()
    tau = torch.zeros((1, 12), device="cuda")
    ws = saga.alloc_workspace(shape)
    saga.atopn_refresh_threshold(shape, q, kc, 5000, 77, tau, ws)
    torch.cuda.synchronize()
    expect = saga_oracle.refresh_threshold(inp["q"][0].float().numpy(), inp["K0"].float().numpy(), 5000, 77)
    assert np.max(np.abs(tau.cpu().numpy() - expect)) <= gpu_harness.BAND


def _stale_tau(kind, h_q):
    mixed = ([1e30, 0.0, -1e30, 5.0, float("nan"), 1e-30] * 4)[:h_q]
    return {"zero": torch.zeros((1, h_q), device="cuda"), "huge": torch.full((1, h_q), 1e30, device="cuda"),
            "tiny": torch.full((1, h_q), -1e30, device="cuda"),
            "nan": torch.full((1, h_q), float("nan"), device="cuda"),
            "mixed": torch.tensor([mixed], device="cuda")}[kind]


# (h_q, h_k, h_v): 12 heads per key head (the select counts every digit itself) and 4 (the score dump also
# counts the top byte of the scores near the stale threshold, which the select uses when it holds N scores)
STALE_HEADS = [(12, 1, 4), (8, 2, 4)]


@pytest.mark.parametrize("heads", STALE_HEADS, ids=lambda h: f"g{h[0] // h[1]}")
@pytest.mark.parametrize("stale", ["huge", "tiny", "nan", "mixed"])
def test_refresh_with_any_stale_threshold_is_exact(stale, heads):
    """Whatever the stale values in tau (above every score, below every score, NaN, or mixed per row), the
    refreshed threshold is the same bits as with a stale threshold of 0, and the oracle's: counts of the top
    byte taken from just below the stale threshold up are used only when they hold N scores."""
    h_q, h_k, h_v = heads
    wl = small("refresh_stale", h_q=h_q, h_k=h_k, h_v=h_v, d=128, l_kv=5000, n_top=77)
    inp = workload.make_layer(wl, 0, steps=1)
    shape = saga.SagaShape.of(1, h_q, h_k, h_v, 128, 5000)
    kc = inp["K0"].cuda().contiguous()
    q = inp["q"][0].cuda().contiguous()
    ws = saga.alloc_workspace(shape)
    base = torch.zeros((1, h_q), device="cuda")
    saga.atopn_refresh_threshold(shape, q, kc, 5000, 77, base, ws)
    tau = _stale_tau(stale, h_q)
    saga.atopn_refresh_threshold(shape, q, kc, 5000, 77, tau, ws)
    torch.cuda.synchronize()
    assert torch.equal(tau, base)
    expect = saga_oracle.refresh_threshold(inp["q"][0].float().numpy(), inp["K0"].float().numpy(), 5000, 77)
    assert np.max(np.abs(tau.cpu().numpy() - expect)) <= gpu_harness.BAND


@pytest.mark.parametrize("heads", STALE_HEADS, ids=lambda h: f"g{h[0] // h[1]}")
@pytest.mark.parametrize("stale", ["zero", "huge", "mixed"])
def test_refresh_of_long_rows_is_exact(stale, heads):
    """Rows longer than 32K scores, fewer rows than SMs: one thread-block cluster per row finds the N-th
    largest; any stale threshold gives the same bits and the oracle's threshold."""
    h_q, h_k, h_v = heads
    wl = small("refresh_long", h_q=h_q, h_k=h_k, h_v=h_v, d=128, l_kv=40000, n_top=300)
    inp = workload.make_layer(wl, 0, steps=1)
    shape = saga.SagaShape.of(1, h_q, h_k, h_v, 128, 40000)
    kc = inp["K0"].cuda().contiguous()
    q = inp["q"][0].cuda().contiguous()
    ws = saga.alloc_workspace(shape)
    base = torch.zeros((1, h_q), device="cuda")
    saga.atopn_refresh_threshold(shape, q, kc, 40000, 300, base, ws)
    tau = _stale_tau(stale, h_q)
    saga.atopn_refresh_threshold(shape, q, kc, 40000, 300, tau, ws)
    torch.cuda.synchronize()
    assert torch.equal(tau, base)
    expect = saga_oracle.refresh_threshold(inp["q"][0].float().numpy(), inp["K0"].float().numpy(), 40000, 300)
    assert np.max(np.abs(tau.cpu().numpy() - expect)) <= gpu_harness.BAND


def test_refresh_with_overflowing_kept_keys_is_exact():
    """A stale threshold below every score makes each CTA of the cluster select keep every key of its chunk
    during the top-digit pass: with 140000 scores a row (17500 a CTA) they overflow the candidate store, and
    the select collects the N-th largest's bin again; the threshold is the oracle's."""
    L, N = 140000, 300
    wl = small("refresh_overflow", h_q=12, h_k=1, h_v=4, d=128, l_kv=L, n_top=N)
    inp = workload.make_layer(wl, 0, steps=1)
    shape = saga.SagaShape.of(1, 12, 1, 4, 128, L)
    kc = inp["K0"].cuda().contiguous()
    q = inp["q"][0].cuda().contiguous()
    ws = saga.alloc_workspace(shape)
    tau = torch.full((1, 12), -1e30, device="cuda")
    saga.atopn_refresh_threshold(shape, q, kc, L, N, tau, ws)
    torch.cuda.synchronize()
    expect = saga_oracle.refresh_threshold(inp["q"][0].float().numpy(), inp["K0"].float().numpy(), L, N)
    assert np.max(np.abs(tau.cpu().numpy() - expect)) <= gpu_harness.BAND
    assert saga.saga_get_status(ws) == 0


def test_empty_selection_gives_zero():
    """A stale threshold above every score of a later step keeps nothing: output 0, count 0."""
    shape = saga.SagaShape.of(1, 8, 1, 8, 64, 600)
    g = torch.Generator(device="cuda").manual_seed(11)
    sess_inp = {
        "K0": torch.randn((1, 1, 598, 64), device="cuda", generator=g).to(torch.bfloat16),
        "V0": torch.randn((1, 8, 598, 64), device="cuda", generator=g).to(torch.bfloat16),
    }
    from long_context_decoding_saga_b200.session import DecodeSession
    s = DecodeSession(shape, 1, 1, 2, track_selection=True)
    s.prefill(0, sess_inp["K0"], sess_inp["V0"])
    q = torch.randn((1, 1, 8, 64), device="cuda", generator=g).to(torch.bfloat16)
    kn = torch.zeros((1, 1, 1, 64), device="cuda", dtype=torch.bfloat16)
    vn = torch.randn((1, 1, 8, 64), device="cuda", generator=g).to(torch.bfloat16)
    s.step(q, kn, vn)
    torch.cuda.synchronize()
    assert (s.tau > 0).all() and (s.sel_count == 1).all()
    s.step(torch.zeros_like(q), kn, vn)
    torch.cuda.synchronize()
    assert (s.sel_count == 0).all()
    assert (s.out == 0).all()


def test_workspace_too_small_is_rejected():
    shape = saga.SagaShape.of(1, 8, 1, 8, 64, 256)
    ws = torch.zeros(saga.saga_workspace_bytes(shape) - 256, dtype=torch.uint8, device="cuda")
    z = lambda *s, dt=torch.bfloat16: torch.zeros(s, dtype=dt, device="cuda")  # noqa: E731
    with pytest.raises(saga.SagaError) as e:
        saga.saga_decode_attn(shape, z(1, 8, 64), z(1, 1, 256, 64), z(1, 8, 256, 64), 10, 4, 2, 0,
                              z(1, 8, dt=torch.float32), z(1, 8, 64, dt=torch.float32), ws)
    assert e.value.code == saga.SAGA_ERR_WORKSPACE


def test_device_length_out_of_range_is_clamped_and_flagged():
    shape = saga.SagaShape.of(1, 8, 1, 8, 64, 256)
    ws = saga.alloc_workspace(shape)
    z = lambda *s, dt=torch.bfloat16: torch.zeros(s, dtype=dt, device="cuda")  # noqa: E731
    lens = torch.tensor([100000], dtype=torch.int32, device="cuda")
    saga.saga_decode_attn(shape, z(1, 8, 64), z(1, 1, 256, 64), z(1, 8, 256, 64), 10, 4, 2, 0,
                          z(1, 8, dt=torch.float32), z(1, 8, 64, dt=torch.float32), ws, seq_len_dev=lens)
    st = saga.saga_get_status(ws)
    assert st & saga.SAGA_STATUS_LEN_CLAMPED
    assert not st & saga.SAGA_STATUS_TIMEOUT


@pytest.mark.parametrize("wl", [
    small("fused_g12_d128", h_q=12, h_k=1, h_v=4, d=128, l_kv=2085, n_top=50, refresh=3, steps=5),
    small("fused_hv_lt_hk", h_q=8, h_k=4, h_v=2, d=128, l_kv=903, n_top=25, refresh=2, steps=4, batch=2),
    small("fused_dense", h_q=16, h_k=4, h_v=4, d=64, l_kv=700, n_top=workload.DENSE, refresh=1 << 30,
          q_mode="gaussian", planted=0.0, steps=3),
], ids=lambda w: w.name)
def test_fused_append_equals_separate_append(wl):
    """saga_decode_step (append inside the attention kernels) gives the same caches, thresholds, outputs
    and index lists, bit for bit, as saga_kv_append followed by saga_decode_attn."""
    inp = workload.make_layer(wl, 0, device="cuda", steps=wl.steps)
    l_cap = wl.l_kv + wl.steps
    n_top = wl.n_for_kernel(l_cap)
    shape = saga.SagaShape.of(wl.batch, wl.h_q, wl.h_k, wl.h_v, wl.d, l_cap)
    B, hq, hk, hv, d = wl.batch, wl.h_q, wl.h_k, wl.h_v, wl.d
    runs = []
    for fused in (False, True):
        kc = torch.zeros((B, hk, l_cap, d), dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros((B, hv, l_cap, d), dtype=torch.bfloat16, device="cuda")
        kc[:, :, :wl.l_kv] = inp["K0"]
        vc[:, :, :wl.l_kv] = inp["V0"]
        tau = torch.zeros((B, hq), dtype=torch.float32, device="cuda")
        ws = saga.alloc_workspace(shape, "cuda")
        outs, idxs = [], []
        for t in range(wl.steps):
            L = wl.l_kv + t + 1
            out = torch.zeros((B, hq, d), dtype=torch.float32, device="cuda")
            cnt = torch.zeros((B, hq), dtype=torch.int32, device="cuda")
            idx = torch.zeros((B, hq, l_cap), dtype=torch.int32, device="cuda")
            if fused:
                saga.saga_decode_step(shape, inp["q"][t], inp["k_new"][t], inp["v_new"][t], kc, vc, L, n_top,
                                      wl.refresh, t, tau, out, ws, sel_count=cnt, sel_idx=idx)
            else:
                saga.saga_kv_append(shape, kc, vc, inp["k_new"][t], inp["v_new"][t], L - 1)
                saga.saga_decode_attn(shape, inp["q"][t], kc, vc, L, n_top, wl.refresh, t, tau, out, ws,
                                      sel_count=cnt, sel_idx=idx)
            outs.append((out, tau.clone(), cnt))
            idxs.append(idx)
        torch.cuda.synchronize()
        runs.append((kc, vc, outs, idxs))
    (k0, v0, o0, i0), (k1, v1, o1, i1) = runs
    assert torch.equal(k0, k1) and torch.equal(v0, v1)
    for t in range(wl.steps):
        for a, b in zip(o0[t], o1[t]):
            assert torch.equal(a, b), f"step {t}"
        c = o0[t][2]
        for bb in range(B):
            for j in range(hq):
                n = int(c[bb, j])
                assert torch.equal(i0[t][bb, j, :n], i1[t][bb, j, :n])


def test_plain_stream_order_matches():
    """With programmatic dependent launch turned off (SAGA_PDL=0) the path still matches the oracle and
    gives the same bits as with it on."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = (
        "import sys, torch; sys.path.insert(0, %r)\n"
        "from tests import gpu_harness; from tests.test_gpu_parity import small\n"
        "wl = small('pdl', h_q=12, h_k=1, h_v=4, d=128, l_kv=3001, n_top=70, refresh=3, steps=6)\n"
        "_, s = gpu_harness.run_parity(wl, wl.steps, graphs=True)\n"
        "torch.save({'out': s.out.cpu(), 'tau': s.tau.cpu()}, sys.argv[1])\n" % root)
    import tempfile
    res = {}
    with tempfile.TemporaryDirectory() as tmp:
        for flag in ("0", "1"):
            path = os.path.join(tmp, f"pdl_{flag}.pt")
            env = dict(os.environ, SAGA_PDL=flag)
            r = subprocess.run([sys.executable, "-c", code, path], env=env, cwd=root, capture_output=True,
                               text=True, timeout=600)
            assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
            res[flag] = torch.load(path)
    assert torch.equal(res["0"]["out"], res["1"]["out"]) and torch.equal(res["0"]["tau"], res["1"]["tau"])


def test_refresh_select_heavy_bin_falls_back():
    """The refresh's parallel select when the N-th largest lies in a tie of more than 16384 scores (the
    candidate buffer's size): the single-CTA digit scans take over and the threshold is still that score,
    with every tied token kept."""
    L0, N = 20000, 300
    B, hq, hk, hv, d = 1, 4, 1, 4, 64
    g = torch.Generator().manual_seed(5)
    K = torch.ones((B, hk, L0, d)).to(torch.bfloat16)
    bump = torch.randperm(L0, generator=g)[:50]
    K[0, 0, bump] = 2.0  # 50 larger scores, then a 19950-way tie
    V = torch.randn((B, hv, L0, d), generator=g).to(torch.bfloat16)
    q = torch.full((B, hq, d), 0.25).to(torch.bfloat16)
    kn = torch.ones((B, hk, d)).to(torch.bfloat16)
    vn = torch.randn((B, hv, d), generator=g).to(torch.bfloat16)
    l_cap = L0 + 1
    shape = saga.SagaShape.of(B, hq, hk, hv, d, l_cap)
    kc = torch.zeros((B, hk, l_cap, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros((B, hv, l_cap, d), dtype=torch.bfloat16, device="cuda")
    kc[:, :, :L0] = K.cuda()
    vc[:, :, :L0] = V.cuda()
    tau = torch.zeros((B, hq), device="cuda")
    out = torch.zeros((B, hq, d), device="cuda")
    cnt = torch.zeros((B, hq), dtype=torch.int32, device="cuda")
    idx = torch.zeros((B, hq, l_cap), dtype=torch.int32, device="cuda")
    ws = saga.alloc_workspace(shape, "cuda")
    saga.saga_decode_step(shape, q.cuda(), kn.cuda(), vn.cuda(), kc, vc, l_cap, N, 4, 0, tau, out, ws,
                          sel_count=cnt, sel_idx=idx)
    torch.cuda.synchronize()
    orc = saga_oracle.OracleLayer(K.float().numpy(), V.float().numpy(), hq, N, 4, l_cap=l_cap)
    res = orc.step(q.float().numpy(), kn.float().numpy(), vn.float().numpy())
    assert np.array_equal(tau.cpu().numpy(), res["tau"])  # the tied score, exactly
    assert (cnt.cpu().numpy() == res["keep"].sum(-1)).all()  # every tied token kept (more than N)
    assert int(cnt[0, 0]) > 16384
    assert np.max(np.abs(out.cpu().numpy() - res["out"])) <= gpu_harness.OUT_TOL


def test_read_probe_reads_every_word():
    """The pure-read probe touches every 16-byte chunk: the XOR of its per-CTA sink words equals the XOR of
    all 32-bit words of the buffer (a length that is not a multiple of the grid stride)."""
    g = torch.Generator(device="cuda").manual_seed(9)
    n_words = (37 << 20) // 4 + 4 * 1237
    buf = torch.randint(-(1 << 31), (1 << 31) - 1, (n_words,), generator=g, device="cuda", dtype=torch.int64)
    buf = buf.to(torch.int32)
    sink = torch.zeros(saga.load().saga_read_probe_sink_words(), dtype=torch.int32, device="cuda")
    saga.read_probe(buf, sink)
    torch.cuda.synchronize()
    expect = np.bitwise_xor.reduce(buf.cpu().numpy().view(np.uint32))
    got = np.bitwise_xor.reduce(sink.cpu().numpy().view(np.uint32))
    assert got == expect

