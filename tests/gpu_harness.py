"""Runs the CUDA decode path and the CPU oracle side by side on the same seeded inputs.

Acceptance (per decode step, per layer, batch b, query head j):
* index sets: for every token i whose oracle score lies more than BAND from
  the oracle threshold, "kept on the GPU" equals "kept by the oracle";
* output: max |O_gpu - O_oracle| <= OUT_TOL (bf16 inputs, fp32 accumulation);
* threshold: |tau_gpu - tau_oracle| <= BAND (each side takes the N-th
  largest of its own fp32 scores).
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np
import torch

from long_context_decoding_saga_b200 import saga, workload
from long_context_decoding_saga_b200.session import DecodeSession
from oracle import saga_oracle

BAND = 1e-3
OUT_TOL = 1e-2


@dataclasses.dataclass
class StepReport:
    t: int
    refreshed: bool
    max_out_err: float
    max_tau_err: float
    band_tokens: int
    kept_min: int
    kept_max: int


def keep_mask_from_lists(count: np.ndarray, idx: np.ndarray, L: int) -> np.ndarray:
    B, H = count.shape
    m = np.zeros((B, H, L), dtype=bool)
    for b in range(B):
        for j in range(H):
            c = int(count[b, j])
            sel = idx[b, j, :c]
            assert (np.diff(sel) > 0).all(), "index list not strictly ascending"
            assert c == 0 or (sel[0] >= 0 and sel[-1] < L), "index out of range"
            m[b, j, sel] = True
    return m


def compare_step(res, out_gpu, tau_gpu, count, idx, t) -> StepReport:
    L = res["L"]
    A, tau_o, keep_o = res["scores"], res["tau"], res["keep"]
    keep_g = keep_mask_from_lists(count, idx, L)
    assert (count == keep_g.sum(-1)).all()
    far = np.abs(A.astype(np.float64) - tau_o.astype(np.float64)[..., None]) > BAND
    mism = (keep_g != keep_o) & far
    assert not mism.any(), f"step {t}: {int(mism.sum())} index-set mismatches outside the band"
    err = float(np.max(np.abs(out_gpu.astype(np.float64) - res["out"]))) if out_gpu.size else 0.0
    assert err <= OUT_TOL, f"step {t}: max |out diff| {err}"
    with np.errstate(invalid="ignore"):
        both_inf = np.isneginf(tau_o) & np.isneginf(tau_gpu)
        terr = np.where(both_inf, 0.0, np.abs(tau_gpu.astype(np.float64) - tau_o.astype(np.float64)))
    tmax = float(np.max(terr))
    assert tmax <= BAND, f"step {t}: threshold differs by {tmax}"
    kept = keep_g.sum(-1)
    return StepReport(t, bool(res["refreshed"]), err, tmax, int((~far).sum()), int(kept.min()), int(kept.max()))


def run_parity(wl: workload.Workload, steps: int, layer: int = 0, gen_device: str = "cpu", graphs: bool = False,
               out_dtype=torch.float32, check_steps: Optional[Sequence[int]] = None):
    """Run `steps` decode steps of one layer on the GPU and in the oracle; compare every checked step."""
    inp = workload.make_layer(wl, layer, device=gen_device, steps=steps)
    l_cap = wl.l_kv + steps
    n_top = wl.n_for_kernel(l_cap)
    shape = saga.SagaShape.of(wl.batch, wl.h_q, wl.h_k, wl.h_v, wl.d, l_cap)
    sess = DecodeSession(shape, 1, n_top, wl.refresh, device="cuda", out_dtype=out_dtype, track_selection=True)
    sess.prefill(0, inp["K0"].cuda(), inp["V0"].cuda())
    orc = saga_oracle.OracleLayer(inp["K0"].float().cpu().numpy(), inp["V0"].float().cpu().numpy(), wl.h_q, n_top,
                                  wl.refresh, l_cap=l_cap)
    q_all = inp["q"].cuda()
    k_all = inp["k_new"].cuda()
    v_all = inp["v_new"].cuda()
    reports = []
    for t in range(steps):
        q, kn, vn = q_all[t:t + 1], k_all[t:t + 1], v_all[t:t + 1]
        if graphs:
            if t == 0:
                sess.step(q, kn, vn)  # first step eagerly, then record the graphs
                sess.capture()
            else:
                sess.stage(q, kn, vn)
                sess.replay()
        else:
            sess.step(q, kn, vn)
        res = orc.step(inp["q"][t].float().cpu().numpy(), inp["k_new"][t].float().cpu().numpy(),
                       inp["v_new"][t].float().cpu().numpy())
        if check_steps is not None and t not in check_steps:
            continue
        torch.cuda.synchronize()
        out = sess.out[0].float().cpu().numpy()
        tau = sess.tau[0].cpu().numpy()
        cnt = sess.sel_count[0].cpu().numpy()
        idx = sess.sel_idx[0].cpu().numpy()
        reports.append(compare_step(res, out, tau, cnt, idx, t))
    status = saga.saga_get_status(sess.workspace)
    assert status & saga.SAGA_STATUS_TIMEOUT == 0
    return reports, sess
