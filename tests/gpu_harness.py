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


# ---------------------------------------------------------------------------- full-size sampled parity
def oracle_rows(inp, h_q, h_k, h_v, n_top, refresh, t, b, h):
    """The oracle's result at decode step t for the query heads of key head h, batch b, one group at a time.

    inp holds float32 numpy copies of the bf16 inputs: "K"[(b, h)] and "V"[(b, u)] the prefilled rows
    [l_kv, d] of one head, "q" [steps, B, h_q, d], "k_new" [steps, B, h_k, d], "v_new" [steps, B, h_v, d].
    Rebuilds the caches at steps r = t - t % R and t, takes the threshold from step r's own scores (the
    refresh step) and applies it at step t.  Returns dict(out, tau, keep, scores).
    """
    G = h_q // h_k
    js = list(range(h * G, (h + 1) * G))
    l_kv = inp["K"][(b, h)].shape[0]
    r = t - t % refresh

    def cache(rows0, new, head):
        return np.concatenate([rows0, new[:t + 1, b, head]], axis=0)[None, None]  # [1, 1, L, d]

    Kh = cache(inp["K"][(b, h)], inp["k_new"], h)
    L = Kh.shape[2]
    # eq. 2 for the group's query heads against key head h (the group as the oracle's query heads)
    A_t = saga_oracle.scores(inp["q"][t, b, js][None], Kh, L)[0]  # [G, L]
    L_r = l_kv + r + 1
    if n_top >= L_r:
        tau = np.full(G, -np.inf, dtype=np.float32)
    else:
        A_r = A_t if r == t else saga_oracle.scores(inp["q"][r, b, js][None], Kh, L_r)[0]
        tau = np.array([saga_oracle.nth_largest(A_r[g], n_top) for g in range(G)], dtype=np.float32)
    keep = saga_oracle.select(A_t[None], tau[None])[0]
    outs = np.zeros((G, inp["K"][(b, h)].shape[1]))
    for g, j in enumerate(js):
        u = saga_oracle.value_head(j, h_q, h_v)
        Vh = cache(inp["V"][(b, u)], inp["v_new"], u)
        outs[g] = saga_oracle.sparse_attention(A_t[None, g:g + 1], keep[None, g:g + 1], Vh, L)[0, 0]
    return {"out": outs, "tau": tau, "keep": keep, "scores": A_t}


def run_full_sampled(wl: workload.Workload, check_layers: Sequence[int], check_steps: Sequence[int],
                     check_groups: Sequence[tuple], layers: Optional[int] = None, track: bool = False):
    """All layers of `wl` per step through CUDA-graph replays with a device-side length (the benchmark's
    launch configuration).  Returns the GPU rows of the checked (layer, step, batch, key head) groups, the
    inputs those groups need (float32 numpy) and the N passed to the kernels."""
    nl = wl.layers if layers is None else layers
    steps = max(check_steps) + 1
    l_cap = wl.l_kv + steps
    n_top = wl.n_for_kernel(l_cap)
    shape = saga.SagaShape.of(wl.batch, wl.h_q, wl.h_k, wl.h_v, wl.d, l_cap)
    sess = DecodeSession(shape, nl, n_top, wl.refresh, device="cuda", track_selection=track)
    G = wl.h_q // wl.h_k
    qs, ks, vs, inputs = [], [], [], {}
    for i in range(nl):
        inp = workload.make_layer(wl, i, device="cuda", steps=steps)
        sess.prefill(i, inp["K0"], inp["V0"])
        qs.append(inp["q"])
        ks.append(inp["k_new"])
        vs.append(inp["v_new"])
        if i in check_layers:
            keep = {"K": {}, "V": {}}
            for (b, h) in check_groups:
                keep["K"][(b, h)] = inp["K0"][b, h].float().cpu().numpy()
                for j in range(h * G, (h + 1) * G):
                    u = saga_oracle.value_head(j, wl.h_q, wl.h_v)
                    if (b, u) not in keep["V"]:
                        keep["V"][(b, u)] = inp["V0"][b, u].float().cpu().numpy()
            for k in ("q", "k_new", "v_new"):
                keep[k] = inp[k].float().cpu().numpy()
            inputs[i] = keep
        del inp
    q_all, k_all, v_all = torch.stack(qs, 1), torch.stack(ks, 1), torch.stack(vs, 1)
    del qs, ks, vs
    got = {}

    def grab(t):
        torch.cuda.synchronize()
        for i in check_layers:
            for (b, h) in check_groups:
                js = slice(h * G, (h + 1) * G)
                row = {"out": sess.out[i, b, js].cpu().numpy().astype(np.float64),
                       "tau": sess.tau[i, b, js].cpu().numpy()}
                if track:
                    row["count"] = sess.sel_count[i, b, js].cpu().numpy()
                    row["idx"] = sess.sel_idx[i, b, js].cpu().numpy()
                got[(i, t, b, h)] = row

    sess.step(q_all[0], k_all[0], v_all[0])  # step 0 eagerly, then the step graphs (as the benchmark does)
    sess.capture()
    if 0 in check_steps:
        grab(0)
    for t in range(1, steps):
        sess.stage(q_all[t], k_all[t], v_all[t])
        sess.replay()
        if t in check_steps:
            grab(t)
    torch.cuda.synchronize()
    status = saga.saga_get_status(sess.workspace)
    assert status & saga.SAGA_STATUS_TIMEOUT == 0
    del sess
    return got, inputs, n_top


def check_full_sampled(wl, got, inputs, n_top, track):
    """Compares every grabbed group with the oracle; returns the largest output difference."""
    worst = 0.0
    for (i, t, b, h), row in got.items():
        res = oracle_rows(inputs[i], wl.h_q, wl.h_k, wl.h_v, n_top, wl.refresh, t, b, h)
        err = float(np.max(np.abs(row["out"] - res["out"])))
        assert err <= OUT_TOL, f"layer {i} step {t} b {b} h {h}: max |out diff| {err}"
        worst = max(worst, err)
        with np.errstate(invalid="ignore"):
            both = np.isneginf(res["tau"]) & np.isneginf(row["tau"])
            terr = np.where(both, 0.0, np.abs(row["tau"].astype(np.float64) - res["tau"].astype(np.float64)))
        assert float(np.max(terr)) <= BAND, f"layer {i} step {t}: threshold differs by {float(np.max(terr))}"
        if track:
            L = res["scores"].shape[1]
            keep_g = keep_mask_from_lists(row["count"][None], row["idx"][None], L)[0]
            far = np.abs(res["scores"].astype(np.float64) - res["tau"].astype(np.float64)[:, None]) > BAND
            mism = (keep_g != res["keep"]) & far
            assert not mism.any(), f"layer {i} step {t}: {int(mism.sum())} index mismatches outside the band"
    return worst


# ---------------------------------------------------------------------------- full-size parity, every layer and step
def layer_inputs_on_gpu(wl, steps):
    """Every layer's inputs, drawn with the seeded generator on the CPU (so that a worker process can draw
    the same bytes again) and moved to the GPU."""
    layers = []
    for i in range(wl.layers):
        inp = workload.make_layer(wl, i, device="cpu", steps=steps)
        layers.append({k: v.cuda() for k, v in inp.items()})
        del inp
    return layers


def run_full_all(wl, inputs, steps, track=False, record_idx=False, layer_batched=False):
    """All layers of `wl` per step through CUDA-graph replays with a device-side length (the benchmark's
    launch configuration) for `steps` steps.  Returns, per layer, per step: out, tau and (track) the kept
    counts and (record_idx) each row's kept positions.  layer_batched: every layer of a step in one call."""
    l_cap = wl.l_kv + steps
    n_top = wl.n_for_kernel(l_cap)
    shape = saga.SagaShape.of(wl.batch, wl.h_q, wl.h_k, wl.h_v, wl.d, l_cap)
    sess = DecodeSession(shape, wl.layers, n_top, wl.refresh, device="cuda", track_selection=track,
                         layer_batched=layer_batched)
    for i, inp in enumerate(inputs):
        sess.prefill(i, inp["K0"], inp["V0"])
    q_all = torch.stack([inp["q"] for inp in inputs], 1)
    k_all = torch.stack([inp["k_new"] for inp in inputs], 1)
    v_all = torch.stack([inp["v_new"] for inp in inputs], 1)
    per_layer = [[None] * steps for _ in range(wl.layers)]
    H = wl.batch * wl.h_q

    def grab(t):
        torch.cuda.synchronize()
        out = sess.out.float().cpu().numpy()
        tau = sess.tau.cpu().numpy()
        cnt = sess.sel_count.cpu().numpy() if track else None
        idx = None
        if record_idx:
            m = max(1, int(cnt.max()))
            idx = sess.sel_idx[..., :m].cpu().numpy()
        for i in range(wl.layers):
            row = {"out": out[i], "tau": tau[i]}
            if track:
                row["count"] = cnt[i]
            if record_idx:
                flat_c = cnt[i].reshape(H)
                flat_i = idx[i].reshape(H, -1)
                row["idx"] = [flat_i[r, :flat_c[r]].copy() for r in range(H)]
            per_layer[i][t] = row

    sess.step(q_all[0], k_all[0], v_all[0])  # step 0 eagerly, then the step graphs (as the benchmark does)
    sess.capture()
    grab(0)
    for t in range(1, steps):
        sess.stage(q_all[t], k_all[t], v_all[t])
        sess.replay()
        grab(t)
    status = saga.saga_get_status(sess.workspace)
    assert status & saga.SAGA_STATUS_TIMEOUT == 0
    del sess
    return per_layer, n_top, l_cap


def check_full_all(wl, per_layer, n_top, l_cap, steps, workers=None):
    """Every layer against the stepping oracle, one layer per worker process (spawned: the parent holds a
    CUDA context).  Returns the workers' summaries."""
    import concurrent.futures
    import multiprocessing
    import os
    cores = len(os.sched_getaffinity(0))
    workers = workers or max(1, min(wl.layers, cores // 2, 16))
    threads = max(1, cores // workers)
    from tests import fullsize_oracle
    tasks = [{"wl": wl, "layer": i, "steps": steps, "n_top": n_top, "l_cap": l_cap, "gpu": per_layer[i],
              "threads": threads} for i in range(wl.layers)]
    ctx = multiprocessing.get_context("spawn")
    with concurrent.futures.ProcessPoolExecutor(max_workers=workers, mp_context=ctx) as ex:
        return list(ex.map(fullsize_oracle.check_layer, tasks))
