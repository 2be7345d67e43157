"""Benchmark of the SAGA + Atop-N decode-attention step on B200.

One step = one decode step of every layer of the workload: for each layer,
one saga_decode_step call (the new token's key/value rows are appended by
the attention kernels, then the attention step: Atop-N threshold refresh on
t % R == 0, else reuse).  The step runs as a CUDA graph
replay; caches live in HBM.  Default workload: the Qwen2.5-1.5B-shaped SAGA
configuration at 128K context (h_q=12, d=128, h_k=1, h_v=4, N=512, R=32,
28 layers, batch 1 per GPU).

Printed JSON (rank 0, one line):
  value        whole-job algorithmic HBM GB/s (all ranks; bytes per the
               key/value read model below), inputs already resident
  ms_per_step  max over ranks of the mean step time
  e2e          the same metric with this step's q/k_new/v_new copied from
               pinned host memory and every layer's output copied back,
               inside the timed region
  roofline     the context-split attention kernel: algorithmic bytes of one
               layer-step / its in-step time (the reuse step's time per
               layer, shared with the combine in proportion to their
               CUDA-event durations measured in isolation, which are also
               reported) vs the measured HBM copy bandwidth, and vs the
               pure-read ceiling of the library's read probe
  read_probe   that ceiling: one streaming read of 4 GiB, best of 5
  workloads    (N=1) the other configurations, timed the same way with a
               short window each: Llama-SAGA 32K, dense GQA 128K and the
               128K sweep points at batch 1/4/16 with 1 and 8 key heads
  cpu_baseline the CPU oracle on a bounded sample (rank 0, N=1)

Algorithmic bytes of one layer-step:
  2*B*d*(h_k*L + min(h_q*N, h_v*L)) + 2*B*h_q*d (q) + 4*B*h_q*d (fp32 out)
(every cached key of every key head, N value rows per query head or each value
row once when N covers the context, the query, the output).

`--impl reference` times the CPU oracle as it stands on this host's cores
(the reference arm; rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode-attn µs/step and achieved HBM GB/s (% roofline) at 128K ctx, h_k=1..8"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_PATH = os.path.join(ROOT, "profiles", "split_kernel_traffic.json")
FALLBACK_HBM_GBS = 6650.0


def layer_bytes(wl, L):
    n = L if wl.dense else wl.n_top
    keys = wl.h_k * L
    vals = min(wl.h_q * n, wl.h_v * L)
    return 2 * wl.batch * wl.d * (keys + vals) + 2 * wl.batch * wl.h_q * wl.d + 4 * wl.batch * wl.h_q * wl.d


def code_tokens(text):
    """C/CUDA source with comments removed and whitespace collapsed (string and character literals kept
    as written), so that a comment edit leaves the kernel's hash unchanged."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
            out.append(" ")
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash():
    """Hash of the split kernel's sources (code only): the key of the recorded DRAM-traffic figure."""
    h = hashlib.sha256()
    for f in ("saga_kernels.cu", "saga_device.cuh", "saga_internal.h"):
        with open(os.path.join(ROOT, "long_context_decoding_saga_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(code_tokens(fh.read()).encode())
    return h.hexdigest()[:16]


def load_peak():
    try:
        with open(PEAKS_PATH) as f:
            v = float(json.load(f)["hbm_gbs"])
            return v, "measured"
    except Exception:  # noqa: BLE001
        return FALLBACK_HBM_GBS, "fallback"


def load_traffic(workload_name):
    try:
        with open(TRAFFIC_PATH) as f:
            t = json.load(f)
        if t.get("kernel_hash") != kernel_source_hash() or t.get("workload") != workload_name:
            return None
        return float(t["bytes_per_launch"])
    except Exception:  # noqa: BLE001
        return None


class ClockSampler:
    """SM clock and clock-event reasons sampled during the timed region.

    Polls NVML from a thread every `period` seconds, plus one sample when it
    starts and one when it stops, so even a timed region of a few ms is
    covered.  Reads only; changes no setting.  Falls back to nvidia-smi when
    the NVML binding is missing.
    """

    REASONS = (("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20), ("hw_thermal_slowdown", 0x40),
               ("sw_power_cap", 0x4))

    def __init__(self, device_index, period=0.002):
        self.device_index = device_index
        self.period = period
        self.samples = []  # (sm_mhz, max_mhz, reason_bits)
        self._stop = threading.Event()
        self.thread = None
        self.handle = None
        self.nvml = None

    def _open(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.device_index)
        bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
        self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        self.nvml = pynvml

    def _sample(self):
        n = self.nvml
        sm = n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM)
        mx = n.nvmlDeviceGetMaxClockInfo(self.handle, n.NVML_CLOCK_SM)
        get_reasons = getattr(n, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            n.nvmlDeviceGetCurrentClocksThrottleReasons
        self.samples.append((sm, mx, int(get_reasons(self.handle))))

    def _loop(self):
        while not self._stop.wait(self.period):
            try:
                self._sample()
            except Exception:  # noqa: BLE001
                return

    def start(self):
        try:
            self._open()
            self._sample()
        except Exception:  # noqa: BLE001
            self.handle = None
            return
        self.thread = threading.Thread(target=self._loop, daemon=True)
        self.thread.start()

    def stop(self):
        if self.handle is None:
            return None
        self._stop.set()
        self.thread.join(timeout=2)
        try:
            self._sample()
        except Exception:  # noqa: BLE001
            pass
        sm = [x[0] for x in self.samples]
        reasons = sorted({name for _, _, bits in self.samples for name, bit in self.REASONS if bits & bit})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(x[1] for x in self.samples),
                "reasons": reasons, "samples": len(self.samples), "source": "nvml"}


def oracle_threads():
    """Threads the numpy oracle can use (its BLAS pool; sorts and exps are single-threaded)."""
    n = len(os.sched_getaffinity(0))
    try:
        from threadpoolctl import threadpool_info
        blas = [int(i.get("num_threads", 0)) for i in threadpool_info() if i.get("user_api") == "blas"]
        if blas:
            n = max(blas)
    except Exception:  # noqa: BLE001
        pass
    return n


def cpu_baseline(wl, seconds_budget=10.0, max_steps=512):
    """The oracle as it stands, on a bounded sample: consecutive decode steps of layer 0 at full size,
    from a refresh step on, until `seconds_budget` has passed and the steps cover whole refresh periods
    (or three times the budget has passed, or `max_steps` steps were made)."""
    from long_context_decoding_saga_b200 import workload
    from oracle import saga_oracle

    cores = oracle_threads()
    inp = workload.make_layer(wl, 0, device="cpu", steps=max_steps)
    orc = saga_oracle.OracleLayer(inp["K0"].float().numpy(), inp["V0"].float().numpy(), wl.h_q,
                                  wl.n_for_kernel(wl.l_kv + max_steps), wl.refresh, l_cap=wl.l_kv + max_steps)
    t0 = time.perf_counter()
    done, nbytes, refreshes = 0, 0, 0
    for t in range(max_steps):
        orc.step(inp["q"][t].float().numpy(), inp["k_new"][t].float().numpy(), inp["v_new"][t].float().numpy())
        done += 1
        nbytes += layer_bytes(wl, wl.l_kv + t + 1)
        refreshes += int(t % wl.refresh == 0)
        el = time.perf_counter() - t0
        whole = wl.refresh > 1024 or (t + 1) % wl.refresh == 0
        if (el > seconds_budget and whole) or el > 3 * seconds_budget:
            break
    dt = time.perf_counter() - t0
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} consecutive decode steps of layer 0 at full size ({refreshes} of them refresh "
                      f"steps), numpy oracle, {dt:.1f} s",
            "us_per_layer_step": dt / done * 1e6, "us_per_step_scaled": dt / done * 1e6 * wl.layers}


def refresh_count(first, steps, refresh):
    """Refresh steps (t % refresh == 0) among t = first .. first + steps - 1."""
    return sum(1 for t in range(first, first + steps) if t % refresh == 0)


def alignment_from(first, refresh, steps):
    """Untimed steps to run before a window of `steps` steps that would start at step `first`, so that
    the window holds the nearest whole number to steps / R of refresh steps (halves rounded up):
    exactly steps / R when R divides it, else the nearer of floor and ceil.  None for a schedule that
    never refreshes again."""
    if refresh > 1024:
        return 0
    target = int(steps / refresh + 0.5)
    for a in range(refresh):
        if refresh_count(first + a, steps, refresh) == target:
            return a
    return 0


def alignment_steps(warmup, refresh, steps):
    """alignment_from for the timed window, which follows the first (eager) step and the warm-up."""
    return alignment_from(1 + warmup, refresh, steps)


def step_plan(warmup, steps, refresh, e2e=True):
    """The decode steps a run makes, in order: 1 eager step, `warmup` untimed steps, A untimed steps that
    place the timed window, K = `steps` timed steps, A2 untimed steps that place the end-to-end window,
    E end-to-end steps, T kernel-timing replays; `total` sizes the caches (l_kv + total)."""
    A = alignment_steps(warmup, refresh, steps)
    E = max(4, min(steps, 64)) if e2e else 0
    A2 = alignment_from(1 + warmup + A + steps, refresh, E) if E else 0
    T = max(2, min(steps, 8))
    return {"A": A, "E": E, "A2": A2, "T": T, "total": 1 + warmup + A + steps + A2 + E + T,
            "timed_first": 1 + warmup + A, "e2e_first": 1 + warmup + A + steps + A2}


def step_means(step_ms, kinds, refresh):
    """Mean refresh-step and reuse-step times (µs) of the timed steps and, when both kinds were timed,
    their amortized mean over one refresh period."""
    ref = [t for t, k in zip(step_ms, kinds) if k]
    reuse = [t for t, k in zip(step_ms, kinds) if not k]
    out = {"refresh_mean_us": statistics.mean(ref) * 1e3 if ref else None,
           "reuse_mean_us": statistics.mean(reuse) * 1e3 if reuse else None}
    if ref and reuse and refresh <= 1024:
        out["amortized_us"] = (out["refresh_mean_us"] + (refresh - 1) * out["reuse_mean_us"]) / refresh
    return out


def gather_rank_stats(local, world):
    """Every rank's timing record, in rank order (one all_gather over the process group: NCCL or gloo)."""
    if world == 1:
        return [local]
    import torch.distributed as dist
    out = [None] * world
    dist.all_gather_object(out, local)
    return out


def combine_rank_stats(per_rank, steps):
    """Whole-job figures under weak scaling: the bytes of all ranks over the slowest rank's time."""
    ms_max = max(r["ms"] for r in per_rank)
    total = sum(r["bytes"] for r in per_rank)
    e_ms = max(r["e2e_ms"] for r in per_rank)
    e_total = sum(r["e2e_bytes"] for r in per_rank)
    return {"value": total / (ms_max / 1e3) / 1e9, "ms_max": ms_max, "ms_per_step": ms_max / steps,
            "e2e_value": e_total / (e_ms / 1e3) / 1e9 if e_ms > 0 else None}


def workload_config(wl, world):
    """The `config` object of the JSON line: the workload and its shape, identical for both arms (the
    run-specific window and L2 handling go in a separate `window` object)."""
    return {"workload": wl.name, "batch_per_gpu": wl.batch, "l_kv": wl.l_kv, "h_q": wl.h_q, "h_k": wl.h_k,
            "h_v": wl.h_v, "d": wl.d, "n_top": wl.n_top if not wl.dense else "dense", "refresh": wl.refresh,
            "layers": wl.layers, "parallelism": f"replicas{world}"}


def run_reference(args, wl, rank, world):
    if rank != 0:
        return 0
    # each step: a bounded sample of the workload (layer 0, one decode step, full size)
    from long_context_decoding_saga_b200 import workload
    from oracle import saga_oracle
    inp = workload.make_layer(wl, 0, device="cpu", steps=args.warmup + args.steps)
    l_cap = wl.l_kv + args.warmup + args.steps
    orc = saga_oracle.OracleLayer(inp["K0"].float().numpy(), inp["V0"].float().numpy(), wl.h_q,
                                  wl.n_for_kernel(l_cap), wl.refresh, l_cap=l_cap)
    times, nbytes = [], 0
    for t in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        orc.step(inp["q"][t].float().numpy(), inp["k_new"][t].float().numpy(), inp["v_new"][t].float().numpy())
        dt = time.perf_counter() - t0
        if t >= args.warmup:
            times.append(dt)
            nbytes += layer_bytes(wl, wl.l_kv + t + 1)
    total = sum(times)
    value = nbytes / total / 1e9
    cores = oracle_threads()
    sample = (f"each timed step: one decode step of layer 0 of the workload at full size (a bounded sample of "
              f"the {wl.layers}-layer step; ms_per_step is that one layer-step as timed), numpy oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total / len(times) * 1e3, "timed_unit": "one layer-step (layer 0)",
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, world),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def make_session(wl, dev, rank, total_steps, layer_batched=False):
    """A DecodeSession holding every layer of `wl` (caches prefilled with the seeded synthetic rows, one
    rank's seed per rank) and the per-step inputs of `total_steps` decode steps, stacked [steps, layers, ...].
    layer_batched: all layers of a step in one call (batch = layers x B)."""
    import torch

    from long_context_decoding_saga_b200 import saga, workload
    from long_context_decoding_saga_b200.session import DecodeSession

    l_cap = wl.l_kv + total_steps
    n_top = wl.n_for_kernel(l_cap)
    shape = saga.SagaShape.of(wl.batch, wl.h_q, wl.h_k, wl.h_v, wl.d, l_cap)
    sess = DecodeSession(shape, wl.layers, n_top, wl.refresh, device=dev, layer_batched=layer_batched)
    qs, ks, vs = [], [], []
    for i in range(wl.layers):
        inp = workload.make_layer(wl.with_(seed=wl.seed + 7919 * rank), i, device=dev, steps=total_steps)
        sess.prefill(i, inp["K0"], inp["V0"])
        qs.append(inp["q"])
        ks.append(inp["k_new"])
        vs.append(inp["v_new"])
        del inp
    q_all = torch.stack(qs, dim=1)  # [steps, layers, B, h_q, d]
    k_all = torch.stack(ks, dim=1)
    v_all = torch.stack(vs, dim=1)
    del qs, ks, vs
    torch.cuda.synchronize()
    return sess, (q_all, k_all, v_all), shape, n_top, l_cap


def l2_flush_wanted(wl, mode, l2_bytes):
    """Whether timed steps get a 2 x L2 write between them: a step whose streamed bytes are under twice the
    L2 would find part of its inputs still in L2 from the step before."""
    step_bytes = wl.layers * layer_bytes(wl, wl.l_kv)
    return mode == "on" or (mode == "auto" and step_bytes < 2 * l2_bytes), step_bytes


def l2_note(flush, step_bytes, l2_bytes):
    if flush:
        return "flushed between timed steps (a 2 x L2 write outside each step's events)"
    if step_bytes >= 2 * l2_bytes:
        return "inputs exceed twice the L2 (all layers' caches cycle through L2 each step)"
    return "inputs fit in twice the L2; not flushed (--flush-l2 off)"


def timed_window(sess, inputs, cur, K, wl, flush, scratch):
    """K decode steps (graph replays), each bracketed by CUDA events: back to back (the end mark of one step
    starts the next) or, with `flush`, one by one with the L2 write outside the events.  Returns per-step
    ms, which steps refreshed, the algorithmic bytes and the next input index."""
    import torch
    q_all, k_all, v_all = inputs
    marks = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    kinds, nbytes = [], 0
    for s_i in range(K):
        nbytes += wl.layers * layer_bytes(wl, sess.length + 1)
        kinds.append(sess.t % wl.refresh == 0)
        if flush or s_i == 0:
            marks[s_i][0].record()
        sess.stage(q_all[cur], k_all[cur], v_all[cur])
        sess.replay()
        marks[s_i][1].record()
        if flush:
            scratch.fill_(float(s_i))
        cur += 1
    torch.cuda.synchronize()
    step_ms = []
    for s_i in range(K):
        start_ev = marks[s_i][0] if (flush or s_i == 0) else marks[s_i - 1][1]
        step_ms.append(start_ev.elapsed_time(marks[s_i][1]))
    return step_ms, kinds, nbytes, cur


def read_peak_probe(dev, gib=4, repeats=5):
    """The pure-read HBM ceiling: the library's read probe over a 4 GiB buffer (32 x the L2), best of
    `repeats` CUDA-event timings."""
    import torch

    from long_context_decoding_saga_b200 import saga
    buf = torch.empty(gib << 30, dtype=torch.uint8, device=dev)
    buf.fill_(1)
    sink = saga.read_probe(buf)  # warm-up
    best = None
    for _ in range(repeats):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        saga.read_probe(buf, sink)
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b)
        best = ms if best is None else min(best, ms)
    del buf
    return {"gbs": (gib << 30) / (best / 1e3) / 1e9, "bytes": gib << 30, "best_ms": best, "repeats": repeats,
            "kernel": "saga_read_probe (16-byte streaming loads, 4 in flight per thread)"}


# Workloads timed after the headline, in the same process, each with a short window: the Llama-shaped SAGA
# configuration at 32K, the dense GQA configuration at 128K, and the 128K sweep points at batch 1, 4 and 16
# with 1 and 8 key heads (N = 256, R = 16).  The batch-4/16 points hold fewer layers (their caches are
# 0.6-4.3 GB per layer); every entry says how many it ran.
EXTRA_WORKLOADS = (
    ("llama3.2-1b_saga_32k", 0),
    ("llama3.2-1b_dense_gqa_128k", 0),
    ("sweep_l131072_b1_hk1_n256_r16", 0),
    ("sweep_l131072_b1_hk8_n256_r16", 0),
    ("sweep_l131072_b4_hk1_n256_r16", 8),
    ("sweep_l131072_b4_hk8_n256_r16", 8),
    ("sweep_l131072_b16_hk1_n256_r16", 4),
    ("sweep_l131072_b16_hk8_n256_r16", 4),
)

# The same step with every layer in one call (the layers as a batch of layers x B: one kernel hand-off
# chain per step instead of one per layer; needs all layers' queries of the step at once).
LAYER_BATCHED_WORKLOADS = (
    "qwen2.5-1.5b_saga_128k",
    "llama3.2-1b_saga_32k",
    "llama3.2-1b_dense_gqa_128k",
    "sweep_l4096_b1_hk2_n256_r16",
)


def time_key_head_merge(dev, tokens=4096, hidden=2048, d=64, h_q=32, h_k=8, repeats=3):
    """The closed-form key-head merge on a Llama-3.2-1B-shaped teacher (8 key heads merged into 4), synthetic
    bf16 X and Q, fp32 W_K: the whole call (transposes, tensor-core Gram products, fp64 pseudoinverses,
    losses and matching), best of `repeats` CUDA-event timings after one warm-up call."""
    import torch

    from long_context_decoding_saga_b200 import saga
    g = torch.Generator(device=dev).manual_seed(123)
    x = torch.randn((tokens, hidden), generator=g, device=dev).to(torch.bfloat16)
    q = torch.randn((tokens, h_q, d), generator=g, device=dev).to(torch.bfloat16)
    w = torch.randn((h_k, hidden, d), generator=g, device=dev) * hidden ** -0.5
    loss, pairing, merged, ws = saga.key_head_merge(x, q, w, h_k)
    best = None
    for _ in range(repeats):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        saga.key_head_merge(x, q, w, h_k, workspace=ws)
        b.record()
        torch.cuda.synchronize()
        best = a.elapsed_time(b) if best is None else min(best, a.elapsed_time(b))
    gram_flop = 2.0 * hidden * hidden * tokens + 2.0 * d * d * tokens * h_q
    status = saga.saga_get_status(ws)
    del x, q, w, ws, merged
    return {"tokens": tokens, "hidden": hidden, "d": d, "h_q": h_q, "h_k": h_k, "us": best * 1e3,
            "gram_tflop": gram_flop / 1e12, "gram_tflops_over_whole_call": gram_flop / (best / 1e3) / 1e12,
            "pairing": pairing.cpu().tolist(), "status_word": status}


QKV_SHAPES = (  # (name, batch, hidden, h_q, h_k, h_v, d): the SAGA students' decode-step projections
    ("llama32_1b_saga_b1", 1, 2048, 32, 2, 8, 64),
    ("llama32_1b_saga_b16", 16, 2048, 32, 2, 8, 64),
    ("qwen25_1p5b_saga_b1", 1, 1536, 12, 1, 4, 128),
    ("qwen25_1p5b_saga_b16", 16, 1536, 12, 1, 4, 128),
)


def time_qkv_projection(dev, peak_gbs, layers=24, replays=5):
    """The fused QKV projection + KV-cache append (eq. 1 with SAGA head counts) as a model runs it: one
    launch per layer, each layer with its own weights (24 layers of distinct weights exceed L2 for both
    shapes, so every launch streams its weights from HBM), replayed as one CUDA graph; per-launch time =
    graph time / layers, best of `replays`.  Algorithmic bytes per launch: the weight matrix, x, the
    query and the new key/value rows."""
    import torch

    from long_context_decoding_saga_b200 import saga
    out = {}
    for name, B, D, h_q, h_k, h_v, d in QKV_SHAPES:
        g = torch.Generator(device=dev).manual_seed(7)
        n_cols = (h_q + h_k + h_v) * d
        shape = saga.SagaShape.of(B, h_q, h_k, h_v, d, 64)
        xs = [torch.randn((B, D), generator=g, device=dev).to(torch.bfloat16) for _ in range(layers)]
        ws = [(torch.randn((n_cols, D), generator=g, device=dev) * D ** -0.5).to(torch.bfloat16)
              for _ in range(layers)]
        q = torch.empty((B, h_q, d), dtype=torch.bfloat16, device=dev)
        kc = torch.zeros((B, h_k, 64, d), dtype=torch.bfloat16, device=dev)
        vc = torch.zeros((B, h_v, 64, d), dtype=torch.bfloat16, device=dev)
        work = saga.alloc_qkv_workspace(shape, D, dev)
        stream = torch.cuda.Stream(device=dev)
        with torch.cuda.stream(stream):
            for i in range(layers):  # eager warm-up (also sets the kernels' shared-memory limits)
                saga.saga_qkv_project(shape, xs[i], ws[i], q, kc, vc, 5, workspace=work, stream=stream)
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for i in range(layers):
                saga.saga_qkv_project(shape, xs[i], ws[i], q, kc, vc, 5, workspace=work, stream=stream)
        best = None
        for _ in range(replays + 1):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                a.record(stream)
                graph.replay()
                b.record(stream)
            stream.synchronize()
            ms = a.elapsed_time(b) / layers
            best = ms if best is None else min(best, ms)
        nbytes = 2 * (n_cols * D + B * D + B * n_cols)
        gbs = nbytes / (best * 1e-3) / 1e9
        out[name] = {"batch": B, "hidden": D, "h_q": h_q, "h_k": h_k, "h_v": h_v, "d": d, "us_per_launch": best * 1e3,
                     "bytes_per_launch": nbytes, "gbs": gbs, "frac_of_peak": gbs / peak_gbs, "layers": layers,
                     "gpu_launches": layers * (replays + 1), "status_word": saga.saga_get_status(work),
                     "kernel": "saga_qkv_kernel (CUDA cores)" if B == 1 else "saga_qkv_mma_kernel (tcgen05)"}
        del graph, xs, ws, q, kc, vc, work
    return out


def time_extra_workload(wl, dev, rank, args, peak, l2_bytes, layer_batched=False):
    """One entry of the `workloads` object: graph-replayed decode steps of `wl` (K = max(16, R) when R is
    at most 64, so the window holds refresh and reuse steps in their proportion), inputs resident."""
    import torch
    W = 3
    K = wl.refresh if wl.refresh <= 64 and wl.refresh > 16 else 16
    plan = step_plan(W, K, wl.refresh, e2e=False)
    sess, inputs, _, _, _ = make_session(wl, dev, rank, plan["total"], layer_batched=layer_batched)
    q_all, k_all, v_all = inputs
    sess.step(q_all[0], k_all[0], v_all[0])
    sess.capture(torch.cuda.Stream(dev))
    cur = 1
    for _ in range(W + plan["A"]):
        sess.stage(q_all[cur], k_all[cur], v_all[cur])
        sess.replay()
        cur += 1
    torch.cuda.synchronize()
    flush, step_bytes = l2_flush_wanted(wl, args.flush_l2, l2_bytes)
    scratch = torch.empty(2 * l2_bytes // 4, dtype=torch.float32, device=dev) if flush else None
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    sampler.start()
    step_ms, kinds, nbytes, cur = timed_window(sess, inputs, cur, K, wl, flush, scratch)
    clocks = sampler.stop()
    ms = sum(step_ms)
    gbs = nbytes / (ms / 1e3) / 1e9
    entry = {"layers": wl.layers, "batch": wl.batch, "h_k": wl.h_k, "l_kv": wl.l_kv,
             "n_top": wl.n_top if not wl.dense else "dense", "refresh": wl.refresh, "steps": K,
             "refresh_steps": int(sum(kinds)), "us_per_step": ms / K * 1e3, "gb_s": gbs, "frac": gbs / peak,
             "step_us": step_means(step_ms, kinds, wl.refresh), "l2": l2_note(flush, step_bytes, l2_bytes),
             "clocks": clocks, "status_word": None, "layers_in_one_call": layer_batched,
             "launches_per_step": {"reuse": sess.launches_per_step(False), "refresh": sess.launches_per_step(True)}}
    from long_context_decoding_saga_b200 import saga
    entry["status_word"] = saga.saga_get_status(sess.workspace)
    del sess, inputs, q_all, k_all, v_all, scratch
    torch.cuda.empty_cache()
    return entry


def kernel_timing(sess, shape, n_top, wl, inputs, cur, T, stream):
    """Per-layer durations of the context-split attention kernel and of the cross-split combine on reuse
    steps, each bracketed by CUDA events on the launching stream inside a freshly recorded graph (the events
    serialise the kernels: these are isolated durations, without the launch overlap of the real step)."""
    import torch

    from long_context_decoding_saga_b200 import saga
    q_all, k_all, v_all = inputs
    split_ms, comb_ms = [], []
    if wl.refresh <= 1 or T <= 0:
        return split_ms, comb_ms, cur
    # per layer: start of the split kernel, end of the split kernel = start of the combine; the combine of
    # layer i ends where layer i + 1's split kernel starts (nothing else runs in between)
    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(2)) for _ in range(wl.layers)]
    g = torch.cuda.CUDAGraph()
    L_est = sess.length + 1
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=stream):
        sess.seq_len_dev.add_(1)
        for i in range(wl.layers):
            saga.saga_trace_next_attention(evs[i][0], evs[i][1])
            saga.saga_decode_step(shape, sess.q_buf[i], sess.k_buf[i], sess.v_buf[i], sess.k_cache[i],
                                  sess.v_cache[i], L_est, n_top, wl.refresh, 1, sess.tau[i], sess.out[i],
                                  sess.workspace, seq_len_dev=sess.seq_len_dev)
    sess.seq_len_dev.fill_(sess.length)
    for _ in range(T):
        sess.stage(q_all[cur], k_all[cur], v_all[cur])
        if sess.t % wl.refresh == 0:  # keep the refresh schedule: refresh steps run with the step graphs
            sess.replay()
            cur += 1
            continue
        g.replay()
        sess.length += 1
        sess.t += 1
        cur += 1
        torch.cuda.synchronize()
        split_ms.extend(a.elapsed_time(b) for a, b in evs)
        comb_ms.extend(evs[i][1].elapsed_time(evs[i + 1][0]) for i in range(wl.layers - 1))
    del g
    return split_ms, comb_ms, cur


def run_saga(args, wl, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from long_context_decoding_saga_b200 import build as build_mod
    from long_context_decoding_saga_b200 import saga, workload

    build_mod.build()
    saga.load()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)

    W, K = args.warmup, args.steps
    plan = step_plan(W, K, wl.refresh, not args.no_e2e)
    A, E, A2, T = plan["A"], plan["E"], plan["A2"], plan["T"]
    sess, inputs, shape, n_top, l_cap = make_session(wl, dev, rank, plan["total"])
    q_all, k_all, v_all = inputs

    # step 0 eagerly (warms launch attributes), then record the step graphs
    sess.step(q_all[0], k_all[0], v_all[0])
    stream = torch.cuda.Stream(dev)
    sess.capture(stream)
    cur = 1

    def replay_range(n):
        nonlocal cur
        for _ in range(n):
            sess.stage(q_all[cur], k_all[cur], v_all[cur])
            sess.replay()
            cur += 1

    replay_range(W + A)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    flush, step_bytes = l2_flush_wanted(wl, args.flush_l2, l2_bytes)
    scratch = torch.empty(2 * l2_bytes // 4, dtype=torch.float32, device=dev) if flush else None
    sampler = ClockSampler(dev.index if dev.index is not None else local_rank)
    sampler.start()
    torch.cuda.nvtx.range_push("bench_timed")
    step_ms, kinds, bytes_timed, cur = timed_window(sess, inputs, cur, K, wl, flush, scratch)
    torch.cuda.nvtx.range_pop()
    clocks = sampler.stop()
    ms = sum(step_ms)
    step_stats = step_means(step_ms, kinds, wl.refresh)
    refresh_steps = int(sum(kinds))
    del scratch
    launches = refresh_steps * sess.launches_per_step(True) + (K - refresh_steps) * sess.launches_per_step(False)
    if world > 1:
        dist.barrier()

    # end to end: pinned host inputs in, every layer's output out, inside the timed region
    e2e, e_bytes = None, 0
    if E > 0:
        replay_range(A2)
        hq = [q_all[cur + s].cpu().pin_memory() for s in range(E)]
        hk = [k_all[cur + s].cpu().pin_memory() for s in range(E)]
        hv = [v_all[cur + s].cpu().pin_memory() for s in range(E)]
        hout = torch.empty(sess.out.shape, dtype=sess.out.dtype, pin_memory=True)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e_refresh = 0
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record()
        for s in range(E):
            e_bytes += wl.layers * layer_bytes(wl, sess.length + 1)
            e_refresh += int(sess.t % wl.refresh == 0)
            sess.stage(hq[s], hk[s], hv[s])
            sess.replay()
            hout.copy_(sess.out, non_blocking=True)
        a1.record()
        torch.cuda.synchronize()
        e_ms = a0.elapsed_time(a1)
        cur += E
        h2d = (hq[0].numel() * 2 + hk[0].numel() * 2 + hv[0].numel() * 2)
        d2h = hout.numel() * hout.element_size()
        e2e = {"value": e_bytes / (e_ms / 1e3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e_ms / E, "steps": E, "refresh_steps": e_refresh}

    # dominant kernel: the split-context attention kernel of reuse steps (with the fused append) and the
    # combine after it, isolated durations
    split_ms, comb_ms, cur = kernel_timing(sess, shape, n_top, wl, inputs, cur, T, stream)
    # kept-count statistics of the last step (layer 0), from one untimed call with index lists; it
    # rewrites that layer's output and threshold with the same values and leaves the caches alone
    kept = None
    try:
        cnt = torch.zeros((wl.batch, wl.h_q), dtype=torch.int32, device=dev)
        idx = torch.zeros((wl.batch, wl.h_q, l_cap), dtype=torch.int32, device=dev)
        saga.saga_decode_attn(shape, sess.q_buf[0], sess.k_cache[0], sess.v_cache[0], sess.length, n_top,
                              wl.refresh, sess.t - 1, sess.tau[0], sess.out[0], sess.workspace, sel_count=cnt,
                              sel_idx=idx)
        c = cnt.float().cpu()
        kept = {"layer": 0, "L": sess.length, "n_top": n_top, "min": int(c.min()), "mean": float(c.mean()),
                "max": int(c.max())}
        del idx
    except Exception as exc:  # noqa: BLE001  (reported, never fatal to the benchmark line)
        kept = {"error": str(exc)[:200]}
    status = saga.saga_get_status(sess.workspace)
    L_mid = sess.length

    # ---- gather over ranks (every rank takes part, whatever it measured)
    local = {"ms": ms, "bytes": bytes_timed, "e2e_ms": e2e["ms_per_step"] * E if e2e else 0.0,
             "e2e_bytes": e_bytes if e2e else 0.0}
    job = combine_rank_stats(gather_rank_stats(local, world), K)
    if rank != 0:
        return 0
    del sess, inputs, q_all, k_all, v_all
    torch.cuda.empty_cache()
    value = job["value"]
    ms_per_step = job["ms_per_step"]
    peak, peak_kind = load_peak()
    read = read_peak_probe(dev)
    roofline = None
    if split_ms and comb_ms and step_stats.get("reuse_mean_us"):
        # in-step time of the split kernel: the reuse step's time per layer, shared between the split kernel
        # and the combine in proportion to their isolated durations (in the step they overlap through
        # programmatic dependent launch, so the isolated durations add up to more than the step)
        s_mean, c_mean = statistics.mean(split_ms), statistics.mean(comb_ms)
        share = s_mean / (s_mean + c_mean)
        k_in_step = step_stats["reuse_mean_us"] / wl.layers * share
        nbytes = layer_bytes(wl, L_mid)
        achieved = nbytes / (k_in_step / 1e6) / 1e9
        roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                    "traffic": load_traffic(wl.name), "kernel": "saga_split_kernel (reuse step, per layer)",
                    "kernel_us_mean": k_in_step, "kernel_us_serialized": s_mean * 1e3,
                    "combine_us_serialized": c_mean * 1e3, "share_of_layer": share,
                    "achieved_serialized": nbytes / (s_mean / 1e3) / 1e9, "bytes_per_launch": nbytes,
                    "launches_timed": len(split_ms), "peak_kind": peak_kind,
                    "read_peak": read["gbs"], "frac_of_read_peak": achieved / read["gbs"]}
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms_per_step, "us_per_step": ms_per_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(wl, world),
        "window": {"l2": l2_note(flush, step_bytes, l2_bytes), "refresh_steps_timed": refresh_steps,
                   "alignment_steps": A},
        "step_us": step_stats,
        "frac_of_peak": value / peak,
        "kept": kept,
        "roofline": roofline,
        "read_probe": read,
        "e2e": ({"value": job["e2e_value"], "unit": "GB/s",
                 "h2d_bytes_per_step": e2e["h2d_bytes_per_step"] * world,
                 "d2h_bytes_per_step": e2e["d2h_bytes_per_step"] * world, "steps": e2e["steps"],
                 "refresh_steps": e2e["refresh_steps"]} if e2e else None),
        "gpu_launches": launches,
        "clocks": clocks,
        "status_word": status,
    }
    if world == 1 and not args.no_extra:
        extras = {}
        for name, layers in EXTRA_WORKLOADS:
            ewl = workload.by_name(name)
            if layers:
                ewl = ewl.with_(layers=layers)
            try:
                extras[name] = time_extra_workload(ewl, dev, 0, args, peak, l2_bytes)
            except Exception as exc:  # noqa: BLE001  (reported, never fatal to the benchmark line)
                extras[name] = {"error": str(exc)[:300]}
        line["workloads"] = extras
        batched = {}
        for name in LAYER_BATCHED_WORKLOADS:
            try:
                batched[name] = time_extra_workload(workload.by_name(name), dev, 0, args, peak, l2_bytes,
                                                    layer_batched=True)
            except Exception as exc:  # noqa: BLE001  (reported, never fatal to the benchmark line)
                batched[name] = {"error": str(exc)[:300]}
        line["layers_in_one_call"] = batched
        try:
            line["qkv_projection"] = time_qkv_projection(dev, peak)
        except Exception as exc:  # noqa: BLE001  (reported, never fatal to the benchmark line)
            line["qkv_projection"] = {"error": str(exc)[:300]}
        try:
            line["key_head_merge"] = time_key_head_merge(dev)
        except Exception as exc:  # noqa: BLE001  (reported, never fatal to the benchmark line)
            line["key_head_merge"] = {"error": str(exc)[:300]}
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(wl)
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=32)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="saga", choices=["saga", "reference"])
    ap.add_argument("--workload", default="qwen2.5-1.5b_saga_128k")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the extra workloads timed after the headline (the `workloads` object)")
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (profiling runs)")
    ap.add_argument("--only", default="", choices=["", "qkv", "merge"],
                    help="time only the QKV projection or the key-head merge and print their object (profiling runs)")
    ap.add_argument("--flush-l2", default="auto", choices=["auto", "on", "off"],
                    help="write 2 x L2 between timed steps (auto: when a step streams less than 2 x L2)")
    args = ap.parse_args()
    from long_context_decoding_saga_b200 import workload
    wl = workload.by_name(args.workload)
    if args.layers > 0:
        wl = wl.with_(layers=args.layers)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.only:
        import torch

        from long_context_decoding_saga_b200 import build, saga
        build.build()
        saga.load()
        dev = torch.device("cuda", 0)
        peak, _ = load_peak()
        if args.only == "qkv":
            print(json.dumps({"qkv_projection": time_qkv_projection(dev, peak)}), flush=True)
        else:
            print(json.dumps({"key_head_merge": time_key_head_merge(dev)}), flush=True)
        return 0
    if args.impl == "reference":
        return run_reference(args, wl, rank, world)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    try:
        return run_saga(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
