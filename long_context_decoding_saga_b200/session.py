"""Multi-layer decode session over libsaga.

Holds one K and one V cache per layer (K and V stored separately, each with
its own head count), the per-layer Atop-N thresholds, a workspace shared by
the layers (their calls are sequential on one stream) and the output of every
layer.  A decode step is, for every layer, one saga_decode_step call: the
new token's key/value rows are appended by the attention kernels, then the
attention step runs (refresh on t % R == 0).

`capture()` records one decode step of all layers into two CUDA graphs (a
refresh step and a reuse step).  The graphs read the sequence length from a
device int (the length argument the C ABI takes for graph replays) that a
one-element add at the start of each replay advances; inputs are staged into
static buffers before each replay.

With `layer_batched=True` the layers' caches, thresholds, inputs and outputs
are slices of layer-major buffers, and a step is ONE saga_decode_step call
with batch = layers x B: every (layer, batch) row is an independent row of
the batched call, so the results are those of the per-layer calls, and the
step pays one kernel hand-off chain instead of one per layer.  This needs
every layer's query of the step at once, as this session's step() takes
them; a model whose next layer's query depends on this layer's output calls
the layers one by one.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import saga


class DecodeSession:
    def __init__(self, shape: saga.SagaShape, layers: int, n_top: int, refresh: int, device="cuda",
                 out_dtype=torch.float32, track_selection: bool = False, layer_batched: bool = False):
        self.shape = shape
        self.layers = layers
        self.n_top = n_top
        self.refresh = refresh
        self.device = torch.device(device)
        self.layer_batched = layer_batched
        B, hq, hk, hv, d, lc = shape.astuple()
        bf = torch.bfloat16
        if layer_batched:
            self.batched_shape = saga.SagaShape.of(layers * B, hq, hk, hv, d, lc)
            self.k_all = torch.zeros((layers, B, hk, lc, d), dtype=bf, device=device)
            self.v_all = torch.zeros((layers, B, hv, lc, d), dtype=bf, device=device)
            self.k_cache = [self.k_all[i] for i in range(layers)]
            self.v_cache = [self.v_all[i] for i in range(layers)]
        else:
            self.k_cache = [torch.zeros((B, hk, lc, d), dtype=bf, device=device) for _ in range(layers)]
            self.v_cache = [torch.zeros((B, hv, lc, d), dtype=bf, device=device) for _ in range(layers)]
        self.tau = torch.zeros((layers, B, hq), dtype=torch.float32, device=device)
        self.out = torch.zeros((layers, B, hq, d), dtype=out_dtype, device=device)
        self.workspace = saga.alloc_workspace(self.batched_shape if layer_batched else shape, device)
        self.sel_count = self.sel_idx = None
        if track_selection:
            self.sel_count = torch.zeros((layers, B, hq), dtype=torch.int32, device=device)
            self.sel_idx = torch.zeros((layers, B, hq, lc), dtype=torch.int32, device=device)
        self.length = 0  # tokens in the caches
        self.t = 0       # next decode step
        # graph state
        self.seq_len_dev = torch.zeros(1, dtype=torch.int32, device=device)
        self.q_buf = torch.zeros((layers, B, hq, d), dtype=bf, device=device)
        self.k_buf = torch.zeros((layers, B, hk, d), dtype=bf, device=device)
        self.v_buf = torch.zeros((layers, B, hv, d), dtype=bf, device=device)
        self.graphs = {}

    def prefill(self, layer: int, K0: torch.Tensor, V0: torch.Tensor):
        """Copy a layer's prefilled rows (bf16 [B, h_k, l, d], [B, h_v, l, d]) into its caches."""
        l = K0.shape[2]
        self.k_cache[layer][:, :, :l].copy_(K0)
        self.v_cache[layer][:, :, :l].copy_(V0)
        self.length = l

    def _layer_step(self, i, q, k_new, v_new, seq_len, step, seq_len_dev=None):
        saga.saga_decode_step(self.shape, q, k_new, v_new, self.k_cache[i], self.v_cache[i], seq_len, self.n_top,
                              self.refresh, step, self.tau[i], self.out[i], self.workspace,
                              sel_count=None if self.sel_count is None else self.sel_count[i],
                              sel_idx=None if self.sel_idx is None else self.sel_idx[i], seq_len_dev=seq_len_dev)

    def _all_layers_step(self, q, k_new, v_new, seq_len, step, seq_len_dev=None):
        """Every layer in one call: the layer-major buffers viewed as a batch of layers x B."""
        B, hq, hk, hv, d, lc = self.shape.astuple()
        LB = self.layers * B
        saga.saga_decode_step(self.batched_shape, q.reshape(LB, hq, d), k_new.reshape(LB, hk, d),
                              v_new.reshape(LB, hv, d), self.k_all.view(LB, hk, lc, d),
                              self.v_all.view(LB, hv, lc, d), seq_len, self.n_top, self.refresh, step,
                              self.tau.view(LB, hq), self.out.view(LB, hq, d), self.workspace,
                              sel_count=None if self.sel_count is None else self.sel_count.view(LB, hq),
                              sel_idx=None if self.sel_idx is None else self.sel_idx.view(LB, hq, lc),
                              seq_len_dev=seq_len_dev)

    def step(self, q, k_new, v_new):
        """One decode step of every layer with host-side lengths (q: [layers, B, h_q, d], ...)."""
        if self.length >= self.shape.l_cap:
            raise RuntimeError("cache capacity exhausted")
        L = self.length + 1
        if self.layer_batched:
            self._all_layers_step(q.contiguous(), k_new.contiguous(), v_new.contiguous(), L, self.t)
        else:
            for i in range(self.layers):
                self._layer_step(i, q[i], k_new[i], v_new[i], L, self.t)
        self.length = L
        self.t += 1
        return self.out

    # ------------------------------------------------------------------ CUDA graphs
    def capture(self, stream: Optional[torch.cuda.Stream] = None):
        """Record a refresh step and a reuse step of all layers as CUDA graphs."""
        L_est = min(self.shape.l_cap, self.length + 1)
        stream = stream or torch.cuda.Stream(self.device)
        for kind, step in (("refresh", 0), ("reuse", 1 if self.refresh > 1 else 0)):
            g = torch.cuda.CUDAGraph()
            # warm the launch-attribute caches outside capture
            torch.cuda.synchronize(self.device)
            with torch.cuda.graph(g, stream=stream):
                self.seq_len_dev.add_(1)
                if self.layer_batched:
                    self._all_layers_step(self.q_buf, self.k_buf, self.v_buf, L_est, step,
                                          seq_len_dev=self.seq_len_dev)
                else:
                    for i in range(self.layers):
                        self._layer_step(i, self.q_buf[i], self.k_buf[i], self.v_buf[i], L_est, step,
                                         seq_len_dev=self.seq_len_dev)
            self.graphs[kind] = g
        self.seq_len_dev.fill_(self.length)
        torch.cuda.synchronize(self.device)

    def stage(self, q, k_new, v_new, non_blocking=True):
        self.q_buf.copy_(q, non_blocking=non_blocking)
        self.k_buf.copy_(k_new, non_blocking=non_blocking)
        self.v_buf.copy_(v_new, non_blocking=non_blocking)

    def replay(self):
        """One decode step of all layers from the staged inputs."""
        if self.length >= self.shape.l_cap:
            raise RuntimeError("cache capacity exhausted")
        kind = "refresh" if self.t % self.refresh == 0 else "reuse"
        self.graphs[kind].replay()
        self.length += 1
        self.t += 1
        return self.out

    def launches_per_step(self, refresh_step: bool) -> int:
        """Kernels of this library launched per decode step (the append is fused into the first of them)."""
        dense = self.n_top >= self.shape.l_cap
        if refresh_step and not dense:
            per_layer = 4  # score dump (+append), radix select, from-scores, combine
        elif refresh_step and dense:
            per_layer = 3  # threshold fill, split (+append), combine
        else:
            per_layer = 2  # split (+append), combine
        return per_layer if self.layer_batched else self.layers * per_layer
