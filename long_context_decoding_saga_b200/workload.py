"""Seeded synthetic decode workloads for the SAGA + Atop-N decode step.

This module only draws inputs: the initial K/V caches of each layer, the
query of every decode step and the key/value row that each step appends.  It
holds none of the attention arithmetic (no scores, no threshold, no softmax),
so the CUDA path and the CPU oracle can both be fed from it without sharing
any of the method's code.

The paper ("More Value per Key: Asymmetric Sparse Attention for Faster LLM
Decoding") measures end-to-end decoding on Llama-3.2-1B and Qwen2.5-1.5B at up
to 128K tokens (Fig. 2 table) and gives no inputs of its own, so the caches
here are model-shaped random tensors:

* K and V rows are bf16 draws from N(0, 1).
* "planted" workloads mark a fixed fraction of the cached positions of every
  (layer, batch, key head) as query-correlated: such a key is
  0.7 * u + 0.3 * z with u ~ N(0, I) drawn once per (layer, batch, key head)
  and z ~ N(0, I) per row.  Each query head j draws 16 of the planted
  positions of its own key head once, and its query at step t is
  0.7 * mean(those 16 keys) + 0.3 * eps_t with fresh eps_t ~ N(0, I).  An
  appended key is planted with the same probability.  Scores are therefore
  heavy-tailed and drift a little from step to step, which is the regime
  the Atop-N threshold reuse relies on (Atop-N, step 2).
* the tiny workload draws the 16 indices from all cached positions, with no
  planted cluster.
* the dense GQA workload draws q from N(0, 1) as well.

The query head j is tied to key head floor(j * h_k / h_q) when queries are
built from keys; that is the contiguous grouping the attention step uses.

Every draw goes through a torch.Generator seeded from (workload seed, layer),
on the device the caller names; the same seed on the same device type gives
the same bytes.
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Dict, Optional

import torch

DENSE = -1  # n_top sentinel: "keep every cached token" (no threshold)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic decode workload.

    n_top == DENSE means the N of the Atop-N rule covers the whole context,
    so no threshold ever applies; callers pass N = l_cap to the kernels.
    """

    name: str
    batch: int
    h_q: int
    h_k: int
    h_v: int
    d: int
    l_kv: int
    layers: int
    steps: int
    n_top: int
    refresh: int
    planted: float
    q_mode: str  # "cached_mean" | "planted_mean" | "gaussian"
    seed: int

    @property
    def dense(self) -> bool:
        return self.n_top == DENSE

    def l_cap(self, extra_steps: int = 0) -> int:
        """Cache capacity: the prefilled tokens plus one per decode step."""
        return self.l_kv + self.steps + extra_steps

    def n_for_kernel(self, l_cap: int) -> int:
        return l_cap if self.dense else self.n_top

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five synthetic configurations (tiny, Llama-SAGA 32K, Qwen-SAGA 128K,
# dense GQA 128K, and the Llama-shaped sweep).
TINY = Workload("tiny_1k", 1, 8, 1, 8, 64, 1024, 1, 32, 64, 8, 0.0, "cached_mean", 1001)
LLAMA_SAGA_32K = Workload("llama3.2-1b_saga_32k", 1, 32, 2, 8, 64, 32768, 16, 64, 256, 16, 0.01,
                          "planted_mean", 1002)
QWEN_SAGA_128K = Workload("qwen2.5-1.5b_saga_128k", 1, 12, 1, 4, 128, 131072, 28, 32, 512, 32, 0.005,
                          "planted_mean", 1003)
DENSE_GQA_128K = Workload("llama3.2-1b_dense_gqa_128k", 1, 32, 8, 8, 64, 131072, 16, 32, DENSE, 1 << 30,
                          0.0, "gaussian", 1004)

CONFIGS = {w.name: w for w in (TINY, LLAMA_SAGA_32K, QWEN_SAGA_128K, DENSE_GQA_128K)}

SWEEP_L_KV = (4096, 16384, 65536, 131072)
SWEEP_BATCH = (1, 4, 16)
SWEEP_H_K = (1, 2, 4, 8)
SWEEP_N = (64, 256, 1024)
SWEEP_R = (1, 16, 64)


def sweep_point(l_kv: int, batch: int, h_k: int, n_top: int, refresh: int) -> Workload:
    """A point of the Llama-3.2-1B-shaped sweep (h_q=32, d=64, h_v=8, 16 layers)."""
    key = f"sweep:{l_kv}:{batch}:{h_k}:{n_top}:{refresh}".encode()
    seed = int.from_bytes(hashlib.sha256(key).digest()[:4], "little")
    return Workload(f"sweep_l{l_kv}_b{batch}_hk{h_k}_n{n_top}_r{refresh}", batch, 32, h_k, 8, 64, l_kv, 16,
                    max(2 * refresh, 16), n_top, refresh, 0.01, "planted_mean", seed)


def by_name(name: str) -> Workload:
    """A configuration by name, or a sweep point by its name
    (sweep_l<l_kv>_b<batch>_hk<h_k>_n<N>_r<R>)."""
    if name in CONFIGS:
        return CONFIGS[name]
    import re
    m = re.fullmatch(r"sweep_l(\d+)_b(\d+)_hk(\d+)_n(\d+)_r(\d+)", name)
    if m is None:
        raise KeyError(f"unknown workload {name!r}")
    return sweep_point(*(int(x) for x in m.groups()))


def sweep_points():
    for l_kv in SWEEP_L_KV:
        for b in SWEEP_BATCH:
            for h_k in SWEEP_H_K:
                for n in SWEEP_N:
                    for r in SWEEP_R:
                        yield sweep_point(l_kv, b, h_k, n, r)


def _layer_seed(seed: int, layer: int, salt: int = 0) -> int:
    h = hashlib.sha256(f"{seed}:{layer}:{salt}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _randn(g: torch.Generator, shape, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def make_layer(wl: Workload, layer: int, device="cpu", steps: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Draw one layer's inputs.

    Returns bf16 tensors on `device`:
      K0    [B, h_k, l_kv, d]   initial key cache
      V0    [B, h_v, l_kv, d]   initial value cache
      q     [S, B, h_q, d]      query of decode step t = 0..S-1
      k_new [S, B, h_k, d]      key appended at step t
      v_new [S, B, h_v, d]      value appended at step t
    """
    device = torch.device(device)
    S = wl.steps if steps is None else steps
    B, hq, hk, hv, d, l = wl.batch, wl.h_q, wl.h_k, wl.h_v, wl.d, wl.l_kv
    g = torch.Generator(device=device)
    g.manual_seed(_layer_seed(wl.seed, layer))

    K = _randn(g, (B, hk, l, d), device)
    V = _randn(g, (B, hv, l, d), device).to(torch.bfloat16)
    k_new = _randn(g, (S, B, hk, d), device)
    v_new = _randn(g, (S, B, hv, d), device).to(torch.bfloat16)
    eps = _randn(g, (S, B, hq, d), device)
    group = torch.arange(hq, device=device) * hk // hq  # key head that query head j is built from

    if wl.q_mode == "gaussian":
        q = eps
    elif wl.q_mode == "cached_mean":
        idx = torch.randint(0, l, (B, hq, 16), generator=g, device=device)
        Kb = K.to(torch.bfloat16).float()
        src = Kb[torch.arange(B, device=device)[:, None, None], group[None, :, None], idx]  # [B,hq,16,d]
        q = 0.7 * src.mean(dim=2)[None] + 0.3 * eps
    elif wl.q_mode == "planted_mean":
        n_pl = max(16, int(round(wl.planted * l)))
        u = _randn(g, (B, hk, 1, d), device)
        # planted positions: a fixed-size random subset per (b, key head)
        keys = torch.rand((B, hk, l), generator=g, device=device)
        pos = keys.topk(n_pl, dim=-1).indices  # [B,hk,n_pl]
        planted_rows = 0.7 * u + 0.3 * torch.gather(K, 2, pos[..., None].expand(-1, -1, -1, d))
        K.scatter_(2, pos[..., None].expand(-1, -1, -1, d), planted_rows)
        # appended keys are planted with the same probability
        coin = torch.rand((S, B, hk, 1), generator=g, device=device) < wl.planted
        k_new = torch.where(coin, 0.7 * u.squeeze(2)[None] + 0.3 * k_new, k_new)
        # each query head averages 16 of its key head's planted keys
        pick = torch.rand((B, hq, n_pl), generator=g, device=device).topk(16, dim=-1).indices
        rows = torch.gather(pos[:, group, :], 2, pick)  # [B,hq,16] token positions
        Kb = K.to(torch.bfloat16).float()
        src = Kb[torch.arange(B, device=device)[:, None, None], group[None, :, None], rows]
        q = 0.7 * src.mean(dim=2)[None] + 0.3 * eps
    else:
        raise ValueError(f"unknown q_mode {wl.q_mode!r}")

    return {
        "K0": K.to(torch.bfloat16).contiguous(),
        "V0": V.contiguous(),
        "q": q.to(torch.bfloat16).contiguous(),
        "k_new": k_new.to(torch.bfloat16).contiguous(),
        "v_new": v_new.contiguous(),
    }


def alloc_caches(wl: Workload, l_cap: int, layer_inputs: Dict[str, torch.Tensor], device) -> Dict[str, torch.Tensor]:
    """Caches of capacity l_cap holding the l_kv prefilled rows (rest zero)."""
    B, hk, hv, d, l = wl.batch, wl.h_k, wl.h_v, wl.d, wl.l_kv
    kc = torch.zeros((B, hk, l_cap, d), dtype=torch.bfloat16, device=device)
    vc = torch.zeros((B, hv, l_cap, d), dtype=torch.bfloat16, device=device)
    kc[:, :, :l].copy_(layer_inputs["K0"])
    vc[:, :, :l].copy_(layer_inputs["V0"])
    return {"k_cache": kc, "v_cache": vc}
