"""The seeded input generator (CPU): determinism, shapes, the planted
structure of the configurations, and workload lookup by name."""
import pytest
import torch

from long_context_decoding_saga_b200 import workload as W


def test_same_seed_same_bytes_and_layers_differ():
    wl = W.TINY.with_(l_kv=300, steps=3)
    a = W.make_layer(wl, 0, steps=3)
    b = W.make_layer(wl, 0, steps=3)
    c = W.make_layer(wl, 1, steps=3)
    for k in a:
        assert torch.equal(a[k], b[k])
    assert not torch.equal(a["K0"], c["K0"])


def test_shapes_and_dtypes():
    wl = W.Workload("t", 2, 12, 1, 4, 128, 257, 1, 5, 16, 2, 0.05, "planted_mean", 3)
    x = W.make_layer(wl, 0)
    assert x["K0"].shape == (2, 1, 257, 128) and x["V0"].shape == (2, 4, 257, 128)
    assert x["q"].shape == (5, 2, 12, 128) and x["k_new"].shape == (5, 2, 1, 128) and x["v_new"].shape == (5, 2, 4, 128)
    assert all(v.dtype == torch.bfloat16 for v in x.values())


def test_planted_keys_cluster_around_their_key_head_direction():
    # 5% of 2000 positions planted as 0.7 u + 0.3 z: their mean is close to 0.7 u, the rest average to ~0
    wl = W.Workload("p", 1, 4, 2, 4, 64, 2000, 1, 2, 16, 2, 0.05, "planted_mean", 9)
    K = W.make_layer(wl, 0)["K0"].float()
    for h in range(2):
        norms = K[0, h].norm(dim=-1)
        proj = K[0, h] @ K[0, h].mean(0)
        top = proj.topk(100).indices  # planted rows dominate the mean direction
        assert norms[top].mean() < norms.mean() + 1.0
        assert (proj[top] > proj.median()).all()


def test_sweep_has_every_point_and_names_round_trip():
    pts = list(W.sweep_points())
    assert len(pts) == 4 * 3 * 4 * 3 * 3
    assert len({p.name for p in pts}) == len(pts)
    for p in pts[::37]:
        assert W.by_name(p.name) == p
    assert W.by_name("qwen2.5-1.5b_saga_128k") is W.QWEN_SAGA_128K
    with pytest.raises(KeyError):
        W.by_name("nope")
