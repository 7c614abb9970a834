"""The seeded input recipe (CPU): shapes, dtypes and spreads as documented in
inputs.py, determinism per seed, random routing without replacement, the
skew bias, and a shared expert that leaves every other draw unchanged."""
import math

import torch

from mixture_experts_layer_39_b200.inputs import CONFIGS, custom_config, make_inputs


def test_shapes_and_dtypes():
    cfg = custom_config(300, 256, 128, 6, 2, random_routing=True, shared_ff=128)
    g = make_inputs(cfg, seed=1)
    T, d, f, E, k = cfg.T, cfg.d, cfg.f, cfg.E, cfg.k
    want = {"x": (T, d), "w_r": (E, d), "w_gu": (E, 2 * f, d), "w_d": (E, d, f), "dy": (T, d),
            "w_gu_s": (2 * 128, d), "w_d_s": (d, 128)}
    for name, shape in want.items():
        assert tuple(g[name].shape) == shape, name
        assert g[name].dtype == torch.bfloat16 and g[name].is_contiguous(), name
    assert g["route"].dtype == torch.int32 and tuple(g["route"].shape) == (T, k)
    assert g["bias"] is None


def test_spreads_match_the_recipe():
    cfg = custom_config(4096, 512, 256, 8, 4)
    g = make_inputs(cfg, seed=2)
    for name, std in (("x", 1.0), ("dy", 1.0), ("w_r", 1 / math.sqrt(512)),
                      ("w_gu", 1 / math.sqrt(512)), ("w_d", 1 / math.sqrt(512))):
        v = g[name].double()
        n = v.numel()
        assert abs(v.mean().item()) < 5 * std / math.sqrt(n), name       # 5 standard errors
        assert abs(v.std().item() / std - 1.0) < 5 / math.sqrt(2 * n) + 2e-3, name
        assert v.unique().numel() > 1000, name  # never constant: timing depends on values


def test_same_seed_same_draws_other_seed_differs():
    cfg = CONFIGS["tiny"]
    a, b, c = make_inputs(cfg, seed=5), make_inputs(cfg, seed=5), make_inputs(cfg, seed=6)
    for name in ("x", "w_r", "w_gu", "w_d", "dy"):
        assert torch.equal(a[name], b[name]), name
        assert not torch.equal(a[name], c[name]), name


def test_random_routing_without_replacement():
    cfg = custom_config(20000, 128, 128, 16, 4, random_routing=True)
    r = make_inputs(cfg, seed=3)["route"].long()
    assert r.min().item() >= 0 and r.max().item() < cfg.E
    srt = r.sort(dim=1).values
    assert bool((srt[:, 1:] != srt[:, :-1]).all())           # k distinct experts per token
    counts = torch.bincount(r.reshape(-1), minlength=cfg.E).double()
    expect = cfg.T * cfg.k / cfg.E
    assert float(((counts - expect).abs() / expect).max()) < 0.05  # uniform over experts


def test_skew_bias():
    cfg = custom_config(64, 128, 128, 5, 2, skew_bias=True)
    b = make_inputs(cfg, seed=0)["bias"]
    assert b.dtype == torch.float32
    want = torch.tensor([2.0 * math.log(1.0 / (e + 1)) for e in range(5)], dtype=torch.float32)
    assert torch.allclose(b, want)


def test_shared_expert_drawn_last():
    base = custom_config(256, 128, 128, 4, 2)
    shared = custom_config(256, 128, 128, 4, 2, shared_ff=256)
    a, b = make_inputs(base, seed=9), make_inputs(shared, seed=9)
    for name in ("x", "w_r", "w_gu", "w_d", "dy"):
        assert torch.equal(a[name], b[name]), name
    assert "w_gu_s" not in a and "w_gu_s" in b
