"""The seeded input generator follows its stated recipe (CPU): reproducible
per-layer streams, the cube-prototype structure of the hidden states, the
near-duplicate cubes of the stacked workload, the weight scale, the one-time
rounding to the working dtype and the dense FLOP counts."""
import dataclasses

import numpy as np
import torch

import workloads


def _cfg(**kw):
    # 16 cubes of 32 tokens (8 x 8 x 8 grid, 4 x 4 x 2 cubes) and 64 text tokens
    base = dict(grid=(8, 8, 8), cube=(4, 4, 2), n_text=64, D=512, hq=4, hkv=2, d=64, F=256)
    base.update(kw)
    return workloads.small_config(**base)


def _cube_stats(cfg, x):
    off = cfg.offsets
    means = np.stack([x[off[c]:off[c + 1]].mean(0) for c in range(cfg.n_cubes)])
    var = np.array([x[off[c]:off[c + 1]].var(0).mean() for c in range(cfg.n_cubes)])
    return means, var


def test_streams_are_reproducible_and_distinct():
    cfg = _cfg()
    a = workloads.make_hidden(cfg, workloads.layer_rng(cfg))
    assert np.array_equal(a, workloads.make_hidden(cfg, workloads.layer_rng(cfg)))
    other_seed = dataclasses.replace(cfg, seed=cfg.seed + 1)
    assert not np.array_equal(a, workloads.make_hidden(other_seed, workloads.layer_rng(other_seed)))
    # every layer of a stack draws from its own stream
    assert not np.array_equal(a, workloads.make_hidden(cfg, workloads.layer_rng(cfg, 1)))


def test_hidden_states_are_cube_prototypes_plus_noise():
    cfg = _cfg(sigma=0.3, sigma_range=None)
    x = workloads.make_hidden(cfg, workloads.layer_rng(cfg))
    assert x.shape == (cfg.n_tokens, cfg.D) and x.dtype == np.float32
    n = cfg.n_c
    means, var = _cube_stats(cfg, x)
    # spread inside a cube: sigma^2 (n - 1) / n around the cube's own mean
    assert np.abs(var - 0.09 * (n - 1) / n).max() < 0.01
    # cube means: N(0, 1) prototypes plus noise of variance sigma^2 / n
    assert abs(means.var() - (1.0 + 0.09 / n)) < 0.05
    # text rows: N(0, 1)
    t = x[cfg.n_vis:]
    assert abs(t.mean()) < 0.02 and abs(t.var() - 1.0) < 0.03


def test_per_cube_noise_scale_range():
    cfg = _cfg()                       # sigma_c ~ U(0.1, 1.0) per cube
    x = workloads.make_hidden(cfg, workloads.layer_rng(cfg))
    n = cfg.n_c
    _, var = _cube_stats(cfg, x)
    sig = np.sqrt(var * n / (n - 1))
    assert sig.min() > 0.1 * 0.95 and sig.max() < 1.0 * 1.05
    assert sig.max() / sig.min() > 3.0  # the scales really differ from cube to cube


def test_near_duplicate_cubes():
    cfg = _cfg(structure="near_dup", sigma=None, sigma_range=None)
    x = workloads.make_hidden(cfg, workloads.layer_rng(cfg))
    n, C = cfg.n_c, cfg.n_cubes
    means, var = _cube_stats(cfg, x)
    sig = np.sqrt(var * n / (n - 1))
    dup = []
    for c in range(1, C):
        # a copied prototype leaves the two cube means about 0.3 apart (noise
        # only); fresh prototypes are about sqrt(2 D) = 32 apart
        dist = np.sqrt(((means[:c] - means[c]) ** 2).sum(1)).min()
        dup.append(dist < 3.0)
        assert dist < 3.0 or dist > 20.0
        assert abs(sig[c] - (0.05 if dup[-1] else 0.5)) < 0.01
    assert sum(dup) == (C - 1) // 2
    assert abs(sig[0] - 0.5) < 0.01    # the first cube always takes a fresh prototype


def test_weight_scale():
    cfg = _cfg()
    rng = workloads.layer_rng(cfg)
    workloads.make_hidden(cfg, rng)
    w = workloads.make_weights(cfg, rng, with_o=True)
    shapes = {"W_q": (cfg.D, cfg.hq * cfg.d), "W_k": (cfg.D, cfg.hkv * cfg.d),
              "W_v": (cfg.D, cfg.hkv * cfg.d), "W_gate": (cfg.F, cfg.D), "W_up": (cfg.F, cfg.D),
              "W_down": (cfg.D, cfg.F), "W_o": (cfg.hq * cfg.d, cfg.D)}
    for k, shp in shapes.items():
        assert w[k].shape == shp
        assert abs(w[k].std() - 0.02) < 0.02 * 0.03, k
        assert abs(w[k].mean()) < 0.02 * 0.03, k


def test_rounded_once_and_projected():
    cfg = _cfg()
    lay = workloads.make_layer(cfg)
    for k in ("x", "W_gate", "W_up", "W_down", "Q", "K", "V"):
        assert lay[k].dtype == torch.bfloat16, k
    x = lay["x"].float()
    for name, W, h in (("Q", lay["W_q"], cfg.hq), ("K", lay["W_k"], cfg.hkv),
                       ("V", lay["W_v"], cfg.hkv)):
        ref = (x @ W.float()).to(torch.bfloat16).view(cfg.n_tokens, h, cfg.d)
        got = lay[name]
        assert got.shape == (cfg.n_tokens, h, cfg.d)
        # the same fp32 product rounded once; summation order may move a value
        # across a rounding boundary, by one bf16 step at most
        diff = (got.float() - ref.float()).abs()
        step = ref.float().abs().clamp_min(1e-30) * 2.0 ** -7
        assert (diff <= step).all(), name
    fp = workloads.make_layer(_cfg(dtype="fp32"))
    assert fp["x"].dtype == torch.float32 and fp["Q"].dtype == torch.float32


def test_upstream_gradients_have_their_own_stream():
    cfg = _cfg()
    up = workloads.make_upstream(cfg)
    assert up["dO"].shape == (cfg.n_tokens, cfg.hq, cfg.d) and up["dO"].dtype == torch.bfloat16
    assert up["dy"].shape == (cfg.n_tokens, cfg.D) and up["dy"].dtype == torch.float32
    again = workloads.make_upstream(cfg)
    assert torch.equal(up["dO"], again["dO"]) and torch.equal(up["dy"], again["dy"])
    x = workloads.make_hidden(cfg, workloads.layer_rng(cfg))
    assert not np.allclose(up["dy"].numpy()[:4], x[:4])
    assert abs(up["dy"].std().item() - 1.0) < 0.02


def test_dense_flop_counts_of_the_64k_layer():
    f = workloads.dense_flops(workloads.CONFIGS[3])
    # causal attention 4 d hq N (N + 1) / 2 and three D x F GEMMs, 2 flops each
    assert abs(f["attn"] / 1e12 - 31.03) < 0.01
    assert abs(f["ffn"] / 1e12 - 26.80) < 0.01
