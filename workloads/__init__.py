"""Seeded synthetic inputs for the AdaSpark layer (shared by the tests, the bench
and the smoke check).

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no partition, no scores, no selection, no FFN).  Tokens are
produced directly in cube-major order: cube c owns rows
[offsets[c], offsets[c+1]) of the visual prefix, and the text rows follow.

Recipe (one ``numpy.random.Generator(PCG64(seed))`` per layer, draws in this
fixed order, all normal draws in float32):

1. cube prototypes  [C, D] ~ N(0, 1)
2. per-cube sigma_c: a constant (``sigma``) or U(sigma_lo, sigma_hi)
3. token noise      [N_v, D] ~ N(0, 1); x_t = proto_c + sigma_c * noise_t
4. text tokens      [N_t, D] ~ N(0, 1)
5. W_q [D, hq*d], W_k [D, hkv*d], W_v [D, hkv*d] ~ N(0, 0.02^2)
6. W_gate [F, D], W_up [F, D], W_down [D, F] ~ N(0, 0.02^2)
7. (stacked layers only) W_o [hq*d, D] ~ N(0, 0.02^2)

The "near-duplicate" structure of the 4-layer 262K-token stack replaces steps
1-3 for its first layer: a seeded half of the cubes 1..C-1 copy the prototype
of a uniformly drawn earlier cube with noise 0.05, the rest take a fresh
prototype with noise 0.5.

Every tensor is rounded once to the working dtype (bf16 round-to-nearest-even
via torch, or kept fp32), and those exact values are what both the CUDA path
and the oracle read.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np

BASE_SEED = 20260408


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    """Sizes of one AdaSpark layer workload.

    ``grid`` is (T, H, W) of the video token grid, ``cube`` is (h, w, t) of a
    cube.  ``cube_sizes`` overrides the uniform cube size (used for truncated
    edge cubes in tests); when None all cubes hold h*w*t tokens and the grid
    must divide evenly.
    """
    name: str
    grid: tuple          # (T, H, W)
    cube: tuple          # (h, w, t)
    n_text: int
    D: int
    hq: int
    hkv: int
    d: int
    F: int
    dtype: str           # "bf16" or "fp32"
    p: float = 0.7
    sigma: Optional[float] = 0.3           # constant noise scale, or None
    sigma_range: Optional[tuple] = None    # (lo, hi) for U(lo, hi) per cube
    structure: str = "proto"               # "proto" or "near_dup"
    n_layers: int = 1
    seed: int = BASE_SEED
    cube_sizes: Optional[tuple] = None

    @property
    def n_vis(self) -> int:
        T, H, W = self.grid
        return T * H * W

    @property
    def n_tokens(self) -> int:
        return self.n_vis + self.n_text

    @property
    def n_c(self) -> int:
        h, w, t = self.cube
        return h * w * t

    @property
    def sizes(self) -> np.ndarray:
        if self.cube_sizes is not None:
            s = np.asarray(self.cube_sizes, dtype=np.int64)
            assert int(s.sum()) == self.n_vis
            return s
        T, H, W = self.grid
        h, w, t = self.cube
        assert T % t == 0 and H % h == 0 and W % w == 0, "grid must divide evenly"
        C = (T // t) * (H // h) * (W // w)
        return np.full(C, self.n_c, dtype=np.int64)

    @property
    def n_cubes(self) -> int:
        return int(self.sizes.shape[0])

    @property
    def offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.sizes)]).astype(np.int32)


def _cfg(i, **kw):
    return LayerConfig(seed=BASE_SEED + i, **kw)


# The five workloads: Qwen2.5-VL-3B / 7B layer shapes (heads, head size, hidden and FFN
# widths) on video-token grids of 18K to 256K tokens, plus a tiny fp32 case.
CONFIGS = {
    1: _cfg(1, name="tiny-fp32", grid=(8, 8, 8), cube=(4, 4, 2), n_text=32, D=256,
            hq=4, hkv=1, d=64, F=512, dtype="fp32", sigma=0.3),
    2: _cfg(2, name="qwen2.5-vl-3b-18k", grid=(32, 24, 24), cube=(4, 4, 4), n_text=128,
            D=2048, hq=16, hkv=2, d=128, F=11008, dtype="bf16", sigma=0.3),
    3: _cfg(3, name="qwen2.5-vl-7b-64k", grid=(64, 32, 32), cube=(4, 4, 4), n_text=256,
            D=3584, hq=28, hkv=4, d=128, F=18944, dtype="bf16", sigma=None,
            sigma_range=(0.1, 1.0)),
    4: _cfg(4, name="qwen2.5-vl-7b-128k", grid=(128, 32, 32), cube=(4, 4, 4), n_text=256,
            D=3584, hq=28, hkv=4, d=128, F=18944, dtype="bf16", sigma=None,
            sigma_range=(0.1, 1.0)),
    5: _cfg(5, name="qwen2.5-vl-7b-256k-x4", grid=(256, 32, 32), cube=(4, 4, 4), n_text=512,
            D=3584, hq=28, hkv=4, d=128, F=18944, dtype="bf16", sigma=None,
            structure="near_dup", n_layers=4),
}

# The sweep of the 128K workload: p values x cube shapes. The inputs depend on
# the cube shape only (seed + 100 * shape index), so the p sweep reuses them.
SWEEP_4 = [(p, cube) for cube in ((4, 4, 4), (8, 8, 2)) for p in (0.5, 0.7, 0.9, 1.0)]


def sweep_config(idx: int) -> LayerConfig:
    p, cube = SWEEP_4[idx]
    shape = 0 if cube == (4, 4, 4) else 1
    return dataclasses.replace(CONFIGS[4], p=p, cube=cube, seed=BASE_SEED + 4 + 100 * shape,
                               name=f"qwen2.5-vl-7b-128k-p{p}-{cube[0]}x{cube[1]}x{cube[2]}")


def _round(a: np.ndarray, dtype: str):
    """Round a float32 array to the working dtype; returns a torch CPU tensor."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    return t.clone()


def _normal(rng, shape, scale=1.0):
    a = rng.standard_normal(shape, dtype=np.float32)
    if scale != 1.0:
        a *= np.float32(scale)
    return a


def make_hidden(cfg: LayerConfig, rng) -> np.ndarray:
    """Steps 1-4: the layer input x [N, D] (float32, not yet rounded)."""
    sizes = cfg.sizes
    C, D = cfg.n_cubes, cfg.D
    x = np.empty((cfg.n_tokens, D), dtype=np.float32)
    if cfg.structure == "near_dup":
        fresh = _normal(rng, (C, D))
        proto = fresh.copy()
        dup = np.zeros(C, dtype=bool)
        if C > 1:
            chosen = rng.permutation(C - 1)[: (C - 1) // 2] + 1
            dup[chosen] = True
        for c in range(1, C):
            if dup[c]:
                proto[c] = proto[int(rng.integers(0, c))]
        sig = np.where(dup, 0.05, 0.5).astype(np.float32)
    else:
        proto = _normal(rng, (C, D))
        if cfg.sigma_range is not None:
            lo, hi = cfg.sigma_range
            sig = rng.uniform(lo, hi, C).astype(np.float32)
        else:
            sig = np.full(C, cfg.sigma, dtype=np.float32)
    row = 0
    for c in range(C):
        n = int(sizes[c])
        noise = _normal(rng, (n, D))
        x[row:row + n] = proto[c][None, :] + sig[c] * noise
        row += n
    x[cfg.n_vis:] = _normal(rng, (cfg.n_text, D))
    return x


def make_weights(cfg: LayerConfig, rng, with_o: bool = False) -> dict:
    """Steps 5-7: projection and FFN weights (float32, not yet rounded)."""
    D, F, hq, hkv, d = cfg.D, cfg.F, cfg.hq, cfg.hkv, cfg.d
    w = {}
    w["W_q"] = _normal(rng, (D, hq * d), 0.02)
    w["W_k"] = _normal(rng, (D, hkv * d), 0.02)
    w["W_v"] = _normal(rng, (D, hkv * d), 0.02)
    w["W_gate"] = _normal(rng, (F, D), 0.02)
    w["W_up"] = _normal(rng, (F, D), 0.02)
    w["W_down"] = _normal(rng, (D, F), 0.02)
    if with_o:
        w["W_o"] = _normal(rng, (hq * d, D), 0.02)
    return w


def layer_rng(cfg: LayerConfig, layer: int = 0):
    return np.random.Generator(np.random.PCG64(cfg.seed + 1000 * layer))


def make_layer(cfg: LayerConfig, layer: int = 0, device=None, project_on=None) -> dict:
    """One layer's inputs as torch tensors in the working dtype.

    Returns x [N, D], W_gate/W_up [F, D], W_down [D, F], and Q [N, hq, d],
    K/V [N, hkv, d] computed as x·W (the harness projection, no RoPE).  The
    projection runs in torch on ``project_on`` (a device, default CPU in fp32)
    and its result is rounded to the working dtype; it is an input to the
    method, identical for both sides of any comparison.  ``device`` moves the
    returned tensors.
    """
    import torch
    rng = layer_rng(cfg, layer)
    x32 = make_hidden(cfg, rng)
    w32 = make_weights(cfg, rng, with_o=cfg.n_layers > 1)
    out = {"x": _round(x32, cfg.dtype)}
    del x32
    for k, v in w32.items():
        out[k] = _round(v, cfg.dtype)
    out.update(project_qkv(cfg, out["x"], out["W_q"], out["W_k"], out["W_v"], project_on))
    if device is not None:
        out = {k: v.to(device) for k, v in out.items()}
    return out


def make_upstream(cfg: LayerConfig, layer: int = 0) -> dict:
    """Upstream gradients for the backward pass, from their own stream (seed +
    500 + 1000 * layer): dO [N, hq, d] in the working dtype (the attention
    output's type) and dy [N, D] float32 (the FFN output's type), both N(0, 1).
    Torch CPU tensors."""
    import torch
    rng = np.random.Generator(np.random.PCG64(cfg.seed + 500 + 1000 * layer))
    dO = _normal(rng, (cfg.n_tokens, cfg.hq, cfg.d))
    dy = _normal(rng, (cfg.n_tokens, cfg.D))
    return {"dO": _round(dO, cfg.dtype), "dy": torch.from_numpy(dy)}


def make_stack(cfg: LayerConfig, layer: int) -> dict:
    """Stacked workload (several independent layers): the first layer draws the
    hidden state then its weights from its own stream; later layers draw only
    their weights (W_q, W_k, W_v, W_gate, W_up, W_down, W_o) from theirs.
    Returns rounded torch CPU tensors ("x" only for layer 0)."""
    rng = layer_rng(cfg, layer)
    out = {}
    if layer == 0:
        out["x"] = _round(make_hidden(cfg, rng), cfg.dtype)
    for k, v in make_weights(cfg, rng, with_o=True).items():
        out[k] = _round(v, cfg.dtype)
    return out


def project_qkv(cfg: LayerConfig, x, W_q, W_k, W_v, project_on=None) -> dict:
    """Q/K/V = x·W in the working dtype (harness step outside the method)."""
    import torch
    dev = torch.device(project_on) if project_on is not None else torch.device("cpu")
    N = x.shape[0]
    res = {}
    for name, W, h in (("Q", W_q, cfg.hq), ("K", W_k, cfg.hkv), ("V", W_v, cfg.hkv)):
        if dev.type == "cpu":
            y = (x.float() @ W.float())
        else:
            y = (x.to(dev) @ W.to(dev)).float()
        res[name] = y.to(x.dtype).reshape(N, h, cfg.d).contiguous().to("cpu")
    return res


def small_config(name="small", grid=(4, 8, 8), cube=(4, 4, 2), n_text=40, D=256, hq=8,
                 hkv=2, d=128, F=512, dtype="bf16", p=0.7, seed=BASE_SEED + 77,
                 sigma=None, sigma_range=(0.1, 1.0), cube_sizes=None,
                 structure="proto") -> LayerConfig:
    """A small layer for element-wise parity (several tiles plus ragged tails)."""
    return LayerConfig(name=name, grid=grid, cube=cube, n_text=n_text, D=D, hq=hq, hkv=hkv,
                       d=d, F=F, dtype=dtype, p=p, sigma=sigma, sigma_range=sigma_range,
                       seed=seed, cube_sizes=cube_sizes, structure=structure)


def dense_flops(cfg: LayerConfig) -> dict:
    """Algorithmic FLOPs of the dense layer (attention: QK^T and PV over the
    causal triangle; FFN: three D x F GEMMs).  Pure counting of sizes."""
    N = cfg.n_tokens
    attn = 4.0 * cfg.d * cfg.hq * N * (N + 1) / 2.0
    ffn = 6.0 * cfg.D * cfg.F * N
    return {"attn": attn, "ffn": ffn}
