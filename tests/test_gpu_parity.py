"""Parity of the CUDA path against the float64 oracle (needs a B200).

Element-wise on sizes the oracle finishes in seconds (several tiles, ragged
tails, truncated and single-token cubes), and on sampled rows / cubes at the
full Qwen2.5-VL-3B-shaped size."""
import numpy as np
import pytest
import torch

import ffn_long_video_b200 as fb
import workloads
from tests import parity

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny-fp32": workloads.CONFIGS[1],
    # 8 query heads / 2 KV heads, 32-token cubes: 8 visual tiles per KV head,
    # a ragged text tile (40 text tokens)
    "small-bf16": workloads.small_config(),
    # the 3B shape (16/2 heads, 64-token cubes) on a 2048-token grid
    "mid-bf16": workloads.small_config(name="mid", grid=(8, 16, 16), cube=(4, 4, 4), n_text=72,
                                       D=512, hq=16, hkv=2, F=1024, seed=99),
    # truncated edge cubes, one of them a single token
    "ragged-bf16": workloads.small_config(name="ragged", grid=(4, 8, 8), cube=(4, 4, 2),
                                          n_text=17, D=256, hq=4, hkv=2, F=256, seed=7,
                                          cube_sizes=(32, 1, 31, 64, 17, 47, 32, 32)),
    "ragged-fp32": workloads.small_config(name="ragged32", grid=(4, 8, 8), cube=(4, 4, 2),
                                          n_text=9, D=128, hq=4, hkv=1, d=64, F=256,
                                          dtype="fp32", seed=8,
                                          cube_sizes=(1, 63, 32, 32, 40, 24, 60, 1, 1, 2)),
    # bf16 with head_dim 64 (one 64-dim half per query and key row)
    "d64-bf16": workloads.small_config(name="d64", grid=(8, 16, 16), cube=(4, 4, 4), n_text=40,
                                       D=256, hq=8, hkv=2, d=64, F=256, seed=15),
    "ragged-d64": workloads.small_config(name="ragged-d64", grid=(4, 8, 8), cube=(4, 4, 2),
                                         n_text=21, D=192, hq=6, hkv=3, d=64, F=384, seed=16,
                                         cube_sizes=(3, 61, 32, 7, 57, 33, 1, 31, 2, 29)),
}


@pytest.fixture(scope="module", params=list(SMALL))
def small_case(request):
    torch.manual_seed(0)
    return parity.make_case(SMALL[request.param])


@pytest.mark.parametrize("p", [0.7, 0.3, 1.0])
def test_attn_small(small_case, p):
    rep = {}
    parity.check_attn(small_case, p=p, report=rep)
    print(small_case["cfg"].name, p, rep)


@pytest.mark.parametrize("p", [0.7, 0.45, 1.0])
def test_ffn_small(small_case, p):
    rep = {}
    parity.check_ffn(small_case, p=p, report=rep)
    print(small_case["cfg"].name, p, rep)


def test_attn_smallest_p_picks_argmax(small_case):
    """p -> 0+: every visual row of cube i > 0 selects exactly one cube."""
    cfg = small_case["cfg"]
    _, sel, _ = parity.run_attn(small_case, p=1e-7)
    off = small_case["off_np"]
    cube = np.searchsorted(off, np.arange(cfg.n_vis), side="right") - 1
    counts = sel.sum(axis=2)
    assert (counts[cube > 0] == 1).all()
    assert (counts[cube == 0] == 0).all()


def test_repeat_runs_identical_sets(small_case):
    """The selection sets are deterministic run to run."""
    _, s1, _ = parity.run_attn(small_case)
    _, s2, _ = parity.run_attn(small_case)
    assert np.array_equal(s1, s2)
    _, a1, _ = parity.run_ffn(small_case)
    _, a2, _ = parity.run_ffn(small_case)
    assert np.array_equal(a1, a2)


# ------------------------------------------------------------------ full sizes
def _sample_tokens(cfg, n, seed):
    rng = np.random.default_rng(seed)
    off = cfg.offsets
    picks = set(rng.choice(cfg.n_vis, size=n, replace=False).tolist())
    picks |= {0, off[1] - 1, off[1], cfg.n_vis - 1}          # first cube, second cube, last
    picks |= set(range(cfg.n_vis, cfg.n_tokens, max(1, cfg.n_text // 8)))  # text rows
    picks.add(cfg.n_tokens - 1)
    return np.array(sorted(picks))


@pytest.mark.parametrize("cfg_id", [2, 3])
def test_full_size_sampled(cfg_id):
    """The 3B-shaped 18K layer and the 7B-shaped 64K layer at full size, in the
    launch configuration the bench times: selection sets and outputs of
    sampled tokens (all heads) and sampled cubes against the oracle."""
    cfg = workloads.CONFIGS[cfg_id]
    case = parity.make_case(cfg)
    rep = {}
    parity.check_attn(case, tokens=_sample_tokens(cfg, 48, cfg_id), report=rep)
    print(cfg.name, "attn", rep)
    rng = np.random.default_rng(cfg_id)
    cubes = np.unique(np.concatenate([[0, cfg.n_cubes - 1],
                                      rng.choice(cfg.n_cubes, 10, replace=False)]))
    rep = {}
    parity.check_ffn(case, cubes=cubes, text=True, report=rep)
    print(cfg.name, "ffn", rep)


@pytest.mark.parametrize("shape", [(4, 4, 4), (8, 8, 2)])
def test_128k_sweep_sampled(shape):
    """The 7B-shaped 128K layer: p in {0.5, 0.7, 0.9, 1.0} on both cube shapes
    (64-token and 128-token cubes), sampled tokens and cubes."""
    idxs = [i for i, (p, c) in enumerate(workloads.SWEEP_4) if c == shape]
    cfg0 = workloads.sweep_config(idxs[0])
    case = parity.make_case(cfg0)
    for i in idxs:
        cfg = workloads.sweep_config(i)
        case["cfg"] = cfg
        rep = {}
        parity.check_attn(case, p=cfg.p, tokens=_sample_tokens(cfg, 24, i), report=rep)
        print(cfg.name, "attn", rep)
        rng = np.random.default_rng(i)
        cubes = np.unique(np.concatenate([[0, cfg.n_cubes - 1],
                                          rng.choice(cfg.n_cubes, 6, replace=False)]))
        rep = {}
        parity.check_ffn(case, p=cfg.p, cubes=cubes, text=(cfg.p == 0.7), report=rep)
        print(cfg.name, "ffn", rep)


def test_262k_four_layer_stack_sampled():
    """Four independently seeded 7B-shaped layers at 262K visual tokens, half of
    the cubes near-duplicates of earlier ones. The harness wires the stack
    (Q/K/V = x W, h = x + out W_o, next x = y scaled to unit RMS per token, in
    place of the RMSNorm a decoder applies between layers, so that the random
    weights do not blow the residual stream up layer after layer); each layer's
    AdaS-Attn and AdaS-FFN are checked against the oracle on that layer's own
    inputs."""
    cfg = workloads.CONFIGS[5]
    ids, off, text, off_np = parity.layout_tensors(cfg)
    x = None
    for layer in range(cfg.n_layers):
        w = {k: v.cuda() for k, v in workloads.make_stack(cfg, layer).items()}
        if layer == 0:
            x = w.pop("x")
        qkv = workloads.project_qkv(cfg, x, w["W_q"], w["W_k"], w["W_v"], project_on="cuda")
        t = {k: v.cuda() for k, v in qkv.items()}
        case = {"cfg": cfg, "t": dict(t), "ids": ids, "off": off, "text": text, "off_np": off_np}
        rep = {}
        out, _, _ = parity.check_attn(case, tokens=_sample_tokens(cfg, 16, 50 + layer), report=rep)
        print(cfg.name, "layer", layer, "attn", rep)
        h = (x.float() + (out.reshape(cfg.n_tokens, -1).float() @ w["W_o"].float())).to(x.dtype)
        del out
        case["t"] = {"x": h, "W_gate": w["W_gate"], "W_up": w["W_up"], "W_down": w["W_down"]}
        rng = np.random.default_rng(60 + layer)
        cubes = np.unique(np.concatenate([[0, cfg.n_cubes - 1],
                                          rng.choice(cfg.n_cubes, 4, replace=False)]))
        rep = {}
        y, _, _ = parity.check_ffn(case, cubes=cubes, text=(layer == 0), report=rep)
        print(cfg.name, "layer", layer, "ffn", rep)
        x = (y * torch.rsqrt(y.pow(2).mean(dim=1, keepdim=True) + 1e-6)).to(x.dtype)
        del y, h, t, qkv, w
        torch.cuda.empty_cache()


# ------------------------------------------------------------------ cut-bin stress
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("fp32", 64)])
def test_attn_uniform_means_closed_form(dtype, d):
    """Every key identical -> every cube mean identical -> P uniform over the c
    preceding cubes: exact ties, the cut bin holds all of them, and the Top-p
    set must be the ceil(p*c) lowest-index cubes (several extra passes)."""
    import math
    import ffn_long_video_b200 as fb
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    C, n, hq, hkv, n_text = 90, 8, 2, 1, 5
    n_vis = C * n
    N = n_vis + n_text
    g = torch.Generator().manual_seed(11)
    Q = torch.randn(N, hq, d, generator=g).to(tdt).cuda()
    K = torch.randn(1, hkv, d, generator=g).expand(N, hkv, d).contiguous().to(tdt).cuda()
    V = torch.randn(N, hkv, d, generator=g).to(tdt).cuda()
    ids = torch.cat([torch.arange(C, dtype=torch.int32).repeat_interleave(n),
                     torch.full((n_text,), -1, dtype=torch.int32)]).cuda()
    off = (torch.arange(C + 1, dtype=torch.int32) * n).cuda()
    for p in (0.7, 0.33):
        out, ws = fb.cube_attn(Q, K, V, ids, off, n_vis, p)
        torch.cuda.synchronize()
        assert fb.read_device_status(ws)[0] == fb.OK
        sel = fb.attn_export_sets(ws, ids, C, n_vis, N, hq, hkv, d,
                                  fb.BF16 if dtype == "bf16" else fb.FP32)
        for t in range(n_vis):
            c = t // n
            if c > 0 and abs(p * c - round(p * c)) < 1e-6:
                continue
            k = math.ceil(p * c) if c > 0 else 0
            want = np.zeros(C, bool)
            want[:k] = True
            for h in range(hq):
                assert np.array_equal(sel[t, h], want), (p, t, h, np.nonzero(sel[t, h])[0][:8])
        st = fb.attn_read_stats(ws)
        assert st["overflow_rows"] > 0          # the extra-pass path ran


def test_attn_flat_random_scores():
    """Unstructured Q/K (near-uniform cube relevance): wide cut bins on many
    rows; sets and outputs still match the oracle."""
    cfg = workloads.small_config(name="flat", grid=(8, 16, 16), cube=(4, 4, 2), n_text=30,
                                 D=256, hq=4, hkv=2, F=256, seed=5)
    g = torch.Generator().manual_seed(3)
    N = cfg.n_tokens
    t = {"Q": torch.randn(N, cfg.hq, cfg.d, generator=g).to(torch.bfloat16).cuda(),
         "K": torch.randn(N, cfg.hkv, cfg.d, generator=g).to(torch.bfloat16).cuda(),
         "V": torch.randn(N, cfg.hkv, cfg.d, generator=g).to(torch.bfloat16).cuda()}
    ids, off, text, off_np = parity.layout_tensors(cfg)
    case = {"cfg": cfg, "t": t, "ids": ids, "off": off, "text": text, "off_np": off_np}
    for p in (0.7, 0.95):
        rep = {}
        parity.check_attn(case, p=p, report=rep)
        print("flat", p, rep)


def test_attn_crowded_cut_bins():
    """Unstructured Q/K over 511 preceding cubes: many rows' cut bins hold more
    scores than the per-row list, so the selection resolves them through the
    finer histogram of the cut bin (and, where a fine bin is crowded too, the
    list passes); sets and outputs still match the oracle on sampled tokens."""
    cfg = workloads.small_config(name="crowded", grid=(16, 32, 32), cube=(4, 4, 2), n_text=16,
                                 D=256, hq=2, hkv=1, F=256, seed=6)
    g = torch.Generator().manual_seed(4)
    N = cfg.n_tokens
    t = {"Q": torch.randn(N, cfg.hq, cfg.d, generator=g).to(torch.bfloat16).cuda(),
         "K": torch.randn(N, cfg.hkv, cfg.d, generator=g).to(torch.bfloat16).cuda(),
         "V": torch.randn(N, cfg.hkv, cfg.d, generator=g).to(torch.bfloat16).cuda()}
    ids, off, text, off_np = parity.layout_tensors(cfg)
    case = {"cfg": cfg, "t": t, "ids": ids, "off": off, "text": text, "off_np": off_np}
    tokens = _sample_tokens(cfg, 96, 7)
    for p in (0.9, 0.5):
        rep = {}
        _, _, ws = parity.check_attn(case, p=p, tokens=tokens, report=rep)
        st = fb.attn_read_stats(ws)
        print("crowded", p, rep, "rows needing extra passes", st["overflow_rows"])
        assert st["overflow_rows"] > 0


def test_attn_d64_training_mode_and_variants():
    """bf16 with head_dim 64 through the training-mode forward (P as a bf16
    pair, fp32 O kept), Top-K and Uniform Sampling, against the oracle."""
    case = parity.make_case(SMALL["d64-bf16"])
    for kw in ({"train": True}, {"k": 3}, {"uniform": 4}):
        rep = {}
        parity.check_attn(case, report=rep, **kw)
        print("d64", kw, rep)
