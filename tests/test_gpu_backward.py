"""Backward pass (selection straight-through) against the float64 oracle
(needs a B200): AdaS-FFN gradients of x and the three weights, AdaS-Attn
gradients of Q, K and V, each on the sets of the library's own forward call."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests import parity

pytestmark = pytest.mark.gpu

CASES = {
    "small": workloads.small_config(),
    # several 128-row tiles and F tiles, 64-token cubes
    "mid": workloads.small_config(name="mid", grid=(8, 16, 16), cube=(4, 4, 4), n_text=72,
                                  D=512, hq=16, hkv=2, F=1024, seed=99),
    # truncated edge cubes incl. a single-token cube; D not a multiple of 256
    "ragged": workloads.small_config(name="ragged", grid=(4, 8, 8), cube=(4, 4, 2), n_text=17,
                                     D=320, hq=4, hkv=2, F=384, seed=7,
                                     cube_sizes=(32, 1, 31, 64, 17, 47, 32, 32)),
}


@pytest.fixture(scope="module", params=list(CASES))
def bcase(request):
    return parity.make_case(CASES[request.param])


@pytest.mark.parametrize("p", [0.7, 0.4, 1.0])
def test_ffn_backward(bcase, p):
    rep = {}
    parity.check_ffn_backward(bcase, p=p, report=rep)
    print(bcase["cfg"].name, p, rep)


@pytest.mark.parametrize("p", [0.7, 0.4, 1.0])
def test_attn_backward(bcase, p):
    rep = {}
    parity.check_attn_backward(bcase, p=p, report=rep)
    print(bcase["cfg"].name, "attn", p, rep)


@pytest.mark.parametrize("p", [0.7, 1.0])
def test_attn_train_forward_and_backward(bcase, p):
    """The training-mode forward: same sets, output within the forward bar; its
    backward (D_r from the fp32 output, one walk over the keys) within the
    gradient bar, and within rounding of the inference forward's backward."""
    rep = {}
    parity.check_attn(bcase, p=p, report=rep, train=True)
    g_train, _ = parity.check_attn_backward(bcase, p=p, report=rep, train=True)
    g_inf, _, _, _ = parity.run_attn_backward(bcase, p=p)
    for a, b, nm in zip(g_train, g_inf, ("dQ", "dK", "dV")):
        d = (a - b).double()
        assert (d.norm() / b.double().norm()).item() < 5e-3, nm
    print(bcase["cfg"].name, "attn train", p, rep)


def test_attn_backward_topk_and_determinism(bcase):
    rep = {}
    g1, _ = parity.check_attn_backward(bcase, k=3, report=rep)
    print(bcase["cfg"].name, "attn top-3", rep)
    g2, _, _, _ = parity.run_attn_backward(bcase, k=3)
    for a, b in zip(g1, g2):      # no atomics: repeat runs agree bit for bit
        assert torch.equal(a, b)


# ------------------------------------------------------------------ full size
@pytest.fixture(scope="module")
def case_18k():
    return parity.make_case(workloads.CONFIGS[2])


def test_backward_full_size_3b_18k(case_18k):
    """The 3B-shaped 18K layer in the bench's launch configuration: gradients on
    rows the oracle can take exactly - dQ of the first, a middle and the last
    cube and of the text rows; dK, dV of the last cube's and the text keys
    (which no other rows admit); dx of those cubes and the text rows - and the
    dV column-sum invariant over every key."""
    case = case_18k
    cfg, t = case["cfg"], case["t"]
    C = cfg.n_cubes
    (dQ, dK, dV), sets, dO, _ = parity.run_attn_backward(case)
    Qc, Kc, Vc, dOc = t["Q"].cpu(), t["K"].cpu(), t["V"].cpu(), dO.cpu()
    off = case["off_np"]
    rep = {}
    for cubes, text in (([C - 1], True), ([0, C // 2], False)):
        *want, mags = oracle.attention_backward_given_sets(Qc, Kc, Vc, dOc, off, cfg.n_vis, sets,
                                                           with_magnitudes=True, cubes=cubes,
                                                           text=text)
        rows = np.concatenate([np.arange(off[c], off[c + 1]) for c in cubes] +
                              ([np.arange(cfg.n_vis, cfg.n_tokens)] if text else []))
        parity.check_grad(dQ.cpu().numpy()[rows], want[0][rows], f"dQ{cubes}", rep, mags[0][rows])
        if text:
            keys = np.arange(off[C - 1], cfg.n_tokens)
            parity.check_grad(dK.cpu().numpy()[keys], want[1][keys], "dK-last", rep, mags[1][keys])
            parity.check_grad(dV.cpu().numpy()[keys], want[2][keys], "dV-last", rep, mags[2][keys])
    g = cfg.hq // cfg.hkv
    colsum = dV.double().sum(0)
    expect = dO.double().reshape(cfg.n_tokens, cfg.hkv, g, cfg.d).sum((0, 2))
    assert ((colsum - expect).norm() / expect.norm()).item() < 2e-3
    assert all(torch.isfinite(x).all() for x in (dQ, dK, dV))

    (dx, dWg, dWu, dWd), act, dy = parity.run_ffn_backward(case)
    cubes = [0, C // 2, C - 1]
    want = oracle.ffn_backward_given_sets(t["x"].cpu(), t["W_gate"].cpu(), t["W_up"].cpu(),
                                          t["W_down"].cpu(), off, cfg.n_vis, act, dy.cpu(),
                                          cubes=cubes, text=True)[0]
    rows = np.concatenate([np.arange(off[c], off[c + 1]) for c in cubes] +
                          [np.arange(cfg.n_vis, cfg.n_tokens)])
    parity.check_grad(dx.cpu().numpy()[rows], want[rows], "dx", rep)
    assert all(torch.isfinite(x).all() for x in (dx, dWg, dWu, dWd))
    print(cfg.name, rep)


EDGE = {
    # no text tokens at all
    "no-text": workloads.small_config(name="notext", grid=(4, 8, 8), cube=(4, 4, 2), n_text=0,
                                      D=256, hq=4, hkv=2, F=256, seed=61),
    # one query head per KV head (g = 1), odd number of 64-key pieces
    "g1-odd": workloads.small_config(name="g1", grid=(4, 8, 8), cube=(4, 4, 4), n_text=9,
                                     D=256, hq=2, hkv=2, F=256, seed=62,
                                     cube_sizes=(64, 64, 64, 63, 1)),
    # a single cube plus a short text tail
    "one-cube": workloads.small_config(name="onecube", grid=(4, 4, 4), cube=(4, 4, 4),
                                       n_text=5, D=256, hq=4, hkv=1, F=256, seed=63),
}


@pytest.mark.parametrize("name", list(EDGE))
def test_backward_edge_layouts(name):
    case = parity.make_case(EDGE[name])
    rep = {}
    parity.check_attn_backward(case, p=0.6, report=rep)
    parity.check_ffn_backward(case, p=0.6, report=rep)
    print(name, rep)
