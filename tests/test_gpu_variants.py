"""Selection variants against the float64 oracle (needs a B200): Top-K cube
selection (the fixed-size strategy of the paper's ablation of selection
strategies; sets bit for bit except at near-ties, P_(k) - P_(k+1) below the
1e-5 margin), Uniform Sampling (the content-independent strategy of the same
ablation; sets exactly) and the AdaS-FFN importance alternatives (energy share,
softmax of norms). Outputs are compared on the library's own sets within the stated
tolerance."""
import numpy as np
import pytest
import torch

import ffn_long_video_b200 as fb
import workloads
from tests import parity
from tests.test_gpu_parity import SMALL, _sample_tokens

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", params=["tiny-fp32", "small-bf16", "mid-bf16", "ragged-bf16"])
def case(request):
    return parity.make_case(SMALL[request.param])


@pytest.mark.parametrize("k", [1, 3, 8, 1000])
def test_topk_small(case, k):
    rep = {}
    parity.check_attn(case, k=k, report=rep)
    print(case["cfg"].name, k, rep)


def test_topk_counts(case):
    """Every visual row of cube c selects exactly min(k, c) cubes."""
    cfg = case["cfg"]
    off = case["off_np"]
    cube = np.searchsorted(off, np.arange(cfg.n_vis), side="right") - 1
    for k in (2, 5):
        _, sel, _ = parity.run_attn(case, k=k)
        counts = sel.sum(axis=2)
        assert (counts == np.minimum(k, cube)[:, None]).all()


def test_topk_full_size_sampled():
    """The 3B-shaped 18K layer with k = 16, sampled tokens (all heads)."""
    cfg = workloads.CONFIGS[2]
    c = parity.make_case(cfg)
    rep = {}
    parity.check_attn(c, k=16, tokens=_sample_tokens(cfg, 32, 5), report=rep)
    print(cfg.name, "top-16", rep)


# ------------------------------------------------- Uniform Sampling
@pytest.mark.parametrize("k", [1, 3, 8, 1000])
def test_uniform_small(case, k):
    """Uniform Sampling (k evenly spaced preceding cubes): sets equal to the
    oracle's exactly (no scores, so no margin), outputs on those sets."""
    rep = {}
    parity.check_attn(case, uniform=k, report=rep)
    print(case["cfg"].name, "uniform", k, rep)


def test_uniform_full_size_sampled():
    """The 7B-shaped 64K layer with 70 evenly spaced cubes (about the mean
    Top-p set size at p = 0.7 there), sampled tokens (all heads)."""
    cfg = workloads.CONFIGS[3]
    c = parity.make_case(cfg)
    rep = {}
    parity.check_attn(c, uniform=70, tokens=_sample_tokens(cfg, 24, 6), report=rep)
    print(cfg.name, "uniform-70", rep)


# ------------------------------------------------- AdaS-FFN importance variants
@pytest.mark.parametrize("importance", ["l2sq", "softmax"])
@pytest.mark.parametrize("p", [0.5, 0.8])
def test_ffn_importance_variants(case, importance, p):
    """The energy share and the softmax of norms (alternatives to the linear
    L2-norm share) against the oracle: active sets bit for bit outside the
    margin, outputs on the library's own sets."""
    rep = {}
    parity.check_ffn(case, p=p, importance=importance, report=rep)
    print(case["cfg"].name, importance, p, rep)
