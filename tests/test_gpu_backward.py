"""Backward pass (selection straight-through) against the float64 oracle
(needs a B200): AdaS-FFN gradients of x and the three weights, AdaS-Attn
gradients of Q, K and V, each on the sets of the library's own forward call."""
import pytest
import torch

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


def test_attn_backward_topk_and_determinism(bcase):
    rep = {}
    g1, _ = parity.check_attn_backward(bcase, k=3, report=rep)
    print(bcase["cfg"].name, "attn top-3", rep)
    g2, _, _, _ = parity.run_attn_backward(bcase, k=3)
    for a, b in zip(g1, g2):      # no atomics: repeat runs agree bit for bit
        assert torch.equal(a, b)
