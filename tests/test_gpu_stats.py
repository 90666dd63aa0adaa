"""The library's realised-sparsity and near-margin counters against the oracle
(needs a B200).

The counters of adaspark_attn_read_stats / adaspark_ffn_read_stats are what the
bench reports at sizes the oracle cannot take in full, so they are checked here
on layers the oracle takes whole: the selected-pair counts exactly, and the
near-margin counts (cuts within 1e-5 of flipping, decided by the library from
fp32 masses) between the oracle's float64 counts at half and twice the margin."""
import numpy as np
import pytest

import ffn_long_video_b200 as fb
import oracle
import workloads
from tests import parity

pytestmark = pytest.mark.gpu

CASES = {
    "3b-heads": workloads.small_config(name="stats-3b", grid=(8, 16, 16), cube=(4, 4, 4),
                                       n_text=64, D=512, hq=16, hkv=2, F=512, seed=71),
    "7b-heads": workloads.small_config(name="stats-7b", grid=(8, 16, 16), cube=(4, 4, 4),
                                       n_text=32, D=512, hq=28, hkv=4, F=512, seed=72),
}


@pytest.fixture(scope="module", params=list(CASES))
def stats_case(request):
    return parity.make_case(CASES[request.param])


def _sandwich(lib, margins):
    lo = int((margins < 0.5 * parity.MARGIN).sum())
    hi = int((margins < 2.0 * parity.MARGIN).sum())
    assert lo <= lib <= hi, (lo, lib, hi)


@pytest.mark.parametrize("p", [0.7, 0.5])
def test_attn_counters(stats_case, p):
    cfg, t = stats_case["cfg"], stats_case["t"]
    out, gsel, ws = parity.run_attn(stats_case, p)
    st = fb.attn_read_stats(ws)
    osel, margin = oracle.select_cubes(t["Q"].cpu(), t["K"].cpu(), stats_case["off_np"],
                                       cfg.n_vis, cfg.hq, cfg.hkv, p, with_margin=True)
    own = np.searchsorted(stats_case["off_np"], np.arange(cfg.n_vis), side="right") - 1
    assert st["visual_rows"] == int((own > 0).sum()) * cfg.hq
    assert st["candidate_pairs"] == int(own.sum()) * cfg.hq
    assert st["selected_pairs"] == int(gsel.sum())
    _sandwich(st["near_margin_rows"], margin[own > 0])


@pytest.mark.parametrize("p", [0.7, 0.5])
def test_ffn_counters(stats_case, p):
    cfg, t = stats_case["cfg"], stats_case["t"]
    y, act, ws = parity.run_ffn(stats_case, p)
    st = fb.ffn_read_stats(ws)
    oact, margins = oracle.ffn_select(t["x"].cpu(), stats_case["off_np"], cfg.n_vis, p,
                                      with_margin=True)
    assert st["active_visual"] == int(act[:cfg.n_vis].sum())
    assert st["skipped_visual"] == cfg.n_vis - int(act[:cfg.n_vis].sum())
    assert st["text_tokens"] == cfg.n_text
    _sandwich(st["near_margin_cubes"], margins)
