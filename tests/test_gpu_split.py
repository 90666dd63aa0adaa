"""The split walk of the bf16 AdaS-Attn forward (adaspark_set_split_rows): a
tile's selected cubes that few of its rows chose run in gathered tiles whose
partial results the rows merge. The selection is unchanged, so the exported
sets equal those of the single walk; the outputs follow the oracle on those
sets at the protocol's tolerances, and stay within bf16 rounding of the single
walk's (needs a B200)."""
import numpy as np
import pytest
import torch

import ffn_long_video_b200 as fb
import workloads
from tests import parity

pytestmark = pytest.mark.gpu

# 4096 visual tokens (32 tiles per head, 64 cubes of 64 tokens), ragged text
CFG = workloads.small_config(name="split", grid=(16, 16, 16), cube=(4, 4, 4), n_text=37, D=256,
                             hq=8, hkv=2, F=256, seed=2718)


@pytest.fixture(scope="module")
def case():
    return parity.make_case(CFG)


def _run(case, rows, p=None, k=None):
    fb.set_split_rows(rows)
    try:
        cfg, t = case["cfg"], case["t"]
        if k is None:
            out, ws = fb.cube_attn(t["Q"], t["K"], t["V"], case["ids"], case["off"], cfg.n_vis,
                                   cfg.p if p is None else p)
        else:
            out, ws = fb.cube_attn_topk(t["Q"], t["K"], t["V"], case["ids"], case["off"],
                                        cfg.n_vis, k)
        torch.cuda.synchronize()
        code, det = fb.read_device_status(ws)
        assert code == fb.OK, (code, hex(det))
        bits = fb.attn_export_bits(ws, case["ids"], cfg.n_cubes, cfg.n_vis, cfg.n_tokens, cfg.hq,
                                   cfg.hkv, cfg.d, fb.BF16)
        return out, bits.clone(), fb.attn_read_stats(ws)
    finally:
        fb.set_split_rows(fb.SPLIT_ROWS_DEFAULT)


@pytest.mark.parametrize("rows", [1, 8, 32, 128])
def test_split_walk_against_single_walk_and_oracle(case, rows):
    single, bits0, st0 = _run(case, 0)
    split, bits1, st1 = _run(case, rows)
    assert torch.equal(bits0, bits1)                 # the same sets
    assert st0["split_pairs"] == 0 and st0["gathered_blocks"] == 0
    assert st1["split_pairs"] > 0, st1
    # the tiles walk fewer blocks; the moved pairs run in gathered blocks
    assert st1["key_blocks"] < st0["key_blocks"], (st0, st1)
    assert st1["gathered_blocks"] >= (st1["split_pairs"] + 127) // 128
    d = (split.float() - single.float()).abs()
    ref = single.float().abs()
    # merged partial outputs in bf16: a few bf16 ulps of the result at most
    assert float((d - 4 * ref * 2.0 ** -8).max()) <= 2e-3, float(d.max())
    # and the split output itself against the oracle on the library's sets
    fb.set_split_rows(rows)
    try:
        rep = {}
        parity.check_attn(case, report=rep)
        print("rows", rows, "split pairs", st1["split_pairs"], "gathered blocks",
              st1["gathered_blocks"], "key blocks", st0["key_blocks"], "->", st1["key_blocks"], rep)
    finally:
        fb.set_split_rows(fb.SPLIT_ROWS_DEFAULT)


def test_split_walk_top_k(case):
    single, bits0, _ = _run(case, 0, k=6)
    split, bits1, st1 = _run(case, 128, k=6)
    assert torch.equal(bits0, bits1)
    assert st1["split_pairs"] > 0
    fb.set_split_rows(128)
    try:
        parity.check_attn(case, k=6)
    finally:
        fb.set_split_rows(fb.SPLIT_ROWS_DEFAULT)


def test_split_walk_small_workspace_runs_single_walk(case):
    """A workspace of the common layout alone (the fp32 figure) runs the single
    walk: no split pairs, output equal to the single walk's."""
    cfg, t = case["cfg"], case["t"]
    single, _, _ = _run(case, 0)
    nbytes = fb.cube_attn_workspace_bytes(cfg.n_tokens, cfg.n_vis, cfg.n_cubes, cfg.hq, cfg.hkv,
                                          cfg.d, fb.FP32)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    out, ws = fb.cube_attn(t["Q"], t["K"], t["V"], case["ids"], case["off"], cfg.n_vis, cfg.p,
                           workspace=ws)
    torch.cuda.synchronize()
    assert fb.attn_read_stats(ws)["split_pairs"] == 0
    assert torch.equal(out, single)


def test_split_walk_backward_after_inference_forward(case):
    """The backward after a split inference forward walks the whole sets (the
    tile lists stay whole) and takes the merged log2-sum-exp: it equals the
    backward after a single-walk forward up to the forward's rounding."""
    cfg, t = case["cfg"], case["t"]
    torch.manual_seed(5)
    dO = (torch.randn(cfg.n_tokens, cfg.hq, cfg.d, device="cuda") * 0.1).to(torch.bfloat16)
    grads = {}
    for rows in (0, 8):
        fb.set_split_rows(rows)
        try:
            out, ws = fb.cube_attn(t["Q"], t["K"], t["V"], case["ids"], case["off"], cfg.n_vis,
                                   cfg.p)
            g = fb.cube_attn_backward(t["Q"], t["K"], t["V"], dO, case["ids"], case["off"],
                                      cfg.n_vis, ws)
            torch.cuda.synchronize()
            grads[rows] = [x.float().clone() for x in g[:3]]
        finally:
            fb.set_split_rows(fb.SPLIT_ROWS_DEFAULT)
    for a, b, nm in zip(grads[0], grads[8], ("dQ", "dK", "dV")):
        scale = float(a.abs().max()) + 1e-12
        assert float((a - b).abs().max()) <= 2e-2 * scale, nm


# gathered tiles over several 64-key pieces (128-token cubes, online softmax
# across the pieces), ragged cubes (pieces shorter than 64 keys) and head_dim 64
MORE = {
    "cubes-8x8x2": workloads.small_config(name="split-8x8x2", grid=(8, 32, 32), cube=(8, 8, 2),
                                          n_text=19, D=256, hq=8, hkv=2, F=256, seed=4242),
    "ragged": workloads.small_config(name="split-ragged", grid=(8, 16, 16), cube=(4, 4, 2),
                                     n_text=23, D=256, hq=6, hkv=3, F=256, seed=4343,
                                     cube_sizes=(121, 81, 88, 115, 75, 100, 107, 29, 8, 39, 37,
                                                 112, 117, 1, 64, 106, 17, 103, 16, 60, 105,
                                                 39, 44, 36, 93, 33, 127, 57, 62, 56)),
    "d64": workloads.small_config(name="split-d64", grid=(16, 16, 16), cube=(4, 4, 4), n_text=37,
                                  D=256, hq=8, hkv=2, d=64, F=256, seed=4444),
}


@pytest.mark.parametrize("name", list(MORE))
def test_split_walk_pieces_ragged_and_d64(name):
    case = parity.make_case(MORE[name])
    single, bits0, st0 = _run(case, 0)
    for rows in (8, 128):
        split, bits1, st1 = _run(case, rows)
        assert torch.equal(bits0, bits1)
        if rows == 128:
            assert st1["split_pairs"] > 0, st1
        d = (split.float() - single.float()).abs()
        assert float((d - 4 * single.float().abs() * 2.0 ** -8).max()) <= 2e-3, (rows,
                                                                                float(d.max()))
        fb.set_split_rows(rows)
        try:
            rep = {}
            parity.check_attn(case, report=rep)
            print(name, "rows", rows, "split pairs", st1["split_pairs"], "gathered blocks",
                  st1["gathered_blocks"], rep)
        finally:
            fb.set_split_rows(fb.SPLIT_ROWS_DEFAULT)
