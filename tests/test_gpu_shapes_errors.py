"""Cube-shape generality and device-detected errors (needs a B200).

Shapes: the 8x8x4 (256-token) cube of the pages' training setting, 1x1x64
tubes, 8x8x1 patches and 8x8x2 cubes, each checked element-wise against the
float64 oracle. Errors: inputs that only the kernels can see as wrong must come
back as ADASPARK_EDEVICE with the matching status bit, and the call must leave
the device usable."""
import numpy as np
import pytest
import torch

import ffn_long_video_b200 as fb
import workloads
from tests import parity

pytestmark = pytest.mark.gpu

SHAPES = {
    # 256-token cubes: four 64-key blocks per cube, two 128-row tiles per cube
    "cube-8x8x4": workloads.small_config(name="c884", grid=(8, 16, 16), cube=(8, 8, 4),
                                         n_text=24, D=256, hq=8, hkv=2, F=512, seed=31),
    # tubes: one spatial position over 64 frames
    "tube-1x1x64": workloads.small_config(name="tube", grid=(64, 4, 4), cube=(1, 1, 64),
                                          n_text=16, D=256, hq=4, hkv=2, F=512, seed=32),
    # patches: an 8x8 window of one frame
    "patch-8x8x1": workloads.small_config(name="patch", grid=(4, 16, 16), cube=(8, 8, 1),
                                          n_text=16, D=256, hq=4, hkv=1, F=512, seed=33),
    # 128-token cubes (the second cube shape of the 128K sweep), small
    "cube-8x8x2": workloads.small_config(name="c882", grid=(4, 16, 16), cube=(8, 8, 2),
                                         n_text=8, D=256, hq=8, hkv=2, F=512, seed=34),
}


@pytest.fixture(scope="module", params=list(SHAPES))
def shape_case(request):
    return parity.make_case(SHAPES[request.param])


@pytest.mark.parametrize("p", [0.7, 0.4])
def test_attn_cube_shapes(shape_case, p):
    rep = {}
    parity.check_attn(shape_case, p=p, report=rep)
    print(shape_case["cfg"].name, p, rep)


@pytest.mark.parametrize("p", [0.7, 0.4])
def test_ffn_cube_shapes(shape_case, p):
    rep = {}
    parity.check_ffn(shape_case, p=p, report=rep)
    print(shape_case["cfg"].name, p, rep)


# ------------------------------------------------------------------ device errors
def _attn_status(Q, K, V, ids, off, n_vis, p=0.7):
    out, ws = fb.cube_attn(Q, K, V, ids, off, n_vis, p)
    torch.cuda.synchronize()
    return fb.read_device_status(ws)


def _small_inputs(n_vis=256, n_text=8, hq=4, hkv=2, d=128, cube=64, scale=1.0, seed=5):
    g = torch.Generator(device="cpu").manual_seed(seed)
    N = n_vis + n_text
    Q = (scale * torch.randn(N, hq, d, generator=g)).to(torch.bfloat16).cuda()
    K = (scale * torch.randn(N, hkv, d, generator=g)).to(torch.bfloat16).cuda()
    V = torch.randn(N, hkv, d, generator=g).to(torch.bfloat16).cuda()
    C = n_vis // cube
    ids = torch.cat([torch.arange(C, dtype=torch.int32).repeat_interleave(cube),
                     torch.full((n_text,), -1, dtype=torch.int32)]).cuda()
    off = (torch.arange(C + 1, dtype=torch.int32) * cube).cuda()
    return Q, K, V, ids, off


def test_cube_larger_than_supported_is_flagged():
    """A 512-token cube exceeds the 256-token limit: BAD_LAYOUT, no selection."""
    Q, K, V, ids, off = _small_inputs(n_vis=1024, cube=512)
    code, detail = _attn_status(Q, K, V, ids, off, 1024)
    assert code == fb.EDEVICE and (detail & fb.DEV_BAD_LAYOUT)


def test_inconsistent_layout_is_flagged():
    """cube_ids that disagree with cube_offsets: BAD_LAYOUT."""
    Q, K, V, ids, off = _small_inputs()
    ids = ids.clone()
    ids[70] = 3          # token 70 lies in cube 1 by the offsets
    code, detail = _attn_status(Q, K, V, ids, off, 256)
    assert code == fb.EDEVICE and (detail & fb.DEV_BAD_LAYOUT)


def test_score_range_is_flagged_and_device_stays_usable():
    """Scores far beyond any attention logit (|q . kbar| / sqrt(d) ~ 1e7) cannot
    be binned by the selection: RANGE is reported instead of a wrong set, and a
    normal call afterwards succeeds."""
    Q, K, V, ids, off = _small_inputs(scale=1.0e4)
    code, detail = _attn_status(Q, K, V, ids, off, 256)
    assert code == fb.EDEVICE and (detail & fb.DEV_RANGE)
    Q, K, V, ids, off = _small_inputs(scale=1.0)
    code, detail = _attn_status(Q, K, V, ids, off, 256)
    assert code == fb.OK, (code, detail)


# AdaS-FFN feeds the down projection in fp16: values beyond its range must be
# reported, not silently saturated or turned into infinities.
_FFN_RANGE_CFG = workloads.small_config(name="ffn-range", grid=(4, 8, 8), cube=(4, 4, 4),
                                        n_text=16, D=256, hq=4, hkv=1, F=512, seed=61)


def _ffn_status(case, **weights):
    t = dict(case["t"], **weights)
    cfg = case["cfg"]
    y, ws = fb.token_ffn(t["x"], t["W_gate"], t["W_up"], t["W_down"], case["ids"], case["off"],
                         case["text"], cfg.n_vis, cfg.p)
    torch.cuda.synchronize()
    return fb.read_device_status(ws)


def test_ffn_activation_beyond_fp16_is_flagged_and_device_stays_usable():
    """Gate and up weights scaled 1000x make silu(g) * u reach ~1e5 > 65504: the
    fp16 store would saturate, so RANGE is reported (code 0x65xx); the same
    layer with its own weights then runs clean."""
    case = parity.make_case(_FFN_RANGE_CFG)
    t = case["t"]
    code, detail = _ffn_status(case, W_gate=(t["W_gate"].float() * 1000).to(torch.bfloat16),
                               W_up=(t["W_up"].float() * 1000).to(torch.bfloat16))
    assert code == fb.EDEVICE and (detail & fb.DEV_RANGE), (code, hex(detail))
    assert (detail >> 8) & 0xff00 == 0x6500, hex(detail)
    code, detail = _ffn_status(case)
    assert code == fb.OK, (code, hex(detail))


def test_ffn_wdown_beyond_fp16_is_flagged():
    """One W_down weight of 70144 (a bf16 value above the fp16 maximum 65504)
    would become infinite in the fp16 copy: RANGE is reported (code 0x66xx)."""
    case = parity.make_case(_FFN_RANGE_CFG)
    wd = case["t"]["W_down"].clone()
    wd[3, 7] = 70000.0
    assert float(wd[3, 7]) > 65504.0
    code, detail = _ffn_status(case, W_down=wd)
    assert code == fb.EDEVICE and (detail & fb.DEV_RANGE), (code, hex(detail))
    assert (detail >> 8) & 0xff00 == 0x6600, hex(detail)


def test_bounded_wait_expiry_reports_timeout_and_device_stays_usable():
    """Every wait inside the attention kernel is bounded. The test hook makes
    each tile withhold the announcement of its first key block and bounds the
    waits by 2e6 SM cycles (about a millisecond): the producer, the MMA issuer
    and the softmax warps wait for a descriptor that never comes, give up,
    report ADASPARK_DEV_TIMEOUT (a location code 0x7xxx of this kernel), free
    their tensor memory and return. A normal call afterwards on the same device
    succeeds and matches the oracle."""
    cfg = workloads.small_config(name="wait-expiry", grid=(4, 8, 8), cube=(4, 4, 4), n_text=16,
                                 D=256, hq=4, hkv=1, F=256, seed=62)
    case = parity.make_case(cfg)
    t = case["t"]
    fb.debug_wait_expiry(True, 2_000_000)
    try:
        _, ws = fb.cube_attn(t["Q"], t["K"], t["V"], case["ids"], case["off"], cfg.n_vis, cfg.p)
        torch.cuda.synchronize()
        code, detail = fb.read_device_status(ws)
    finally:
        fb.debug_wait_expiry(False)
    assert code == fb.EDEVICE and (detail & fb.DEV_TIMEOUT), (code, hex(detail))
    assert (detail >> 8) & 0xf000 == 0x7000, hex(detail)
    parity.check_attn(case)
