"""The whole-layer call (projections on the library's tensor-core GEMM, AdaS-Attn,
output projection with the residual, AdaS-FFN) and RMSNorm against the float64
oracle, stage by stage on the library's own intermediates (needs a B200)."""
import numpy as np
import pytest
import torch

import ffn_long_video_b200 as fb
import oracle
import workloads
from tests import parity

pytestmark = pytest.mark.gpu

LAYERS = {
    "small": workloads.small_config(name="layer-small", grid=(4, 8, 8), cube=(4, 4, 2),
                                    n_text=40, D=256, hq=8, hkv=2, F=512, seed=41),
    # a ragged row count (not a multiple of the 128-row GEMM tile) and 3 KV heads
    "ragged": workloads.small_config(name="layer-ragged", grid=(4, 8, 8), cube=(4, 4, 4),
                                     n_text=23, D=384, hq=6, hkv=3, F=640, seed=42),
    # head_dim 64
    "d64": workloads.small_config(name="layer-d64", grid=(4, 8, 8), cube=(4, 4, 4),
                                  n_text=40, D=256, hq=8, hkv=2, d=64, F=512, seed=43),
}


def _bf16_close(got, want, what):
    """The bf16 output rule of the parity protocol: 2e-2, plus one bf16 ulp of
    the reference where |ref| >= 8; rel-L2 5e-3."""
    rel = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))
    worst = parity.excess_over_bf16(got, want)
    assert worst <= 2e-2 and rel <= 5e-3, (what, float(np.abs(got - want).max()), worst, rel)


@pytest.fixture(scope="module", params=list(LAYERS))
def layer_case(request):
    cfg = LAYERS[request.param]
    w = workloads.make_stack(cfg, 0)
    dev = "cuda"
    ids, off, text, off_np = parity.layout_tensors(cfg, dev)
    t = {k: v.to(dev) for k, v in w.items()}
    # [in, out] draws -> the [out, in] layout of the layer call
    Wt = {k: t[k].t().contiguous() for k in ("W_q", "W_k", "W_v", "W_o")}
    return {"cfg": cfg, "t": t, "Wt": Wt, "ids": ids, "off": off, "text": text, "off_np": off_np}


@pytest.mark.parametrize("p_attn,p_ffn", [(0.7, 0.7), (0.5, 0.9)])
def test_layer_stages(layer_case, p_attn, p_ffn):
    c = layer_case
    cfg, t, Wt = c["cfg"], c["t"], c["Wt"]
    y, ws = fb.layer(t["x"], Wt["W_q"], Wt["W_k"], Wt["W_v"], Wt["W_o"], t["W_gate"], t["W_up"],
                     t["W_down"], c["ids"], c["off"], c["text"], cfg.n_vis, cfg.hq, cfg.hkv,
                     p_attn, p_ffn)
    torch.cuda.synchronize()
    code, detail = fb.read_device_status(ws)
    assert code == fb.OK, (code, detail)
    buf = fb.layer_buffers(ws, cfg.n_tokens, cfg.n_vis, cfg.n_cubes, cfg.hq, cfg.hkv, cfg.d,
                           cfg.D, cfg.F)
    x = t["x"].cpu()
    # projections
    for name, W, heads in (("Q", Wt["W_q"], cfg.hq), ("K", Wt["W_k"], cfg.hkv),
                           ("V", Wt["W_v"], cfg.hkv)):
        want = oracle.linear(x, W.cpu())
        got = buf[name].float().cpu().numpy().reshape(cfg.n_tokens, heads * cfg.d)
        _bf16_close(got, want, name)
    # AdaS-Attn on the library's Q, K, V
    case = {"cfg": cfg, "t": {"Q": buf["Q"], "K": buf["K"], "V": buf["V"]}, "ids": c["ids"],
            "off": c["off"], "text": c["text"], "off_np": c["off_np"]}
    out, _, _ = parity.check_attn(case, p=p_attn)
    a = buf["a"]
    assert torch.equal(a, out)                 # the layer's attention = the standalone call
    # output projection with the residual, on the library's attention output
    want_h = x.double().numpy() + oracle.linear(a.reshape(cfg.n_tokens, -1).cpu(), Wt["W_o"].cpu())
    _bf16_close(buf["h"].float().cpu().numpy(), want_h, "h")
    # AdaS-FFN on the library's h
    case["t"] = {"x": buf["h"], "W_gate": t["W_gate"], "W_up": t["W_up"], "W_down": t["W_down"]}
    y2, act, _ = parity.check_ffn(case, p=p_ffn)
    # the layer's FFN = the standalone call: computed rows bit for bit; compensated
    # rows up to the order of the fp32 atomic sums behind the cube means
    act = torch.from_numpy(act).to(y.device)
    assert torch.equal(y[act], y2[act])
    assert torch.allclose(y[~act], y2[~act], rtol=1e-5, atol=1e-6)


def test_layer_rejects_fp32_and_bad_p(layer_case):
    c = layer_case
    cfg, t, Wt = c["cfg"], c["t"], c["Wt"]
    args = (t["x"], Wt["W_q"], Wt["W_k"], Wt["W_v"], Wt["W_o"], t["W_gate"], t["W_up"],
            t["W_down"], c["ids"], c["off"], c["text"], cfg.n_vis, cfg.hq, cfg.hkv)
    with pytest.raises(fb.AdasparkError):
        fb.layer(args[0].float(), *args[1:], 0.7, 0.7)
    with pytest.raises(fb.AdasparkError):
        fb.layer(*args, 0.0, 0.7)
    with pytest.raises(fb.AdasparkError):
        fb.layer(*args, 0.7, 1.5)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_rmsnorm(dtype):
    g = torch.Generator(device="cpu").manual_seed(3)
    x = (3.0 * torch.randn(37, 320, generator=g)).to(dtype).cuda()
    w = torch.randn(320, generator=g).to(torch.bfloat16).cuda()
    for weight in (None, w):
        got = fb.rmsnorm(x, weight, eps=1e-6).float().cpu().numpy()
        want = oracle.rmsnorm(x.cpu(), None if weight is None else weight.cpu(), 1e-6)
        _bf16_close(got, want, "rmsnorm")
