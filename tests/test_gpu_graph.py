"""The AdaS-Attn / AdaS-FFN forward and backward calls inside a CUDA graph
(needs a B200): no host synchronization or allocation happens inside the calls
once buffers and workspaces exist, so the whole step can be captured once and
replayed; the replay matches eager execution."""
import pytest
import torch

import ffn_long_video_b200 as fb
import workloads
from tests import parity

pytestmark = pytest.mark.gpu


def test_forward_backward_graph_replay_matches_eager():
    cfg = workloads.small_config(name="graph", grid=(8, 16, 16), cube=(4, 4, 4), n_text=72,
                                 D=512, hq=16, hkv=2, F=1024, seed=99)
    case = parity.make_case(cfg)
    t, ids, off, text = case["t"], case["ids"], case["off"], case["text"]
    up = workloads.make_upstream(cfg)
    dO, dy = up["dO"].cuda(), up["dy"].cuda()
    N, n_vis, C = cfg.n_tokens, cfg.n_vis, cfg.n_cubes
    dev = t["Q"].device
    out = torch.empty_like(t["Q"])
    y = torch.empty((N, cfg.D), dtype=torch.float32, device=dev)
    ws = lambda nb: torch.empty(nb, dtype=torch.uint8, device=dev)
    aws = ws(fb.cube_attn_workspace_bytes(N, n_vis, C, cfg.hq, cfg.hkv, cfg.d, fb.BF16))
    fws = ws(fb.token_ffn_workspace_bytes(N, n_vis, C, cfg.D, cfg.F, fb.BF16))
    abw = ws(fb.cube_attn_backward_workspace_bytes(N, n_vis, C, cfg.hq, cfg.hkv, cfg.d))
    fbw = ws(fb.token_ffn_backward_workspace_bytes(N, n_vis, C, cfg.D, cfg.F))
    f32 = dict(dtype=torch.float32, device=dev)
    g = {"dQ": torch.empty((N, cfg.hq, cfg.d), **f32), "dK": torch.empty((N, cfg.hkv, cfg.d), **f32),
         "dV": torch.empty((N, cfg.hkv, cfg.d), **f32), "dx": torch.empty((N, cfg.D), **f32),
         "dWg": torch.empty((cfg.F, cfg.D), **f32), "dWu": torch.empty((cfg.F, cfg.D), **f32),
         "dWd": torch.empty((cfg.D, cfg.F), **f32)}

    def step(stream):
        fb.cube_attn(t["Q"], t["K"], t["V"], ids, off, n_vis, cfg.p, out=out, workspace=aws,
                     stream=stream)
        fb.token_ffn(t["x"], t["W_gate"], t["W_up"], t["W_down"], ids, off, text, n_vis, cfg.p,
                     y=y, workspace=fws, stream=stream)
        fb.cube_attn_backward(t["Q"], t["K"], t["V"], dO, ids, off, n_vis, aws, dQ=g["dQ"],
                              dK=g["dK"], dV=g["dV"], workspace=abw, stream=stream)
        fb.token_ffn_backward(t["W_gate"], t["W_up"], t["W_down"], off, n_vis, dy, fws,
                              dx=g["dx"], dW_gate=g["dWg"], dW_up=g["dWu"], dW_down=g["dWd"],
                              workspace=fbw, stream=stream)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step(s)                                   # eager, warms up the library
    torch.cuda.synchronize()
    eager = {"out": out.clone(), "y": y.clone(), **{k: v.clone() for k, v in g.items()}}
    for w in (aws, fws, abw, fbw):
        assert fb.read_device_status(w)[0] == fb.OK
    act = torch.from_numpy(fb.ffn_export_active(fws, N, n_vis, C, cfg.D, cfg.F, fb.BF16)).to(dev)

    for v in (out, y, *g.values()):
        v.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        step(s)
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    for w in (aws, fws, abw, fbw):
        assert fb.read_device_status(w)[0] == fb.OK
    # deterministic results bit for bit; the FFN's compensated rows and the
    # weight gradients up to the order of their fp32 atomic cube sums
    assert torch.equal(out, eager["out"])
    for k in ("dQ", "dK", "dV"):
        assert torch.equal(g[k], eager[k]), k
    assert torch.equal(y[act], eager["y"][act])
    assert torch.allclose(y, eager["y"], rtol=1e-5, atol=1e-6)
    for k in ("dx", "dWg", "dWu", "dWd"):
        assert torch.allclose(g[k], eager[k], rtol=1e-4, atol=1e-5), k
