"""adaspark_cube_attn_noalloc: AdaS-Attn for callers that cannot allocate
device memory (plugins handed only their input/output buffers, loops that must
not allocate, processes whose device memory another allocator owns).

Checked through the C ABI against adaspark_cube_attn, which runs with a
caller-allocated workspace, on two calls in a row (different p, so state left
in the shared scratch array by the first call would show up in the second).
Both calls run the same deterministic kernels on the same inputs (the
allocation-free call always runs the single walk, so the workspace call runs
with the split walk turned off), so their outputs must agree bit for bit; the workspace call itself is checked against
the oracle (its selection sets, and its output on those sets), which pins the
allocation-free call to the oracle as well. This file sorts last so that a
stop-at-first-failure run has already run every other test."""
import ctypes

import pytest
import torch

import ffn_long_video_b200 as fb
import workloads
from tests import parity

pytestmark = pytest.mark.gpu

MAX_BYTES = 32 << 20   # ADASPARK_NOALLOC_SCRATCH_BYTES


def _noalloc_fn():
    fn = fb.lib().adaspark_cube_attn_noalloc
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    fn.restype = i32
    fn.argtypes = [vp, vp, vp, i32, vp, vp] + [i32] * 6 + [ctypes.c_float, vp, vp]
    return fn


def _call(fn, case, p, out):
    cfg, t = case["cfg"], case["t"]
    return fn(ctypes.c_void_p(t["Q"].data_ptr()), ctypes.c_void_p(t["K"].data_ptr()),
              ctypes.c_void_p(t["V"].data_ptr()), fb.BF16,
              ctypes.c_void_p(case["ids"].data_ptr()), ctypes.c_void_p(case["off"].data_ptr()),
              cfg.n_cubes, cfg.n_vis, cfg.n_tokens, cfg.hq, cfg.hkv, cfg.d, p,
              ctypes.c_void_p(out.data_ptr()),
              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_workspace_call_twice():
    cfg = workloads.small_config(name="noalloc", grid=(8, 8, 8), cube=(4, 4, 4), n_text=40,
                                 D=256, hq=8, hkv=2, F=256, seed=314)
    # the single walk's workspace (the common layout: the fp32 figure)
    assert fb.cube_attn_workspace_bytes(cfg.n_tokens, cfg.n_vis, cfg.n_cubes, cfg.hq, cfg.hkv,
                                        cfg.d, fb.FP32) <= MAX_BYTES
    case = parity.make_case(cfg)
    fn = _noalloc_fn()
    try:
        fb.set_split_rows(0)
        for p in (0.7, 0.4):
            # the workspace call, with its sets and output checked against the oracle
            want, _, _ = parity.check_attn(case, p)
            got = torch.full_like(want, float("nan"))
            assert _call(fn, case, p, got) == fb.OK
            torch.cuda.synchronize()
            assert torch.equal(got, want), p
    finally:
        fb.set_split_rows(fb.SPLIT_ROWS_DEFAULT)


def test_noalloc_rejects_sizes_beyond_its_array():
    cfg = workloads.CONFIGS[3]   # the 64K-token layer needs far more than the array holds
    need = fb.cube_attn_workspace_bytes(cfg.n_tokens, cfg.n_vis, cfg.n_cubes, cfg.hq, cfg.hkv,
                                        cfg.d, fb.FP32)
    assert need > MAX_BYTES
    fn = _noalloc_fn()
    dummy = ctypes.c_void_p(256)
    rc = fn(dummy, dummy, dummy, fb.BF16, dummy, dummy, cfg.n_cubes, cfg.n_vis, cfg.n_tokens,
            cfg.hq, cfg.hkv, cfg.d, 0.7, dummy, None)
    assert rc == fb.EINVAL
