"""The C-ABI library without a GPU: it loads, exports every function that
include/adaspark.h declares, runs the host-only partition (checked against the
oracle), and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

import ffn_long_video_b200 as fb
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "adaspark.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(adaspark_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    L = fb.lib()
    names = _declared()
    assert len(names) >= 16
    for n in names:
        assert hasattr(L, n), n


@pytest.mark.parametrize("grid,cube,n_text", [
    ((8, 8, 8), (4, 4, 2), 32),
    ((5, 7, 3), (2, 3, 2), 3),
    ((64, 32, 32), (4, 4, 4), 256),
    ((3, 1, 1), (1, 1, 1), 0),
])
def test_partition_matches_oracle(grid, cube, n_text):
    T, H, W = grid
    ch, cw, ct = cube
    perm, ids, off = fb.cube_partition(T, H, W, ch, cw, ct, n_text)
    operm, oids, ooff, C = oracle.cube_partition(T, H, W, ch, cw, ct, n_text)
    assert np.array_equal(perm, operm)
    assert np.array_equal(ids, oids)
    assert np.array_equal(off, ooff)
    assert fb.cube_count(T, H, W, ch, cw, ct) == C


def test_partition_rejects_bad_sizes():
    P = ctypes.POINTER(ctypes.c_int32)
    buf = (ctypes.c_int32 * 16)()
    n = ctypes.c_int32(0)
    L = fb.lib()
    assert L.adaspark_cube_partition(0, 2, 2, 1, 1, 1, 0, buf, buf, buf, ctypes.byref(n)) == fb.EINVAL
    assert L.adaspark_cube_partition(2, 2, 2, 1, 1, 1, -1, buf, buf, buf, ctypes.byref(n)) == fb.EINVAL
    assert L.adaspark_cube_partition(2, 2, 2, 1, 1, 1, 0, None, buf, buf, ctypes.byref(n)) == fb.EINVAL
    assert L.adaspark_cube_count(2, 2, 2, 0, 1, 1, ctypes.byref(n)) == fb.EINVAL


def test_workspace_queries():
    assert fb.cube_attn_workspace_bytes(65792, 65536, 1024, 28, 4, 128, fb.BF16) > 0
    assert fb.cube_attn_workspace_bytes(544, 512, 16, 4, 1, 64, fb.FP32) > 0
    assert fb.cube_attn_workspace_bytes(544, 512, 16, 5, 2, 64, fb.FP32) == 0   # hq % hkv
    assert fb.cube_attn_workspace_bytes(544, 512, 16, 4, 1, 64, fb.BF16) > 0    # bf16, d = 64
    assert fb.cube_attn_workspace_bytes(544, 512, 16, 4, 1, 96, fb.BF16) == 0   # d in {64, 128}
    # the backward is built for d = 128 only
    assert fb.cube_attn_backward_workspace_bytes(544, 512, 16, 4, 1, 64) == 0
    assert fb.cube_attn_workspace_bytes(544, 600, 16, 4, 1, 64, fb.FP32) == 0   # n_vis > n_tokens
    assert fb.token_ffn_workspace_bytes(65792, 65536, 1024, 3584, 18944, fb.BF16) > 0
    assert fb.token_ffn_workspace_bytes(544, 512, 16, 250, 512, fb.FP32) == 0


def test_calls_reject_bad_arguments_before_the_device():
    L = fb.lib()
    dummy = ctypes.c_void_p(256)
    ws_bytes = fb.cube_attn_workspace_bytes(544, 512, 16, 4, 1, 64, fb.FP32)
    args = [dummy, dummy, dummy, fb.FP32, dummy, dummy, 16, 512, 544, 4, 1, 64]
    for p in (0.0, -0.5, 1.5, float("nan")):
        assert L.adaspark_cube_attn(*args, p, dummy, dummy, ws_bytes, None) == fb.EINVAL
    assert L.adaspark_cube_attn(*args, 0.7, dummy, dummy, ws_bytes - 1, None) == fb.EINVAL
    assert L.adaspark_cube_attn(*args, 0.7, None, dummy, ws_bytes, None) == fb.EINVAL
    assert L.adaspark_cube_attn(*args, 0.7, dummy, ctypes.c_void_p(257), ws_bytes, None) == fb.EINVAL
    for k in (0, -3):
        assert L.adaspark_cube_attn_topk(*args, k, dummy, dummy, ws_bytes, None) == fb.EINVAL
    assert L.adaspark_cube_attn_topk(*args, 4, dummy, dummy, ws_bytes - 1, None) == fb.EINVAL
    for k in (0, -3):
        assert L.adaspark_cube_attn_uniform(*args, k, dummy, dummy, ws_bytes, None) == fb.EINVAL
    assert L.adaspark_cube_attn_uniform(*args, 4, dummy, dummy, ws_bytes - 1, None) == fb.EINVAL
    # the wait-expiry test hook takes bounds of 1e5 .. 2e9 cycles; off is always accepted
    for cycles in (0, 99_999, 2_000_000_001):
        assert L.adaspark_debug_wait_expiry(1, cycles) == fb.EINVAL
    assert L.adaspark_debug_wait_expiry(0, 0) == fb.OK
    fws = fb.token_ffn_workspace_bytes(544, 512, 16, 256, 512, fb.FP32)
    fargs = [dummy] * 4 + [fb.FP32, dummy, dummy, dummy, 16, 512, 544, 256, 512]
    assert L.adaspark_token_ffn(*fargs, 2.0, dummy, dummy, fws, None) == fb.EINVAL
    assert L.adaspark_token_ffn(*fargs, 0.7, dummy, dummy, fws - 8, None) == fb.EINVAL
    for code in (-1, 3):
        assert L.adaspark_token_ffn_ex(*fargs, 0.7, code, dummy, dummy, fws, None) == fb.EINVAL
    assert fb.status_string(fb.EDEVICE) == "device-side check failed"


def test_backward_layer_and_train_calls_reject_bad_arguments_before_the_device():
    L = fb.lib()
    d = ctypes.c_void_p(256)
    # the attention backward is built for head_dim 128: bf16 with d = 64 is
    # refused before any device work
    assert L.adaspark_cube_attn_backward(d, d, d, d, fb.BF16, d, d, 16, 512, 544, 4, 1, 64, d, d,
                                         d, d, d, 1 << 30, None) == fb.EUNSUPPORTED
    # workspace queries: bf16 only for the backward and the training forward
    assert fb.cube_attn_backward_workspace_bytes(65792, 65536, 1024, 28, 4, 128) > 0
    assert fb.cube_attn_backward_workspace_bytes(544, 512, 16, 4, 1, 64, fb.FP32) == 0
    assert fb.token_ffn_backward_workspace_bytes(65792, 65536, 1024, 3584, 18944) > 0
    assert fb.token_ffn_backward_workspace_bytes(544, 512, 16, 256, 512, fb.FP32) == 0
    # the common layout (the fp32 figure) plus the fp32 output of a training call;
    # the bf16 inference figure adds the split walk's region instead
    common = fb.cube_attn_workspace_bytes(65792, 65536, 1024, 28, 4, 128, fb.FP32)
    inf = fb.cube_attn_workspace_bytes(65792, 65536, 1024, 28, 4, 128, fb.BF16)
    assert fb.cube_attn_train_workspace_bytes(65792, 65536, 1024, 28, 4, 128) == \
        common + 65792 * 28 * 128 * 4
    assert inf > common
    # the split walk's threshold: 0 .. 128 rows
    assert L.adaspark_set_split_rows(-1) == fb.EINVAL
    assert L.adaspark_set_split_rows(129) == fb.EINVAL
    assert L.adaspark_set_split_rows(0) == fb.OK
    assert L.adaspark_set_split_rows(fb.SPLIT_ROWS_DEFAULT) == fb.OK
    # attention backward: fp32 unsupported, bad sizes / pointers / workspace rejected
    ab = fb.cube_attn_backward_workspace_bytes(544, 512, 16, 4, 1, 128)
    aargs = [d] * 4
    geo = [d, d, 16, 512, 544, 4, 1, 128]
    assert L.adaspark_cube_attn_backward(*aargs, fb.FP32, *geo, d, d, d, d, d, ab, None) == \
        fb.EUNSUPPORTED
    assert L.adaspark_cube_attn_backward(*aargs, fb.BF16, *geo, d, d, d, d, d, ab - 1, None) == \
        fb.EINVAL
    assert L.adaspark_cube_attn_backward(*aargs, fb.BF16, *geo, None, d, d, d, d, ab, None) == \
        fb.EINVAL
    assert L.adaspark_cube_attn_backward(*aargs, fb.BF16, d, d, 16, 512, 544, 5, 2, 128, d, d, d,
                                         d, d, ab, None) == fb.EINVAL                 # hq % hkv
    # training forward: fp32 unsupported, too small a workspace rejected
    tw = fb.cube_attn_train_workspace_bytes(544, 512, 16, 4, 1, 128)
    targs = [d, d, d, fb.BF16, d, d, 16, 512, 544, 4, 1, 128, 0.7, d, d]
    assert L.adaspark_cube_attn_train(*targs, tw - 1, None) == fb.EINVAL
    targs[3] = fb.FP32
    assert L.adaspark_cube_attn_train(*targs, tw, None) == fb.EUNSUPPORTED
    # FFN backward
    fb_ws = fb.token_ffn_backward_workspace_bytes(544, 512, 16, 256, 512)
    fargs = [d, d, d]
    fgeo = [d, 16, 512, 544, 256, 512]
    assert L.adaspark_token_ffn_backward(*fargs, fb.FP32, *fgeo, d, d, d, d, d, d, d, fb_ws,
                                         None) == fb.EUNSUPPORTED
    assert L.adaspark_token_ffn_backward(*fargs, fb.BF16, *fgeo, d, d, d, d, d, d, d, fb_ws - 8,
                                         None) == fb.EINVAL
    assert L.adaspark_token_ffn_backward(*fargs, fb.BF16, *fgeo, None, d, d, d, d, d, d, fb_ws,
                                         None) == fb.EINVAL
    assert L.adaspark_token_ffn_backward(*fargs, fb.BF16, d, 16, 512, 544, 250, 512, d, d, d, d, d,
                                         d, d, fb_ws, None) == fb.EINVAL                # D % 64
    # layer: fp32 unsupported, bad p rejected; RMSNorm: bad sizes rejected
    lw = fb.layer_workspace_bytes(544, 512, 16, 4, 1, 128, 256, 512)
    assert lw > 0
    largs = [d] * 8
    lgeo = [d, d, d, 16, 512, 544, 4, 1, 128, 256, 512]
    assert L.adaspark_layer(*largs, fb.FP32, *lgeo, 0.7, 0.7, d, d, lw, None) == fb.EUNSUPPORTED
    for pa, pf in ((0.0, 0.7), (0.7, 1.5)):
        assert L.adaspark_layer(*largs, fb.BF16, *lgeo, pa, pf, d, d, lw, None) == fb.EINVAL
    assert L.adaspark_layer(*largs, fb.BF16, *lgeo, 0.7, 0.7, d, d, lw - 1, None) == fb.EINVAL
    assert L.adaspark_rmsnorm(d, fb.BF16, None, d, 4, 0, 1e-6, None) == fb.EINVAL
    assert L.adaspark_rmsnorm(d, 7, None, d, 4, 64, 1e-6, None) == fb.EINVAL
