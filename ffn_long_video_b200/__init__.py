"""Python binding of libadaspark.so, the AdaSpark layer hot path for B200.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Torch tensors supply device memory and the current CUDA stream.  The
binding fails loudly when the library is missing; there is no fallback.

Entry points (same names as include/adaspark.h, without the prefix):
``cube_count``, ``cube_partition``, ``cube_attn`` (and ``_train``), ``cube_attn_topk``,
``cube_attn_backward``,
``attn_export_sets``,
``attn_read_stats``, ``token_ffn``, ``token_ffn_backward``, ``ffn_export_active``,
``ffn_read_stats``,
``layer``, ``layer_buffers``, ``rmsnorm``,
``read_device_status``, ``timer_enable``, ``timer_read``, ``launch_count``,
``device_check``, ``status_string``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libadaspark.so")

OK, EINVAL, ECUDA, EUNSUPPORTED, EDEVICE = 0, -1, -2, -3, -4
BF16, FP32 = 0, 1
DEV_BAD_LAYOUT, DEV_TIMEOUT, DEV_RANGE = 0x1, 0x2, 0x4
# AdaS-FFN token importance (ADASPARK_IMPORTANCE_*)
IMPORTANCE_L2_SHARE, IMPORTANCE_L2SQ_SHARE, IMPORTANCE_SOFTMAX = 0, 1, 2


class AdasparkError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)} ({code})")
        self.code = code


class _AttnStats(ctypes.Structure):
    _fields_ = [("visual_rows", ctypes.c_uint64), ("candidate_pairs", ctypes.c_uint64),
                ("selected_pairs", ctypes.c_uint64), ("overflow_rows", ctypes.c_uint64),
                ("tiles", ctypes.c_uint64), ("key_blocks", ctypes.c_uint64),
                ("key_block_keys", ctypes.c_uint64), ("near_margin_rows", ctypes.c_uint64),
                ("split_pairs", ctypes.c_uint64), ("gathered_blocks", ctypes.c_uint64),
                ("reserved", ctypes.c_uint64 * 6)]


class _FfnStats(ctypes.Structure):
    _fields_ = [("active_visual", ctypes.c_uint64), ("skipped_visual", ctypes.c_uint64),
                ("text_tokens", ctypes.c_uint64), ("near_margin_cubes", ctypes.c_uint64),
                ("reserved", ctypes.c_uint64 * 12)]


class _KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_uint64),
                ("total_ms", ctypes.c_double)]


_lib = None


def lib():
    """The loaded ctypes library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(
                f"{_LIB_PATH} is missing: build it with `python -m ffn_long_video_b200._build` "
                "(there is no fallback path)")
        L = ctypes.CDLL(_LIB_PATH)
        vp, i32, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
        i32p = ctypes.POINTER(ctypes.c_int32)
        sigs = {
            "adaspark_status_string": (ctypes.c_char_p, [i32]),
            "adaspark_cube_count": (i32, [i32] * 6 + [i32p]),
            "adaspark_cube_partition": (i32, [i32] * 7 + [i32p] * 4),
            "adaspark_cube_attn_workspace": (sz, [i32] * 7),
            "adaspark_cube_attn": (i32, [vp, vp, vp, i32, vp, vp] + [i32] * 6 + [f32, vp, vp, sz,
                                                                                   vp]),
            "adaspark_cube_attn_topk": (i32, [vp, vp, vp, i32, vp, vp] + [i32] * 7 + [vp, vp, sz,
                                                                                    vp]),
            "adaspark_cube_attn_uniform": (i32, [vp, vp, vp, i32, vp, vp] + [i32] * 7 +
                                           [vp, vp, sz, vp]),
            "adaspark_cube_attn_train_workspace": (sz, [i32] * 7),
            "adaspark_cube_attn_train": (i32, [vp, vp, vp, i32, vp, vp] + [i32] * 6 + [f32, vp, vp,
                                                                                   sz, vp]),
            "adaspark_cube_attn_backward_workspace": (sz, [i32] * 7),
            "adaspark_cube_attn_backward": (i32, [vp] * 4 + [i32, vp, vp] + [i32] * 6 +
                                            [vp] * 5 + [sz, vp]),
            "adaspark_attn_export_sets": (i32, [vp, vp] + [i32] * 7 + [vp, vp]),
            "adaspark_attn_read_stats": (i32, [vp, ctypes.POINTER(_AttnStats), vp]),
            "adaspark_token_ffn_workspace": (sz, [i32] * 6),
            "adaspark_token_ffn": (i32, [vp, vp, vp, vp, i32, vp, vp, vp] + [i32] * 5 +
                                   [f32, vp, vp, sz, vp]),
            "adaspark_token_ffn_ex": (i32, [vp, vp, vp, vp, i32, vp, vp, vp] + [i32] * 5 +
                                      [f32, i32, vp, vp, sz, vp]),
            "adaspark_token_ffn_backward_workspace": (sz, [i32] * 6),
            "adaspark_token_ffn_backward": (i32, [vp, vp, vp, i32, vp] + [i32] * 5 +
                                            [vp] * 7 + [sz, vp]),
            "adaspark_layer_workspace": (sz, [i32] * 9),
            "adaspark_layer_buffers": (i32, [i32] * 9 + [ctypes.POINTER(ctypes.c_size_t)]),
            "adaspark_layer": (i32, [vp] * 8 + [i32, vp, vp, vp] + [i32] * 8 +
                               [f32, f32, vp, vp, sz, vp]),
            "adaspark_rmsnorm": (i32, [vp, i32, vp, vp, i32, i32, f32, vp]),
            "adaspark_ffn_export_active": (i32, [vp] + [i32] * 6 + [vp, vp]),
            "adaspark_ffn_read_stats": (i32, [vp, ctypes.POINTER(_FfnStats), vp]),
            "adaspark_read_device_status": (i32, [vp, ctypes.POINTER(ctypes.c_uint32), vp]),
            "adaspark_timer_enable": (i32, [i32]),
            "adaspark_timer_read": (i32, [ctypes.POINTER(_KernelTime), i32, ctypes.POINTER(i32)]),
            "adaspark_launch_count": (ctypes.c_uint64, []),
            "adaspark_device_check": (i32, [i32]),
            "adaspark_debug_wait_expiry": (i32, [i32, ctypes.c_longlong]),
            "adaspark_set_split_rows": (i32, [i32]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().adaspark_status_string(code).decode()


def _check(code: int, what: str):
    if code != OK:
        raise AdasparkError(code, what)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, device=True):
    if t is None:
        raise ValueError(f"{name} is required")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# ----------------------------------------------------------------- partition
def cube_count(T, H, W, cube_h, cube_w, cube_t) -> int:
    n = ctypes.c_int32(0)
    _check(lib().adaspark_cube_count(T, H, W, cube_h, cube_w, cube_t, ctypes.byref(n)),
           "adaspark_cube_count")
    return n.value


def cube_partition(T, H, W, cube_h, cube_w, cube_t, n_text):
    """Host call: returns (perm, cube_ids, cube_offsets) as int32 numpy arrays."""
    C = cube_count(T, H, W, cube_h, cube_w, cube_t)
    n_vis = T * H * W
    perm = np.empty(n_vis, np.int32)
    ids = np.empty(n_vis + n_text, np.int32)
    off = np.empty(C + 1, np.int32)
    n = ctypes.c_int32(0)
    P = ctypes.POINTER(ctypes.c_int32)
    _check(lib().adaspark_cube_partition(T, H, W, cube_h, cube_w, cube_t, n_text,
                                         perm.ctypes.data_as(P), ids.ctypes.data_as(P),
                                         off.ctypes.data_as(P), ctypes.byref(n)),
           "adaspark_cube_partition")
    assert n.value == C
    return perm, ids, off


# ----------------------------------------------------------------- AdaS-Attn
def cube_attn_workspace_bytes(n_tokens, n_vis, n_cubes, hq, hkv, d, dtype) -> int:
    return int(lib().adaspark_cube_attn_workspace(n_tokens, n_vis, n_cubes, hq, hkv, d, dtype))


def cube_attn(Q, K, V, cube_ids, cube_offsets, n_vis, p, out=None, workspace=None, stream=None,
              train=False):
    """AdaS-Attn on device tensors; returns (out, workspace). ``train`` runs
    adaspark_cube_attn_train (the workspace then also keeps the fp32 output
    that makes the backward pass a single walk over the keys)."""
    import torch
    for t, nm in ((Q, "Q"), (K, "K"), (V, "V"), (cube_ids, "cube_ids"),
                  (cube_offsets, "cube_offsets")):
        _need(t, nm)
    N, hq, d = Q.shape
    hkv = K.shape[1]
    C = cube_offsets.numel() - 1
    dt = _dtype_code(Q)
    if out is None:
        out = torch.empty_like(Q)
    if workspace is None:
        nb = (cube_attn_train_workspace_bytes if train else cube_attn_workspace_bytes)(
            N, n_vis, C, hq, hkv, d, dt)
        if nb == 0:
            raise AdasparkError(EUNSUPPORTED if train and dt == FP32 else EINVAL,
                                "adaspark_cube_attn_workspace")
        workspace = torch.empty(nb, dtype=torch.uint8, device=Q.device)
    fn = lib().adaspark_cube_attn_train if train else lib().adaspark_cube_attn
    _check(fn(_ptr(Q), _ptr(K), _ptr(V), dt, _ptr(cube_ids), _ptr(cube_offsets), C, n_vis, N, hq,
              hkv, d, float(p), _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream)),
           "adaspark_cube_attn_train" if train else "adaspark_cube_attn")
    return out, workspace


def cube_attn_train_workspace_bytes(n_tokens, n_vis, n_cubes, hq, hkv, d, dtype=BF16) -> int:
    return int(lib().adaspark_cube_attn_train_workspace(n_tokens, n_vis, n_cubes, hq, hkv, d,
                                                         dtype))


def cube_attn_topk(Q, K, V, cube_ids, cube_offsets, n_vis, k, out=None, workspace=None,
                   stream=None):
    """AdaS-Attn with Top-K selection (the k most probable preceding cubes);
    returns (out, workspace)."""
    import torch
    for t, nm in ((Q, "Q"), (K, "K"), (V, "V"), (cube_ids, "cube_ids"),
                  (cube_offsets, "cube_offsets")):
        _need(t, nm)
    N, hq, d = Q.shape
    hkv = K.shape[1]
    C = cube_offsets.numel() - 1
    dt = _dtype_code(Q)
    if out is None:
        out = torch.empty_like(Q)
    if workspace is None:
        nb = cube_attn_workspace_bytes(N, n_vis, C, hq, hkv, d, dt)
        if nb == 0:
            raise AdasparkError(EINVAL, "adaspark_cube_attn_workspace")
        workspace = torch.empty(nb, dtype=torch.uint8, device=Q.device)
    _check(lib().adaspark_cube_attn_topk(_ptr(Q), _ptr(K), _ptr(V), dt, _ptr(cube_ids),
                                         _ptr(cube_offsets), C, n_vis, N, hq, hkv, d, int(k),
                                         _ptr(out), _ptr(workspace), workspace.numel(),
                                         _stream(stream)),
           "adaspark_cube_attn_topk")
    return out, workspace


def cube_attn_uniform(Q, K, V, cube_ids, cube_offsets, n_vis, k, out=None, workspace=None,
                      stream=None):
    """AdaS-Attn with Uniform Sampling (k evenly spaced preceding cubes);
    returns (out, workspace)."""
    import torch
    for t, nm in ((Q, "Q"), (K, "K"), (V, "V"), (cube_ids, "cube_ids"),
                  (cube_offsets, "cube_offsets")):
        _need(t, nm)
    N, hq, d = Q.shape
    hkv = K.shape[1]
    C = cube_offsets.numel() - 1
    dt = _dtype_code(Q)
    if out is None:
        out = torch.empty_like(Q)
    if workspace is None:
        nb = cube_attn_workspace_bytes(N, n_vis, C, hq, hkv, d, dt)
        if nb == 0:
            raise AdasparkError(EINVAL, "adaspark_cube_attn_workspace")
        workspace = torch.empty(nb, dtype=torch.uint8, device=Q.device)
    _check(lib().adaspark_cube_attn_uniform(_ptr(Q), _ptr(K), _ptr(V), dt, _ptr(cube_ids),
                                            _ptr(cube_offsets), C, n_vis, N, hq, hkv, d, int(k),
                                            _ptr(out), _ptr(workspace), workspace.numel(),
                                            _stream(stream)),
           "adaspark_cube_attn_uniform")
    return out, workspace


def attn_export_sets(workspace, cube_ids, n_cubes, n_vis, n_tokens, hq, hkv, d, dtype,
                     stream=None):
    """Selected sets of the last cube_attn call as a bool tensor [n_vis, hq, C] (host)."""
    import torch
    W = (n_cubes + 31) // 32
    bits = torch.zeros(max(n_vis, 1) * hq * W, dtype=torch.int32, device=workspace.device)
    _check(lib().adaspark_attn_export_sets(_ptr(workspace), _ptr(cube_ids), n_cubes, n_vis,
                                           n_tokens, hq, hkv, d, dtype, _ptr(bits),
                                           _stream(stream)),
           "adaspark_attn_export_sets")
    b = bits.cpu().numpy().view(np.uint32)[: n_vis * hq * W].reshape(n_vis, hq, W)
    unpacked = np.unpackbits(b.view(np.uint8).reshape(n_vis, hq, W * 4), axis=-1,
                             bitorder="little")
    return unpacked[:, :, :n_cubes].astype(bool)


def attn_export_bits(workspace, cube_ids, n_cubes, n_vis, n_tokens, hq, hkv, d, dtype,
                     stream=None):
    """Selected sets of the last cube_attn call as packed bits on the device:
    int32 [n_vis, hq, ceil(C/32)], bit j of row (t, h) set when cube j is in
    its set (the own cube is not marked)."""
    import torch
    W = (n_cubes + 31) // 32
    bits = torch.zeros(max(n_vis, 1) * hq * W, dtype=torch.int32, device=workspace.device)
    _check(lib().adaspark_attn_export_sets(_ptr(workspace), _ptr(cube_ids), n_cubes, n_vis,
                                           n_tokens, hq, hkv, d, dtype, _ptr(bits),
                                           _stream(stream)),
           "adaspark_attn_export_sets")
    return bits[: n_vis * hq * W].view(n_vis, hq, W)


def attn_read_stats(workspace, stream=None) -> dict:
    st = _AttnStats()
    _check(lib().adaspark_attn_read_stats(_ptr(workspace), ctypes.byref(st), _stream(stream)),
           "adaspark_attn_read_stats")
    return {k: getattr(st, k) for k, _ in _AttnStats._fields_ if k != "reserved"}


# ----------------------------------------------------------------- AdaS-FFN
def token_ffn_workspace_bytes(n_tokens, n_vis, n_cubes, D, F, dtype) -> int:
    return int(lib().adaspark_token_ffn_workspace(n_tokens, n_vis, n_cubes, D, F, dtype))


def token_ffn(x, W_gate, W_up, W_down, cube_ids, cube_offsets, text_mask, n_vis, p, y=None,
              workspace=None, stream=None, importance=IMPORTANCE_L2_SHARE):
    """AdaS-FFN on device tensors; returns (y fp32 [N, D], workspace).
    ``importance`` other than the linear L2 share calls adaspark_token_ffn_ex."""
    import torch
    for t, nm in ((x, "x"), (W_gate, "W_gate"), (W_up, "W_up"), (W_down, "W_down"),
                  (cube_ids, "cube_ids"), (cube_offsets, "cube_offsets"),
                  (text_mask, "text_mask")):
        _need(t, nm)
    N, D = x.shape
    F = W_gate.shape[0]
    C = cube_offsets.numel() - 1
    dt = _dtype_code(x)
    if y is None:
        y = torch.empty((N, D), dtype=torch.float32, device=x.device)
    if workspace is None:
        nb = token_ffn_workspace_bytes(N, n_vis, C, D, F, dt)
        if nb == 0:
            raise AdasparkError(EINVAL, "adaspark_token_ffn_workspace")
        workspace = torch.empty(nb, dtype=torch.uint8, device=x.device)
    if importance == IMPORTANCE_L2_SHARE:
        _check(lib().adaspark_token_ffn(_ptr(x), _ptr(W_gate), _ptr(W_up), _ptr(W_down), dt,
                                        _ptr(cube_ids), _ptr(cube_offsets), _ptr(text_mask), C,
                                        n_vis, N, D, F, float(p), _ptr(y), _ptr(workspace),
                                        workspace.numel(), _stream(stream)),
               "adaspark_token_ffn")
    else:
        _check(lib().adaspark_token_ffn_ex(_ptr(x), _ptr(W_gate), _ptr(W_up), _ptr(W_down), dt,
                                           _ptr(cube_ids), _ptr(cube_offsets), _ptr(text_mask), C,
                                           n_vis, N, D, F, float(p), int(importance), _ptr(y),
                                           _ptr(workspace), workspace.numel(), _stream(stream)),
               "adaspark_token_ffn_ex")
    return y, workspace


def cube_attn_backward_workspace_bytes(n_tokens, n_vis, n_cubes, hq, hkv, d, dtype=BF16) -> int:
    return int(lib().adaspark_cube_attn_backward_workspace(n_tokens, n_vis, n_cubes, hq, hkv, d,
                                                            dtype))


def cube_attn_backward(Q, K, V, dO, cube_ids, cube_offsets, n_vis, fwd_workspace, dQ=None,
                       dK=None, dV=None, workspace=None, stream=None):
    """Backward of AdaS-Attn with the sets of the forward call that filled
    ``fwd_workspace`` held fixed. Returns (dQ, dK, dV, workspace), fp32
    (allocated when not given)."""
    import torch
    for t, nm in ((Q, "Q"), (K, "K"), (V, "V"), (dO, "dO"),
                  (cube_ids, "cube_ids"), (cube_offsets, "cube_offsets"),
                  (fwd_workspace, "fwd_workspace")):
        _need(t, nm)
    N, hq, d = Q.shape
    hkv = K.shape[1]
    C = cube_offsets.numel() - 1
    dt = _dtype_code(Q)
    f32 = torch.float32
    dQ = torch.empty((N, hq, d), dtype=f32, device=Q.device) if dQ is None else dQ
    dK = torch.empty((N, hkv, d), dtype=f32, device=Q.device) if dK is None else dK
    dV = torch.empty((N, hkv, d), dtype=f32, device=Q.device) if dV is None else dV
    if workspace is None:
        nb = cube_attn_backward_workspace_bytes(N, n_vis, C, hq, hkv, d, dt)
        if nb == 0:
            raise AdasparkError(EUNSUPPORTED if dt == FP32 else EINVAL,
                                "adaspark_cube_attn_backward_workspace")
        workspace = torch.empty(nb, dtype=torch.uint8, device=Q.device)
    _check(lib().adaspark_cube_attn_backward(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(dO), dt, _ptr(cube_ids), _ptr(cube_offsets), C,
        n_vis, N, hq, hkv, d, _ptr(fwd_workspace), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(workspace),
        workspace.numel(), _stream(stream)), "adaspark_cube_attn_backward")
    return dQ, dK, dV, workspace


def token_ffn_backward_workspace_bytes(n_tokens, n_vis, n_cubes, D, F, dtype=BF16) -> int:
    return int(lib().adaspark_token_ffn_backward_workspace(n_tokens, n_vis, n_cubes, D, F, dtype))


def token_ffn_backward(W_gate, W_up, W_down, cube_offsets, n_vis, dy, fwd_workspace, dx=None,
                       dW_gate=None, dW_up=None, dW_down=None, workspace=None, stream=None):
    """Backward of AdaS-FFN with the active set of the forward call that filled
    ``fwd_workspace`` held fixed. Returns (dx, dW_gate, dW_up, dW_down, workspace),
    all fp32 (allocated when not given)."""
    import torch
    for t, nm in ((W_gate, "W_gate"), (W_up, "W_up"), (W_down, "W_down"),
                  (cube_offsets, "cube_offsets"), (dy, "dy"), (fwd_workspace, "fwd_workspace")):
        _need(t, nm)
    N, D = dy.shape
    F = W_gate.shape[0]
    C = cube_offsets.numel() - 1
    dt = _dtype_code(W_gate)
    dev = dy.device
    f32 = torch.float32
    dx = torch.empty((N, D), dtype=f32, device=dev) if dx is None else dx
    dW_gate = torch.empty((F, D), dtype=f32, device=dev) if dW_gate is None else dW_gate
    dW_up = torch.empty((F, D), dtype=f32, device=dev) if dW_up is None else dW_up
    dW_down = torch.empty((D, F), dtype=f32, device=dev) if dW_down is None else dW_down
    if workspace is None:
        nb = token_ffn_backward_workspace_bytes(N, n_vis, C, D, F, dt)
        if nb == 0:
            raise AdasparkError(EUNSUPPORTED if dt == FP32 else EINVAL,
                                "adaspark_token_ffn_backward_workspace")
        workspace = torch.empty(nb, dtype=torch.uint8, device=dev)
    _check(lib().adaspark_token_ffn_backward(
        _ptr(W_gate), _ptr(W_up), _ptr(W_down), dt, _ptr(cube_offsets), C, n_vis, N, D, F,
        _ptr(dy), _ptr(fwd_workspace), _ptr(dx), _ptr(dW_gate), _ptr(dW_up), _ptr(dW_down),
        _ptr(workspace), workspace.numel(), _stream(stream)), "adaspark_token_ffn_backward")
    return dx, dW_gate, dW_up, dW_down, workspace


def layer_workspace_bytes(n_tokens, n_vis, n_cubes, hq, hkv, d, D, F, dtype=BF16) -> int:
    return int(lib().adaspark_layer_workspace(n_tokens, n_vis, n_cubes, hq, hkv, d, D, F, dtype))


def layer(x, W_q, W_k, W_v, W_o, W_gate, W_up, W_down, cube_ids, cube_offsets, text_mask, n_vis,
          hq, hkv, p_attn, p_ffn, y=None, workspace=None, stream=None):
    """A whole AdaSpark layer (projections, AdaS-Attn, output projection with the
    residual, AdaS-FFN); weights in [out, in] layout. Returns (y fp32, workspace)."""
    import torch
    for t, nm in ((x, "x"), (W_q, "W_q"), (W_k, "W_k"), (W_v, "W_v"), (W_o, "W_o"),
                  (W_gate, "W_gate"), (W_up, "W_up"), (W_down, "W_down"),
                  (cube_ids, "cube_ids"), (cube_offsets, "cube_offsets"),
                  (text_mask, "text_mask")):
        _need(t, nm)
    N, D = x.shape
    d = W_q.shape[0] // hq
    F = W_gate.shape[0]
    C = cube_offsets.numel() - 1
    dt = _dtype_code(x)
    if y is None:
        y = torch.empty((N, D), dtype=torch.float32, device=x.device)
    if workspace is None:
        nb = layer_workspace_bytes(N, n_vis, C, hq, hkv, d, D, F, dt)
        if nb == 0:
            raise AdasparkError(EINVAL, "adaspark_layer_workspace")
        workspace = torch.empty(nb, dtype=torch.uint8, device=x.device)
    _check(lib().adaspark_layer(_ptr(x), _ptr(W_q), _ptr(W_k), _ptr(W_v), _ptr(W_o),
                                _ptr(W_gate), _ptr(W_up), _ptr(W_down), dt, _ptr(cube_ids),
                                _ptr(cube_offsets), _ptr(text_mask), C, n_vis, N, hq, hkv, d, D, F,
                                float(p_attn), float(p_ffn), _ptr(y), _ptr(workspace),
                                workspace.numel(), _stream(stream)),
           "adaspark_layer")
    return y, workspace


def layer_buffers(workspace, n_tokens, n_vis, n_cubes, hq, hkv, d, D, F):
    """Views of a layer workspace's intermediates: Q, K, V, a (attention output),
    h (bf16 tensors) and the AdaS-Attn / AdaS-FFN sub-workspaces (uint8)."""
    import torch
    off = (ctypes.c_size_t * 7)()
    _check(lib().adaspark_layer_buffers(n_tokens, n_vis, n_cubes, hq, hkv, d, D, F, BF16, off),
           "adaspark_layer_buffers")
    N = n_tokens

    def view(o, count, shape):
        return workspace[o:o + 2 * count].view(torch.bfloat16).view(*shape)

    attn_b = cube_attn_workspace_bytes(N, n_vis, n_cubes, hq, hkv, d, BF16)
    ffn_b = token_ffn_workspace_bytes(N, n_vis, n_cubes, D, F, BF16)
    return {"Q": view(off[0], N * hq * d, (N, hq, d)), "K": view(off[1], N * hkv * d, (N, hkv, d)),
            "V": view(off[2], N * hkv * d, (N, hkv, d)), "a": view(off[3], N * hq * d, (N, hq, d)),
            "h": view(off[4], N * D, (N, D)),
            "attn_ws": workspace[off[5]:off[5] + attn_b], "ffn_ws": workspace[off[6]:off[6] + ffn_b]}


def rmsnorm(x, weight=None, eps=1e-6, out=None, stream=None):
    """RMSNorm of the rows of x (bf16 or fp32) into a bf16 tensor."""
    import torch
    _need(x, "x")
    n, D = x.shape
    if out is None:
        out = torch.empty((n, D), dtype=torch.bfloat16, device=x.device)
    _check(lib().adaspark_rmsnorm(_ptr(x), _dtype_code(x), _ptr(weight) if weight is not None
                                  else None, _ptr(out), n, D, float(eps), _stream(stream)),
           "adaspark_rmsnorm")
    return out


def ffn_export_active(workspace, n_tokens, n_vis, n_cubes, D, F, dtype, stream=None):
    import torch
    act = torch.empty(n_tokens, dtype=torch.uint8, device=workspace.device)
    _check(lib().adaspark_ffn_export_active(_ptr(workspace), n_tokens, n_vis, n_cubes, D, F,
                                            dtype, _ptr(act), _stream(stream)),
           "adaspark_ffn_export_active")
    return act.cpu().numpy().astype(bool)


def ffn_read_stats(workspace, stream=None) -> dict:
    st = _FfnStats()
    _check(lib().adaspark_ffn_read_stats(_ptr(workspace), ctypes.byref(st), _stream(stream)),
           "adaspark_ffn_read_stats")
    return {k: getattr(st, k) for k, _ in _FfnStats._fields_ if k != "reserved"}


# ----------------------------------------------------------------- status / timing
def read_device_status(workspace, stream=None):
    """(code, detail bits) of the last call on this workspace (synchronizes)."""
    det = ctypes.c_uint32(0)
    code = lib().adaspark_read_device_status(_ptr(workspace), ctypes.byref(det), _stream(stream))
    return code, det.value


def timer_enable(on: bool = True):
    _check(lib().adaspark_timer_enable(1 if on else 0), "adaspark_timer_enable")


def timer_read(max_entries: int = 64) -> dict:
    buf = (_KernelTime * max_entries)()
    n = ctypes.c_int(0)
    _check(lib().adaspark_timer_read(buf, max_entries, ctypes.byref(n)), "adaspark_timer_read")
    return {buf[i].name.decode(): (int(buf[i].launches), float(buf[i].total_ms))
            for i in range(n.value)}


def debug_wait_expiry(on: bool, wait_cycles: int = 2_000_000):
    """Test hook of the bounded waits (adaspark_debug_wait_expiry): while on,
    bf16 AdaS-Attn launches withhold their first key block and give up after
    wait_cycles SM cycles, reporting ADASPARK_DEV_TIMEOUT."""
    _check(lib().adaspark_debug_wait_expiry(1 if on else 0, int(wait_cycles)),
           "adaspark_debug_wait_expiry")


def set_split_rows(rows: int):
    """adaspark_set_split_rows: a tile's selected cube that at most `rows` of its
    rows chose runs in a gathered tile (0: the single walk)."""
    _check(lib().adaspark_set_split_rows(int(rows)), "adaspark_set_split_rows")


SPLIT_ROWS_DEFAULT = 8


def launch_count() -> int:
    return int(lib().adaspark_launch_count())


def device_check(device: int = 0) -> int:
    return int(lib().adaspark_device_check(device))
