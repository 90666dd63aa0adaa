"""Float64 numpy statement of the AdaSpark layer (test infrastructure only).

Sources (page titles and sections; the pages print no code for this method):

* "AdaSpark: Adaptive Sparsity for Efficient Long-Video Understanding"
  (papernotes.org note), sections 整体框架 (overall framework) and 关键设计 1-4
  (key designs: 3D cube partition, AdaS-Attn with the P_i / S_i formula,
  AdaS-FFN with the mean-compensation formula, the shared Top-p knob).
* The same paper's abstract and Figure 2 caption (thelatestinai.com list view):
  relevance is scored over *preceding* cubes; text tokens pass densely through
  the FFN.

Readings taken where the pages leave a step open (each is listed, with its
basis, in the design notes of this repository):

* tokens are in cube-major order, cubes enumerated time-major (t_b, h_b, w_b),
  tokens inside a cube in (t, h, w) order; edge cubes are truncated;
* the index i of P_i is the query's own cube; P_i runs over cubes 0..i-1, the
  own cube is always attended causally, the first cube selects nothing;
* selection is per (query token, query head); query head h reads KV head
  floor(h / (hq / hkv));
* Top-p: order by (probability descending, index ascending), take the smallest
  prefix whose cumulative mass reaches p, at least one element; p >= 1 keeps all;
* the selected cubes and the own-cube causal prefix share one softmax; P_i is
  not used as a weight;
* text tokens are the suffix and attend densely and causally;
* FFN importance is the linear share of the L2 norm inside the cube,
  w_u = ||x_u|| / sum_v ||x_v||; a cube whose norms sum to 0 keeps every token;
* the FFN is SwiGLU without bias, W_down(silu(W_gate x) * W_up x); an active
  or text token gets y = x + FFN(x), a skipped one y = x + mean of FFN over the
  cube's active tokens (unrounded).
"""
from __future__ import annotations

import math

import numpy as np


def _f64(a):
    """Exact float64 copy of a numpy array or torch tensor (bf16 widens exactly)."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# Key design 1: 3D spatio-temporal cube partition.
# ---------------------------------------------------------------------------
def cube_partition(T, H, W, cube_h, cube_w, cube_t, n_text):
    """Split a T x H x W video-token grid into h x w x t cubes.

    Follows the partition of key design 1 (cubes are h x w x t windows of the
    video tokens fed to the LLM).  Returns ``perm`` (perm[k] = raster index
    t*H*W + h*W + w of the k-th token in cube-major order), ``cube_ids`` (cube of
    each cube-major position, then -1 for each of the n_text text tokens),
    ``cube_offsets`` [C+1] and C.  Cubes are enumerated time-major over the cube
    grid; tokens within a cube in (t, h, w) order; edge cubes are truncated.
    """
    if min(T, H, W, cube_h, cube_w, cube_t) <= 0 or n_text < 0:
        raise ValueError("sizes must be positive")
    n_tb = -(-T // cube_t)
    n_hb = -(-H // cube_h)
    n_wb = -(-W // cube_w)
    perm, ids, offsets = [], [], [0]
    c = 0
    for tb in range(n_tb):
        for hb in range(n_hb):
            for wb in range(n_wb):
                for t in range(tb * cube_t, min(T, (tb + 1) * cube_t)):
                    for h in range(hb * cube_h, min(H, (hb + 1) * cube_h)):
                        for w in range(wb * cube_w, min(W, (wb + 1) * cube_w)):
                            perm.append(t * H * W + h * W + w)
                            ids.append(c)
                offsets.append(len(perm))
                c += 1
    ids.extend([-1] * n_text)
    return (np.asarray(perm, np.int32), np.asarray(ids, np.int32),
            np.asarray(offsets, np.int32), c)


# ---------------------------------------------------------------------------
# Key design 2: AdaS-Attn.
# ---------------------------------------------------------------------------
def cube_mean_keys(K, cube_offsets):
    """k_bar[j, kv, :] = mean of K over the tokens of cube j (key design 2,
    "similarity to the cube's mean key").  K: [N, hkv, d]; returns float64
    [C, hkv, d], accumulated token by token."""
    K = _f64(K)
    off = np.asarray(cube_offsets)
    C = len(off) - 1
    out = np.zeros((C,) + K.shape[1:], dtype=np.float64)
    for j in range(C):
        acc = np.zeros(K.shape[1:], dtype=np.float64)
        for t in range(off[j], off[j + 1]):
            acc += K[t]
        out[j] = acc / (off[j + 1] - off[j])
    return out


def cube_scores(q, kbar_rows, d):
    """s_j = q . k_bar_j / sqrt(d_k) for the preceding cubes (key design 2,
    the argument of the softmax in the P_i formula).  q: [..., d],
    kbar_rows: [c, d]."""
    return (_f64(q) @ _f64(kbar_rows).T) / math.sqrt(d)


def softmax(s, axis=-1):
    """Softmax in float64 (the P_i formula of key design 2)."""
    s = np.asarray(s, dtype=np.float64)
    if s.shape[axis] == 0:
        return s.copy()
    m = np.max(s, axis=axis, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=axis, keepdims=True)


def _check_p(p):
    if not (p > 0.0 and p <= 1.0):  # also rejects NaN
        raise ValueError("p must lie in (0, 1]")


def top_p(P, p):
    """Top-p (nucleus) set of a probability vector (S_i of key design 2; the same
    rule drives AdaS-FFN per key designs 3 and 4).

    Order the entries by probability descending, index ascending; keep the
    smallest prefix whose cumulative mass reaches p (at least one entry; every
    entry when the sum never reaches p in floating point).  p >= 1 keeps all.
    Returns a boolean mask over the entries.
    """
    _check_p(p)
    P = np.asarray(P, dtype=np.float64)
    m = P.shape[-1]
    keep = np.zeros(P.shape, dtype=bool)
    if m == 0:
        return keep
    if p >= 1.0:
        keep[...] = True
        return keep
    flat = P.reshape(-1, m)
    kflat = keep.reshape(-1, m)
    order = np.argsort(-flat, axis=1, kind="stable")
    cum = np.cumsum(np.take_along_axis(flat, order, axis=1), axis=1)
    reached = cum >= p
    kstar = np.where(reached.any(axis=1), reached.argmax(axis=1) + 1, m)
    for r in range(flat.shape[0]):
        kflat[r, order[r, :kstar[r]]] = True
    return keep


def top_p_margin(P, p):
    """Distance of a Top-p cut from flipping: the smallest of C_k* - p,
    p - C_(k*-1) (k* > 1) and P_(k*) - P_(k*+1) (k* < m), in the sorted order
    used by ``top_p``.  +inf when nothing can flip (m <= 1 or p >= 1)."""
    _check_p(p)
    P = np.asarray(P, dtype=np.float64)
    m = P.shape[-1]
    flat = P.reshape(-1, m)
    out = np.full(flat.shape[0], np.inf)
    if m <= 1 or p >= 1.0:
        return out.reshape(P.shape[:-1])
    order = np.argsort(-flat, axis=1, kind="stable")
    srt = np.take_along_axis(flat, order, axis=1)
    cum = np.cumsum(srt, axis=1)
    reached = cum >= p
    kstar = np.where(reached.any(axis=1), reached.argmax(axis=1) + 1, m)
    for r in range(flat.shape[0]):
        k = kstar[r]
        cand = [cum[r, k - 1] - p]
        if k > 1:
            cand.append(p - cum[r, k - 2])
        if k < m:
            cand.append(srt[r, k - 1] - srt[r, k])
        out[r] = min(cand)
    return out.reshape(P.shape[:-1])


def top_k(P, k):
    """Top-K set of a probability vector: the fixed-size selection that the
    AdaSpark paper compares with Top-p (ablation table of selection strategies,
    row "Top-K"). The k entries of largest probability in the (probability
    descending, index ascending) order; every entry when there are at most k.
    Returns a boolean mask over the entries."""
    if int(k) != k or k < 1:
        raise ValueError("k must be a positive integer")
    P = np.asarray(P, dtype=np.float64)
    m = P.shape[-1]
    keep = np.zeros(P.shape, dtype=bool)
    if m == 0:
        return keep
    flat = P.reshape(-1, m)
    kflat = keep.reshape(-1, m)
    order = np.argsort(-flat, axis=1, kind="stable")
    kk = min(int(k), m)
    for r in range(flat.shape[0]):
        kflat[r, order[r, :kk]] = True
    return keep


def top_k_margin(P, k):
    """Distance of a Top-K set from flipping: P_(k) - P_(k+1) in the sorted
    order used by ``top_k`` (+inf when there are at most k entries)."""
    P = np.asarray(P, dtype=np.float64)
    m = P.shape[-1]
    flat = P.reshape(-1, m)
    out = np.full(flat.shape[0], np.inf)
    if m > k:
        srt = -np.sort(-flat, axis=1)
        out = srt[:, k - 1] - srt[:, k]
    return out.reshape(P.shape[:-1])


def uniform_cubes(i, k):
    """Uniform Sampling, the content-independent strategy of the AdaSpark
    paper's selection-strategy ablation (the pages name it without defining
    it; reading: k of the i preceding cubes at even spacing from the first,
    j_m = floor(m * i / k) for m = 0..k-1, every preceding cube when i <= k).
    Returns the ascending cube indices."""
    if int(k) != k or k < 1:
        raise ValueError("k must be a positive integer")
    if i <= k:
        return np.arange(i)
    return (np.arange(k) * i) // k


def select_cubes_uniform(cube_offsets, n_vis, hq, k, tokens=None):
    """AdaS-Attn sets under Uniform Sampling (``uniform_cubes``): every query
    head of every token of cube i gets the same set. Returns a boolean array
    sel[len(tokens), hq, C] like ``select_cubes`` (own cube not marked)."""
    off = np.asarray(cube_offsets)
    C = len(off) - 1
    if tokens is None:
        tokens = np.arange(n_vis)
    tokens = np.asarray(tokens)
    cube_of = np.searchsorted(off, tokens, side="right") - 1
    sel = np.zeros((len(tokens), hq, C), dtype=bool)
    for r, i in enumerate(cube_of):
        sel[r, :, uniform_cubes(int(i), k)] = True
    return sel


def select_cubes(Q, K, cube_offsets, n_vis, hq, hkv, p, tokens=None, with_margin=False,
                 k=None, kbar=None):
    """AdaS-Attn cube selection (key design 2, formula P_i and S_i).

    For visual token t in cube i and query head h: P = softmax over the
    preceding cubes j < i of q . k_bar_j / sqrt(d), k_bar of KV head
    floor(h / (hq/hkv)); S = Top-p(P, p), or Top-K(P, k) when ``k`` is given
    (then ``p`` is ignored).  Returns a boolean array
    sel[len(tokens), hq, C] (sel[r, h, j] is True when cube j is selected; the
    own cube is not marked here, it is always attended causally) and, when
    asked, the cut margins [len(tokens), hq] (+inf where nothing can flip).
    ``tokens`` defaults to every visual token.  ``kbar`` may pass the cube mean
    keys of ``cube_mean_keys(K, cube_offsets)`` when the caller has them (they
    belong to the layer, not to the selected rows).
    """
    if k is None:
        _check_p(p)
    off = np.asarray(cube_offsets)
    C = len(off) - 1
    d = Q.shape[-1]
    g = hq // hkv
    if kbar is None:
        kbar = cube_mean_keys(K, off)
    if tokens is None:
        tokens = np.arange(n_vis)
    tokens = np.asarray(tokens)
    cube_of = np.searchsorted(off, tokens, side="right") - 1
    sel = np.zeros((len(tokens), hq, C), dtype=bool)
    margin = np.full((len(tokens), hq), np.inf)
    Qf = _f64(Q[tokens]) if not isinstance(Q, np.ndarray) else _f64(Q)[tokens]
    for i in np.unique(cube_of):
        rows = np.nonzero(cube_of == i)[0]
        if i == 0:
            continue  # no preceding cube: empty set
        for h in range(hq):
            kv = h // g
            s = cube_scores(Qf[rows, h, :], kbar[:i, kv, :], d)   # [rows, i]
            P = softmax(s, axis=1)
            if k is None:
                sel[rows, h, :i] = top_p(P, p)
                if with_margin:
                    margin[rows, h] = top_p_margin(P, p)
            else:
                sel[rows, h, :i] = top_k(P, k)
                if with_margin:
                    margin[rows, h] = top_k_margin(P, k)
    if with_margin:
        return sel, margin
    return sel


def attention_given_sets(Q, K, V, cube_offsets, n_vis, sel, tokens=None):
    """GQA attention restricted to the selected cubes plus the own cube
    (key design 2: each query attends only to the chosen cubes and always keeps
    full attention to its own cube; causal inside the own cube).  Text tokens
    (index >= n_vis) attend densely and causally to every earlier token.

    One softmax over all admitted keys, scale 1/sqrt(d), written as a masked
    dense softmax per (cube, head).  ``sel`` is [len(tokens), hq, C] for the
    tokens in ``tokens`` (rows of text tokens are ignored).  Returns float64
    out [len(tokens), hq, d].
    """
    off = np.asarray(cube_offsets)
    N, hq, d = Q.shape
    hkv = K.shape[1]
    g = hq // hkv
    if tokens is None:
        tokens = np.arange(N)
    tokens = np.asarray(tokens)
    Kf, Vf = _f64(K), _f64(V)
    Qf = _f64(Q)[tokens] if isinstance(Q, np.ndarray) else _f64(Q[tokens])
    out = np.zeros((len(tokens), hq, d), dtype=np.float64)
    key_cube = np.concatenate([np.searchsorted(off, np.arange(n_vis), side="right") - 1,
                               np.full(N - n_vis, -1)])
    pos = np.arange(N)
    scale = 1.0 / math.sqrt(d)
    group = np.where(tokens < n_vis, key_cube[np.minimum(tokens, N - 1)], -1)
    for i in np.unique(group):
        rows = np.nonzero(group == i)[0]
        t = tokens[rows]
        if i < 0:                       # text rows: dense causal over all earlier tokens
            end = int(t.max()) + 1
            base = pos[None, :end] <= t[:, None]
        else:                           # visual rows of cube i
            end = int(off[i + 1])
            base = (key_cube[None, :end] == i) & (pos[None, :end] <= t[:, None])
        for h in range(hq):
            kv = h // g
            if i < 0:
                mask = base
            else:
                kc = key_cube[:end]
                chosen = sel[rows][:, h, :][:, np.maximum(kc, 0)] & (kc < i)[None, :]
                mask = base | chosen
            s = (Qf[rows, h, :] @ Kf[:end, kv, :].T) * scale
            s = np.where(mask, s, -np.inf)
            m = np.max(s, axis=1, keepdims=True)
            e = np.where(mask, np.exp(s - m), 0.0)
            out[rows, h] = (e / e.sum(axis=1, keepdims=True)) @ Vf[:end, kv, :]
    return out


def cube_attn(Q, K, V, cube_offsets, n_vis, p, tokens=None):
    """The whole AdaS-Attn call: selection then restricted attention."""
    hq, hkv = Q.shape[1], K.shape[1]
    sel = select_cubes(Q, K, cube_offsets, n_vis, hq, hkv, p, tokens=tokens)
    return attention_given_sets(Q, K, V, cube_offsets, n_vis, sel, tokens=tokens), sel


# ---------------------------------------------------------------------------
# Key design 3: AdaS-FFN with mean compensation.
# ---------------------------------------------------------------------------
IMPORTANCE = ("l2", "l2sq", "softmax")


def token_importance(norms, importance="l2"):
    """Importance of a cube's tokens from their L2 norms (key design 3 only says
    that importance comes from the L2 norm, followed by the same Top-p rule).
    "l2": the linear share ||x_u|| / sum ||x_v|| (the default reading); the two
    alternatives the pages do not exclude: "l2sq", the energy share ||x_u||^2 / sum ||x_v||^2,
    and "softmax", softmax over the cube of ||x_u||. All three rank tokens in
    the same order as their norms. Returns None when the norms sum to 0 (l2,
    l2sq: no importance is defined; the cube keeps every token)."""
    norms = np.asarray(norms, dtype=np.float64)
    if importance == "l2":
        total = norms.sum()
        return None if total == 0.0 else norms / total
    if importance == "l2sq":
        sq = norms * norms
        total = sq.sum()
        return None if total == 0.0 else sq / total
    if importance == "softmax":
        return softmax(norms)
    raise ValueError(f"importance must be one of {IMPORTANCE}")


def ffn_select(x, cube_offsets, n_vis, p, cubes=None, with_margin=False, importance="l2"):
    """AdaS-FFN token selection (key design 3): inside each cube rank tokens by
    L2 norm, importance w_u = ||x_u|| / sum_v ||x_v|| (or a variant of
    ``token_importance``), keep Top-p(w, p).  Text tokens are always active.
    Returns a boolean ``active`` [N] (entries of cubes not in ``cubes`` are left
    False) and, when asked, per-cube margins."""
    _check_p(p)
    N = x.shape[0]
    off = np.asarray(cube_offsets)
    C = len(off) - 1
    active = np.zeros(N, dtype=bool)
    active[n_vis:] = True
    margins = np.full(C, np.inf)
    if cubes is None:
        cubes = range(C)
    for c in cubes:
        a, b = off[c], off[c + 1]
        Xc = _f64(x[a:b])
        norms = np.sqrt(np.sum(Xc * Xc, axis=1))
        w = token_importance(norms, importance)
        if w is None:
            active[a:b] = True
            continue
        active[a:b] = top_p(w, p)
        if with_margin:
            margins[c] = top_p_margin(w, p)
    if with_margin:
        return active, margins
    return active


def swiglu_ffn(x, W_gate, W_up, W_down):
    """FFN(x) = W_down (silu(W_gate x) * W_up x), no bias, float64."""
    X = _f64(x)
    gate = X @ _f64(W_gate).T
    up = X @ _f64(W_up).T
    h = gate / (1.0 + np.exp(-gate)) * up
    return h @ _f64(W_down).T


def ffn_given_sets(x, W_gate, W_up, W_down, cube_offsets, n_vis, active, cubes=None,
                   text=True):
    """Outputs of AdaS-FFN for a given active set (key design 3): active and text
    tokens y = x + FFN(x); skipped tokens y_k = x_k + m_bar_i with
    m_bar_i = mean of FFN(x_j) over the cube's active tokens.  Returns float64
    y [N, D] (rows of cubes outside ``cubes`` are NaN; text rows NaN when
    ``text`` is False)."""
    N, D = x.shape
    off = np.asarray(cube_offsets)
    C = len(off) - 1
    y = np.full((N, D), np.nan)
    Wg, Wu, Wd = _f64(W_gate), _f64(W_up), _f64(W_down)
    if cubes is None:
        cubes = range(C)
    for c in cubes:
        a, b = off[c], off[c + 1]
        Xc = _f64(x[a:b])
        act = active[a:b]
        f = swiglu_ffn(Xc[act], Wg, Wu, Wd)
        y[a:b][act] = Xc[act] + f
        if (~act).any():
            mbar = f.sum(axis=0) / int(act.sum())
            y[a:b][~act] = Xc[~act] + mbar
    if text and N > n_vis:
        Xt = _f64(x[n_vis:])
        y[n_vis:] = Xt + swiglu_ffn(Xt, Wg, Wu, Wd)
    return y


def token_ffn(x, W_gate, W_up, W_down, cube_offsets, n_vis, p, cubes=None, text=True):
    """The whole AdaS-FFN call: selection then the given-set outputs."""
    active = ffn_select(x, cube_offsets, n_vis, p, cubes=cubes)
    return ffn_given_sets(x, W_gate, W_up, W_down, cube_offsets, n_vis, active,
                          cubes=cubes, text=text), active


# ---------------------------------------------------------------------------
# Around the two modules: the projections and the normalization of a layer.
# ---------------------------------------------------------------------------
def linear(x, W):
    """x W^T in float64 (W in [out, in] layout): the Q/K/V/O projections of the
    layer around AdaS-Attn and AdaS-FFN (the pages place the two modules in a
    decoder layer but say nothing about these matrices)."""
    return _f64(x) @ _f64(W).T


def rmsnorm(x, w=None, eps=1e-6):
    """x / sqrt(mean(x^2) + eps) per row, times w when given, in float64."""
    xf = _f64(x)
    r = 1.0 / np.sqrt(np.mean(xf * xf, axis=-1, keepdims=True) + eps)
    out = xf * r
    return out * _f64(w) if w is not None else out



# ---------------------------------------------------------------------------
# Backward pass for light fine-tuning (the note's "AdaSpark can be adapted with
# a small amount of fine-tuning"), selection straight-through: the cube sets of
# key design 2 and the active sets of key design 3 are held fixed, so no
# gradient reaches the cube mean keys, the relevance softmax, or the token
# norms; everything the sets admit is differentiated as computed.
# ---------------------------------------------------------------------------
def attention_backward_given_sets(Q, K, V, dO, cube_offsets, n_vis, sel, with_magnitudes=False,
                                  cubes=None, text=True):
    """Gradients of ``attention_given_sets`` (all tokens) for the upstream
    gradient dO [N, hq, d], with the sets ``sel`` [N, hq, C] held fixed.

    Per (row, head), with P the row's softmax over its admitted keys and
    dP = dO . V^T: dS = P * (dP - sum(P * dP)); dQ = dS K / sqrt(d); the key
    and value gradients collect dS^T Q / sqrt(d) and P^T dO over every row of
    every query head that reads the KV head (GQA).  Returns float64 (dQ, dK, dV)
    shaped like Q, K, V.  With ``with_magnitudes`` it also returns the same
    three sums taken over absolute values (|dS| |K| / sqrt(d), |dS|^T |Q| /
    sqrt(d), P^T |dO|): the scale a rounding of dS or P enters each gradient
    element with, for comparisons that round those operands.  ``cubes`` /
    ``text`` restrict the query rows to the visual tokens of those cubes and
    (or not) the text tokens: dQ is then exact on those rows (zero elsewhere)
    and dK, dV hold only their contributions, exact for keys that no other row
    admits (e.g. the last cube's keys with ``cubes=[C-1]`` and the text rows).
    """
    off = np.asarray(cube_offsets)
    N, hq, d = Q.shape
    hkv = K.shape[1]
    g = hq // hkv
    Qf, Kf, Vf, dOf = _f64(Q), _f64(K), _f64(V), _f64(dO)
    dQ = np.zeros_like(Qf)
    dK = np.zeros_like(Kf)
    dV = np.zeros_like(Vf)
    mQ, mK, mV = np.zeros_like(Qf), np.zeros_like(Kf), np.zeros_like(Vf)
    key_cube = np.concatenate([np.searchsorted(off, np.arange(n_vis), side="right") - 1,
                               np.full(N - n_vis, -1)])
    pos = np.arange(N)
    scale = 1.0 / math.sqrt(d)
    tokens = np.arange(N)
    group = np.where(tokens < n_vis, key_cube, -1)
    wanted = set(range(len(off) - 1)) if cubes is None else set(int(c) for c in cubes)
    if text:
        wanted.add(-1)
    for i in np.unique(group):
        if int(i) not in wanted:
            continue
        t = np.nonzero(group == i)[0]
        if i < 0:
            end = int(t.max()) + 1
            base = pos[None, :end] <= t[:, None]
        else:
            end = int(off[i + 1])
            base = (key_cube[None, :end] == i) & (pos[None, :end] <= t[:, None])
        for h in range(hq):
            kv = h // g
            if i < 0:
                mask = base
            else:
                kc = key_cube[:end]
                chosen = sel[t][:, h, :][:, np.maximum(kc, 0)] & (kc < i)[None, :]
                mask = base | chosen
            q, k, v, do = Qf[t, h, :], Kf[:end, kv, :], Vf[:end, kv, :], dOf[t, h, :]
            s = np.where(mask, (q @ k.T) * scale, -np.inf)
            m = np.max(s, axis=1, keepdims=True)
            e = np.where(mask, np.exp(s - m), 0.0)
            P = e / e.sum(axis=1, keepdims=True)
            dP = do @ v.T
            dS = P * (dP - np.sum(P * dP, axis=1, keepdims=True))
            dQ[t, h] = (dS @ k) * scale
            dK[:end, kv] += (dS.T @ q) * scale
            dV[:end, kv] += P.T @ do
            if with_magnitudes:
                aS = np.abs(dS)
                mQ[t, h] = (aS @ np.abs(k)) * scale
                mK[:end, kv] += (aS.T @ np.abs(q)) * scale
                mV[:end, kv] += P.T @ np.abs(do)
    if with_magnitudes:
        return dQ, dK, dV, (mQ, mK, mV)
    return dQ, dK, dV


def swiglu_ffn_backward(x, W_gate, W_up, W_down, df, with_magnitudes=False):
    """Gradients of f = swiglu_ffn(x) for the upstream gradient df [n, D]:
    with g = x W_gate^T, u = x W_up^T, silu(g) = g sigma(g), h = silu(g) u,
    dh = df W_down; du = dh silu(g); dg = dh u sigma(g) (1 + g (1 - sigma(g)));
    dx = dg W_gate + du W_up; dW_gate = dg^T x; dW_up = du^T x; dW_down = df^T h.
    Returns float64 (dx, dW_gate, dW_up, dW_down).  With ``with_magnitudes``
    also, per gradient, the scale in which one relative rounding of the
    intermediates df, dg, du and h (each rounded once, the error in df carried
    through dh into dg and du) enters each element: a comparison that rounds
    those intermediates to a format with unit roundoff r stays within about
    r times this scale."""
    X, Wg, Wu, Wd, dF = _f64(x), _f64(W_gate), _f64(W_up), _f64(W_down), _f64(df)
    gate = X @ Wg.T
    up = X @ Wu.T
    sig = 1.0 / (1.0 + np.exp(-gate))
    silu = gate * sig
    h = silu * up
    dh = dF @ Wd
    du = dh * silu
    dsilu_u = up * sig * (1.0 + gate * (1.0 - sig))
    dg = dh * dsilu_u
    dx = dg @ Wg + du @ Wu
    grads = (dx, dg.T @ X, du.T @ X, dF.T @ h)
    if not with_magnitudes:
        return grads
    m_dh = np.abs(dF) @ np.abs(Wd)                  # df's rounding inside dh
    m_dg = np.abs(dsilu_u) * m_dh + np.abs(dg)      # ... carried into dg, plus dg's own
    m_du = np.abs(silu) * m_dh + np.abs(du)
    aX = np.abs(X)
    mags = (m_dg @ np.abs(Wg) + m_du @ np.abs(Wu), m_dg.T @ aX, m_du.T @ aX,
            2.0 * (np.abs(dF).T @ np.abs(h)))         # df and h both rounded
    return grads, mags


def ffn_backward_given_sets(x, W_gate, W_up, W_down, cube_offsets, n_vis, active, dy,
                            cubes=None, text=True, with_magnitudes=False):
    """Gradients of ``ffn_given_sets`` (all cubes and the text rows) for the
    upstream gradient dy [N, D], the active set held fixed.

    A skipped token's output is x_k + m_bar of its cube, so its own gradient is
    dy_k and its dy_k also reaches every active token of the cube through the
    mean: the FFN of active token a receives df_a = dy_a + (sum of dy_k over
    the cube's skipped tokens) / (number of active tokens).  Text tokens get
    df = dy.  Then dx = dy + the FFN's input gradient for computed rows, and
    the weight gradients sum over every computed row.  Returns float64
    (dx [N, D], dW_gate [F, D], dW_up [F, D], dW_down [D, F]).  ``cubes`` /
    ``text`` restrict the rows to those cubes and (or not) the text tokens: dx
    is exact on them (NaN elsewhere) and the weight gradients hold only their
    rows' contributions.  ``with_magnitudes`` adds the rounding scales of
    ``swiglu_ffn_backward`` (zero on the skipped rows' dx, whose gradient is
    dy itself)."""
    N, D = x.shape
    off = np.asarray(cube_offsets)
    C = len(off) - 1
    X, dY = _f64(x), _f64(dy)
    active = np.asarray(active, dtype=bool).copy()
    active[n_vis:] = True
    keep = np.zeros(N, dtype=bool)
    for c in (range(C) if cubes is None else cubes):
        keep[off[c]:off[c + 1]] = True
    keep[n_vis:] = text
    df = np.zeros_like(dY)
    for c in range(C):
        a, b = off[c], off[c + 1]
        if not keep[a:b].any():
            continue
        act = active[a:b]
        df[a:b][act] = dY[a:b][act]
        if (~act).any():
            df[a:b][act] += dY[a:b][~act].sum(axis=0) / int(act.sum())
    df[n_vis:] = dY[n_vis:]
    rows = np.nonzero(active & keep)[0]
    res = swiglu_ffn_backward(X[rows], W_gate, W_up, W_down, df[rows],
                              with_magnitudes=with_magnitudes)
    dxr, dWg, dWu, dWd = res[0] if with_magnitudes else res
    dx = np.where(keep[:, None], dY, np.nan)
    dx[rows] += dxr
    if not with_magnitudes:
        return dx, dWg, dWu, dWd
    mdx = np.zeros_like(dY)
    mdx[rows] = res[1][0]
    return (dx, dWg, dWu, dWd), (mdx, res[1][1], res[1][2], res[1][3])
