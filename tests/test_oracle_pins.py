"""Pins for the float64 oracle: each test checks it against something other than
itself -- brute force on tiny inputs, closed forms, invariants, or an
independent library routine (torch in float64) -- so that a dropped term, a
wrong sign or index, or a transposed operand in the oracle fails here.
All CPU-only."""
import itertools
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

import oracle
from oracle import adaspark_ref as ref


# ---------------------------------------------------------------- partition
@pytest.mark.parametrize("grid,cube,n_text", [
    ((4, 4, 4), (2, 2, 2), 0),
    ((5, 7, 3), (2, 3, 2), 3),      # truncated edge cubes on every axis
    ((8, 8, 8), (4, 4, 2), 32),
    ((3, 1, 1), (1, 1, 1), 1),      # one token per cube
    ((2, 3, 5), (4, 4, 4), 0),      # one cube larger than the grid
])
def test_partition_matches_sorted_order(grid, cube, n_text):
    T, H, W = grid
    ch, cw, ct = cube
    perm, ids, off, C = oracle.cube_partition(T, H, W, ch, cw, ct, n_text)
    # Independent statement: sort raster positions by (cube t, cube h, cube w, t, h, w).
    keys = []
    for t in range(T):
        for h in range(H):
            for w in range(W):
                keys.append(((t // ct, h // ch, w // cw), (t, h, w), t * H * W + h * W + w))
    keys.sort()
    cube_keys = sorted({k[0] for k in keys})
    rank = {k: i for i, k in enumerate(cube_keys)}
    assert C == len(cube_keys)
    assert list(perm) == [k[2] for k in keys]
    assert sorted(perm.tolist()) == list(range(T * H * W))       # bijection
    assert list(ids[:T * H * W]) == [rank[k[0]] for k in keys]
    assert list(ids[T * H * W:]) == [-1] * n_text
    counts = np.bincount(ids[:T * H * W], minlength=C)
    assert list(np.diff(off)) == list(counts)
    assert off[0] == 0 and off[-1] == T * H * W


# ---------------------------------------------------------------- top-p rule
def _brute_top_p(P, p):
    """Minimal cardinality, then maximal mass, then lexicographically smallest."""
    m = len(P)
    best = None
    for k in range(1, m + 1):
        cands = []
        for S in itertools.combinations(range(m), k):
            mass = sum(P[j] for j in S)
            if mass >= p:
                cands.append((-mass, S))
        if cands:
            cands.sort()
            best = cands[0][1]
            break
    assert best is not None
    return set(best)


def test_top_p_brute_force():
    rng = np.random.default_rng(5)
    for trial in range(300):
        m = int(rng.integers(1, 11))
        # integer weights / 1024: every partial sum is exact in binary, so the
        # brute force and the prefix rule see identical masses; small ranges
        # force many ties.
        w = rng.integers(1, 6 if trial % 2 else 200, size=m).astype(np.float64)
        w = np.floor(w / w.sum() * 1024)
        w[0] += 1024 - w.sum()
        if w.min() <= 0:
            continue
        P = w / 1024.0
        # p on the grid (exact equality must count as reached) or between points
        p = float(rng.integers(1, 1024)) / 1024.0
        if trial % 3 == 0:
            p -= 1.0 / 4096.0
        got = set(np.nonzero(oracle.top_p(P, p))[0].tolist())
        assert got == _brute_top_p(P, p), (P, p)


@pytest.mark.parametrize("m,p", [(7, 0.7), (10, 0.55), (13, 0.31), (64, 0.7), (100, 0.905)])
def test_top_p_uniform_closed_form(m, p):
    P = np.full(m, 1.0 / m)
    keep = oracle.top_p(P, p)
    k = math.ceil(p * m)
    assert keep.sum() == k
    assert keep[:k].all()      # ties go to the lower indices


def test_top_p_degenerate():
    P = np.array([0.1, 0.4, 0.4, 0.1])
    assert np.nonzero(oracle.top_p(P, 1e-9))[0].tolist() == [1]   # argmax, first of the tie
    assert oracle.top_p(P, 1.0).all()
    assert oracle.top_p(np.zeros(0), 0.5).shape == (0,)
    # cumulative mass exactly equal to p counts as reached (binary-exact values)
    assert np.nonzero(oracle.top_p(np.array([0.25, 0.5, 0.25]), 0.75))[0].tolist() == [0, 1]
    assert oracle.top_p(np.full(4, 0.25), 0.5).tolist() == [True, True, False, False]
    for bad in (0.0, -0.1, 1.5, float("nan")):
        with pytest.raises(ValueError):
            oracle.top_p(P, bad)


def test_top_p_margin_values():
    P = np.array([0.5, 0.3, 0.2])
    # p = 0.75: k* = 2, C_2 = 0.8, C_1 = 0.5, P_(2) - P_(3) = 0.1
    assert oracle.top_p_margin(P, 0.75) == pytest.approx(min(0.05, 0.25, 0.1))
    assert oracle.top_p_margin(np.array([0.25] * 4), 0.6) == 0.0   # exact tie at the cut


def _brute_top_k(P, k):
    """Among all subsets of size min(k, m): maximal mass, then lexicographically
    lowest index tuple (the tie rule), by enumeration."""
    m = len(P)
    kk = min(k, m)
    best = None
    for S in itertools.combinations(range(m), kk):
        key = (-sum(P[j] for j in S), S)
        if best is None or key < best:
            best = key
    return set(best[1])


def test_top_k_brute_force():
    rng = np.random.default_rng(9)
    for trial in range(300):
        m = int(rng.integers(1, 11))
        k = int(rng.integers(1, 12))
        # binary-exact masses with many ties
        w = rng.integers(1, 5 if trial % 2 else 300, size=m).astype(np.float64) / 1024.0
        got = set(np.nonzero(oracle.top_k(w, k))[0].tolist())
        assert got == _brute_top_k(w, k), (w, k)


@pytest.mark.parametrize("m,k", [(7, 3), (10, 1), (13, 13), (5, 9), (64, 20)])
def test_top_k_uniform_closed_form(m, k):
    keep = oracle.top_k(np.full(m, 1.0 / m), k)
    assert keep.sum() == min(k, m)
    assert keep[:min(k, m)].all()        # ties go to the lower indices


def test_top_k_degenerate_and_margin():
    P = np.array([0.1, 0.4, 0.4, 0.1])
    assert np.nonzero(oracle.top_k(P, 1))[0].tolist() == [1]
    assert np.nonzero(oracle.top_k(P, 3))[0].tolist() == [0, 1, 2]
    assert oracle.top_k(np.zeros(0), 2).shape == (0,)
    for bad in (0, -1, 1.5):
        with pytest.raises(ValueError):
            oracle.top_k(P, bad)
    assert oracle.top_k_margin(np.array([0.5, 0.3, 0.2]), 1) == pytest.approx(0.2)
    assert oracle.top_k_margin(np.array([0.5, 0.3, 0.2]), 2) == pytest.approx(0.1)
    assert oracle.top_k_margin(np.array([0.5, 0.3, 0.2]), 3) == np.inf
    assert oracle.top_k_margin(P, 1) == 0.0     # exact tie at the cut (0.4 / 0.4)
    assert oracle.top_k_margin(P, 2) == pytest.approx(0.3)   # both 0.4 taken


def test_select_top_k_uniform_means():
    """Identical cube means with Top-K: the min(k, c) lowest-index preceding
    cubes (own cube excluded from the candidates)."""
    rng = np.random.default_rng(4)
    C, n, hq, hkv, d = 9, 3, 2, 1, 8
    off = np.arange(C + 1) * n
    N = C * n
    Q = rng.standard_normal((N, hq, d))
    K = np.tile(rng.standard_normal((1, hkv, d)), (N, 1, 1))
    for k in (1, 3, 20):
        sel = oracle.select_cubes(Q, K, off, N, hq, hkv, 0.5, k=k)
        for t in range(N):
            c = t // n
            kk = min(k, c)
            assert (sel[t].sum(axis=1) == kk).all()
            assert sel[t, :, :kk].all() and not sel[t, :, c:].any()


# ---------------------------------------------------------------- cube means
def test_cube_mean_keys_invariants():
    rng = np.random.default_rng(1)
    off = np.array([0, 3, 4, 9, 16])
    K = rng.standard_normal((16, 2, 8))
    kbar = oracle.cube_mean_keys(K, off)
    for j in range(4):
        resid = (K[off[j]:off[j + 1]] - kbar[j]).sum(axis=0)
        assert np.abs(resid).max() < 1e-12
    assert np.array_equal(kbar[1], K[3])                  # single-token cube
    Kc = np.repeat(rng.standard_normal((4, 1, 2, 8)), np.diff(off), axis=0).reshape(16, 2, 8)
    kc = oracle.cube_mean_keys(Kc, off)
    for j in range(4):
        assert np.allclose(kc[j], Kc[off[j]], atol=1e-15)   # constant cube -> that constant


# ---------------------------------------------------------------- AdaS-Attn selection
def _qkv(rng, N, hq, hkv, d, scale=1.0):
    Q = rng.standard_normal((N, hq, d)) * scale
    K = rng.standard_normal((N, hkv, d)) * scale
    V = rng.standard_normal((N, hkv, d))
    return Q, K, V


@pytest.mark.parametrize("p", [0.3, 0.55, 0.7, 0.9])
def test_select_uniform_means_closed_form(p):
    """All cube means equal -> P uniform over the c preceding cubes -> the
    ceil(p*c) lowest-index cubes.  Counting the own cube in P would give
    ceil(p*(c+1)) instead."""
    rng = np.random.default_rng(2)
    C, n, hq, hkv, d = 12, 4, 2, 1, 16
    off = np.arange(C + 1) * n
    N = C * n
    Q = rng.standard_normal((N, hq, d))
    K = np.tile(rng.standard_normal((1, hkv, d)), (N, 1, 1))
    sel = oracle.select_cubes(Q, K, off, N, hq, hkv, p)
    for t in range(N):
        c = t // n
        if c > 0 and abs(p * c - round(p * c)) < 1e-9:
            continue   # p*c on an integer: the cut sits exactly on a rounding tie
        for h in range(hq):
            k = math.ceil(p * c) if c > 0 else 0
            assert sel[t, h].sum() == k
            assert sel[t, h, :k].all()
            assert not sel[t, h, c:].any()
    # discriminates own-cube inclusion for at least one cube
    assert any(math.ceil(p * c) != math.ceil(p * (c + 1)) for c in range(1, C))


def test_select_two_cube_sigmoid_scale_and_sign():
    """Rows of cube 2 see cubes 0 and 1.  q . (kbar_1 - kbar_0) / sqrt(d) = ln 3,
    so P = (1/4, 3/4) exactly in closed form: p = 0.74 keeps cube 1 alone,
    p = 0.76 keeps both.  Dropping 1/sqrt(d) (P_1 ~ 0.99985) or flipping the
    sign (cube 0 preferred) changes the answer."""
    d, n = 64, 2
    off = np.array([0, n, 2 * n, 3 * n])
    N = 3 * n
    Q = np.zeros((N, 1, d))
    K = np.zeros((N, 1, d))
    V = np.zeros((N, 1, d))
    Q[:, 0, 0] = 1.0
    K[0:n, 0, 0] = 0.0
    K[n:2 * n, 0, 0] = math.sqrt(d) * math.log(3.0)
    sel = oracle.select_cubes(Q, K, off, N, 1, 1, 0.74)
    assert sel[2 * n:, 0, :].tolist() == [[False, True, False]] * n
    sel = oracle.select_cubes(Q, K, off, N, 1, 1, 0.76)
    assert sel[2 * n:, 0, :].tolist() == [[True, True, False]] * n
    # cube 1's rows see only cube 0: always selected; cube 0's rows: nothing
    assert sel[n:2 * n, 0, 0].all() and not sel[:n].any()


def test_select_gqa_head_mapping():
    """hq = 4, hkv = 2: heads 0,1 read KV head 0 and heads 2,3 read KV head 1
    (floor(h / g)); the two KV heads prefer opposite cubes."""
    d, n = 8, 2
    off = np.array([0, n, 2 * n, 3 * n])
    N = 3 * n
    Q = np.zeros((N, 4, d))
    Q[:, :, 0] = 1.0
    K = np.zeros((N, 2, d))
    K[0:n, 0, 0] = 20.0      # KV head 0 prefers cube 0
    K[n:2 * n, 1, 0] = 20.0  # KV head 1 prefers cube 1
    sel = oracle.select_cubes(Q, K, off, N, 4, 2, 0.5)
    rows = sel[2 * n:]
    for h, want in ((0, [True, False, False]), (1, [True, False, False]),
                    (2, [False, True, False]), (3, [False, True, False])):
        assert rows[:, h, :].tolist() == [want] * n


# ---------------------------------------------------------------- AdaS-Attn attention
def _sdpa_masked(Q, K, V, mask):
    """torch SDPA in float64 with an explicit boolean mask [hq, N, N]."""
    hq, hkv = Q.shape[1], K.shape[1]
    g = hq // hkv
    q = torch.from_numpy(Q).permute(1, 0, 2)[None]
    k = torch.from_numpy(K).repeat_interleave(g, dim=1).permute(1, 0, 2)[None]
    v = torch.from_numpy(V).repeat_interleave(g, dim=1).permute(1, 0, 2)[None]
    o = Fn.scaled_dot_product_attention(q, k, v, attn_mask=torch.from_numpy(mask)[None])
    return o[0].permute(1, 0, 2).numpy()


def test_attention_dense_equals_causal_sdpa():
    rng = np.random.default_rng(3)
    off = np.array([0, 5, 9, 16, 20, 27])
    n_vis, n_text, hq, hkv, d = 27, 6, 6, 2, 16
    N = n_vis + n_text
    Q, K, V = _qkv(rng, N, hq, hkv, d)
    sel = oracle.select_cubes(Q, K, off, n_vis, hq, hkv, 1.0)
    out = oracle.attention_given_sets(Q, K, V, off, n_vis, sel)
    causal = np.tril(np.ones((N, N), dtype=bool))
    want = _sdpa_masked(Q, K, V, np.broadcast_to(causal, (hq, N, N)).copy())
    assert np.abs(out - want).max() < 1e-12


def test_attention_given_random_sets_equals_masked_sdpa():
    rng = np.random.default_rng(4)
    off = np.array([0, 4, 8, 12, 16, 20, 24])
    n_vis, n_text, hq, hkv, d = 24, 5, 4, 2, 8
    N = n_vis + n_text
    C = len(off) - 1
    Q, K, V = _qkv(rng, N, hq, hkv, d)
    sel = rng.random((N, hq, C)) < 0.4
    out = oracle.attention_given_sets(Q, K, V, off, n_vis, sel)
    cube = np.searchsorted(off, np.arange(n_vis), side="right") - 1
    mask = np.zeros((hq, N, N), dtype=bool)
    for t in range(N):
        for h in range(hq):
            for u in range(t + 1):
                if t >= n_vis:
                    mask[h, t, u] = True
                elif cube[u] == cube[t]:
                    mask[h, t, u] = True
                elif cube[u] < cube[t] and sel[t, h, cube[u]]:
                    mask[h, t, u] = True
    want = _sdpa_masked(Q, K, V, mask)
    assert np.abs(out - want).max() < 1e-12
    # the very first token sees only itself
    g = hq // hkv
    for h in range(hq):
        assert np.array_equal(out[0, h], V[0, h // g])


def test_attention_smallest_p_is_argmax_cube_plus_own():
    rng = np.random.default_rng(6)
    off = np.arange(7) * 4
    n_vis, hq, hkv, d = 24, 2, 1, 8
    Q, K, V = _qkv(rng, n_vis, hq, hkv, d, scale=2.0)
    sel = oracle.select_cubes(Q, K, off, n_vis, hq, hkv, 1e-9)
    kbar = np.stack([K[off[j]:off[j + 1]].mean(axis=0) for j in range(6)])
    for t in range(4, n_vis):
        c = t // 4
        for h in range(hq):
            s = Q[t, h] @ kbar[:c, 0].T
            assert np.nonzero(sel[t, h])[0].tolist() == [int(np.argmax(s))]


# ---------------------------------------------------------------- AdaS-FFN
def _ffn_torch(x, Wg, Wu, Wd):
    x, Wg, Wu, Wd = (torch.from_numpy(np.asarray(a, dtype=np.float64)) for a in (x, Wg, Wu, Wd))
    return Fn.linear(Fn.silu(Fn.linear(x, Wg)) * Fn.linear(x, Wu), Wd).numpy()


def test_swiglu_matches_torch():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((9, 16))
    Wg, Wu, Wd = (rng.standard_normal(s) * 0.3 for s in ((24, 16), (24, 16), (16, 24)))
    assert np.abs(oracle.swiglu_ffn(x, Wg, Wu, Wd) - _ffn_torch(x, Wg, Wu, Wd)).max() < 1e-12


def test_ffn_select_closed_forms():
    rng = np.random.default_rng(8)
    D = 12
    v = rng.standard_normal(D)
    # cube 0: equal norms (sign flips keep the norm) -> uniform -> ceil(p n) lowest
    # cube 1: x_u = a_u v with distinct a_u -> w_u = a_u / sum(a): brute force
    # cube 2: all zeros -> everything active; cube 3: single token
    a = np.array([3.0, 1.0, 4.0, 1.5, 5.0, 9.0, 2.0])
    x = np.concatenate([
        v[None] * np.array([1, -1, 1, -1, 1, -1, 1, 1])[:, None],
        a[:, None] * v[None],
        np.zeros((3, D)),
        v[None] * 2.0,
        rng.standard_normal((4, D)),          # text
    ])
    off = np.array([0, 8, 15, 18, 19])
    n_vis = 19
    for p in (0.3, 0.6, 0.8):
        act = oracle.ffn_select(x, off, n_vis, p)
        k = math.ceil(p * 8)
        assert act[:8].tolist() == [True] * k + [False] * (8 - k)
        w = a / a.sum()
        want = _brute_top_p(w.tolist(), p)
        assert set(np.nonzero(act[8:15])[0].tolist()) == want
        assert act[15:18].all() and act[18] and act[19:].all()
    act = oracle.ffn_select(x, off, n_vis, 1e-9)
    assert np.nonzero(act[8:15])[0].tolist() == [5]     # the largest norm alone


def test_token_importance_closed_forms():
    """Tokens x_u = s_u v with |v| = 1 have norms s_u: the three normalisations
    have closed forms, and p = 0.5 tells them apart on s = (1, 2, 3, 4)."""
    s = np.array([1.0, 2.0, 3.0, 4.0])
    assert np.allclose(oracle.token_importance(s, "l2"), s / 10.0)
    assert np.allclose(oracle.token_importance(s, "l2sq"), s ** 2 / 30.0)
    e = np.exp(s - 4.0)
    assert np.allclose(oracle.token_importance(s, "softmax"), e / e.sum())
    assert oracle.token_importance(np.zeros(3), "l2") is None
    assert oracle.token_importance(np.zeros(3), "l2sq") is None
    assert np.allclose(oracle.token_importance(np.zeros(3), "softmax"), 1.0 / 3.0)
    with pytest.raises(ValueError):
        oracle.token_importance(s, "l1")
    v = np.zeros(6)
    v[2] = 1.0
    x = np.concatenate([s[:, None] * v[None], np.ones((2, 6))])     # one cube + 2 text
    off = np.array([0, 4])
    # l2: 0.4 < 0.5 -> {3, 2}; l2sq: 16/30 >= 0.5 -> {3}; softmax: 0.644 -> {3}
    for imp, want in (("l2", [2, 3]), ("l2sq", [3]), ("softmax", [3])):
        act = oracle.ffn_select(x, off, 4, 0.5, importance=imp)
        assert np.nonzero(act[:4])[0].tolist() == want, imp
        assert act[4:].all()
    # p = 0.85: l2 0.4+0.3+0.2 = 0.9 -> 3 tokens; l2sq 0.533+0.3+0.133 -> 3; softmax 0.644+0.237 -> 2
    for imp, n in (("l2", 3), ("l2sq", 3), ("softmax", 2)):
        assert oracle.ffn_select(x, off, 4, 0.85, importance=imp)[:4].sum() == n, imp


def test_token_ffn_dense_and_compensation():
    rng = np.random.default_rng(9)
    D, F = 16, 24
    off = np.array([0, 6, 7, 15, 22])       # cube 1 holds a single token
    n_vis, n_text = 22, 3
    N = n_vis + n_text
    x = rng.standard_normal((N, D)) * (1.0 + rng.random((N, 1)))
    Wg, Wu, Wd = (rng.standard_normal(s) * 0.3 for s in ((F, D), (F, D), (D, F)))
    full = x + _ffn_torch(x, Wg, Wu, Wd)
    y1, act1 = oracle.token_ffn(x, Wg, Wu, Wd, off, n_vis, 1.0)
    assert act1.all()
    assert np.abs(y1 - full).max() < 1e-12
    y, act = oracle.token_ffn(x, Wg, Wu, Wd, off, n_vis, 0.5)
    f = _ffn_torch(x, Wg, Wu, Wd)
    assert act[6] and np.abs(y[6] - full[6]).max() < 1e-12         # single-token cube
    assert np.abs(y[n_vis:] - full[n_vis:]).max() < 1e-12           # text unaffected by p
    for c in range(4):
        idx = np.arange(off[c], off[c + 1])
        A, S = idx[act[idx]], idx[~act[idx]]
        assert len(A) >= 1
        assert np.abs(y[A] - full[A]).max() < 1e-12
        if len(S):
            mbar = f[A].mean(axis=0)
            assert np.abs((y[S] - x[S]) - mbar[None]).max() < 1e-12   # y_k - x_k = m_bar
            assert np.abs(np.diff(y[S] - x[S], axis=0)).max() < 1e-12  # shared by the cube
    assert (~act[:n_vis]).any()


def test_linear_matches_explicit_sums():
    rng = np.random.default_rng(21)
    x = rng.standard_normal((5, 7))
    W = rng.standard_normal((3, 7))
    want = np.array([[sum(x[i, k] * W[j, k] for k in range(7)) for j in range(3)]
                     for i in range(5)])
    assert np.allclose(oracle.linear(x, W), want, rtol=0, atol=1e-12)


def test_rmsnorm_closed_forms():
    x = np.array([[2.0, -2.0, 2.0, -2.0], [3.0, 4.0, 0.0, 0.0]])
    out = oracle.rmsnorm(x, eps=0.0)
    assert np.allclose(out[0], [1, -1, 1, -1])
    assert np.allclose(out[1], np.array([3, 4, 0, 0]) / np.sqrt(25 / 4))
    assert np.allclose(np.mean(out ** 2, axis=1), 1.0)            # unit RMS
    assert np.allclose(oracle.rmsnorm(7.5 * x, eps=0.0), out)     # scale invariant
    w = np.array([1.0, 2.0, 0.5, 0.0])
    assert np.allclose(oracle.rmsnorm(x, w, eps=0.0), out * w)
    assert np.allclose(oracle.rmsnorm(np.zeros((1, 4)), eps=1e-6), 0.0)



# ---------------------------------------------------------------- backward (fixed sets)
def _central_diff(fn, arrays, eps=1e-6):
    """Gradient of the scalar fn(*arrays) w.r.t. every element of every array by
    central differences (float64)."""
    grads = []
    for a in arrays:
        g = np.zeros_like(a)
        it = np.nditer(a, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            old = a[i]
            a[i] = old + eps
            up = fn(*arrays)
            a[i] = old - eps
            dn = fn(*arrays)
            a[i] = old
            g[i] = (up - dn) / (2 * eps)
        grads.append(g)
    return grads


def _tiny_attn_case(seed, sel_density=0.5):
    rng = np.random.default_rng(seed)
    off = np.array([0, 3, 5, 8])
    n_vis, n_text, hq, hkv, d = 8, 2, 4, 2, 3
    N = n_vis + n_text
    Q, K, V = _qkv(rng, N, hq, hkv, d)
    sel = rng.random((N, hq, 3)) < sel_density
    dO = rng.standard_normal((N, hq, d))
    return off, n_vis, Q, K, V, sel, dO


@pytest.mark.parametrize("seed,density", [(21, 0.5), (22, 0.0), (23, 1.0)])
def test_attention_backward_equals_central_differences(seed, density):
    off, n_vis, Q, K, V, sel, dO = _tiny_attn_case(seed, density)

    def loss(Q, K, V):
        return float(np.sum(dO * oracle.attention_given_sets(Q, K, V, off, n_vis, sel)))

    want = _central_diff(loss, [Q.copy(), K.copy(), V.copy()])
    got = oracle.attention_backward_given_sets(Q, K, V, dO, off, n_vis, sel)
    for g, w in zip(got, want):
        assert np.abs(g - w).max() < 1e-7


def test_attention_backward_dense_equals_autograd():
    rng = np.random.default_rng(24)
    off = np.array([0, 5, 9, 16, 20, 27])
    n_vis, n_text, hq, hkv, d = 27, 6, 6, 2, 16
    N = n_vis + n_text
    g = hq // hkv
    Q, K, V = _qkv(rng, N, hq, hkv, d)
    dO = rng.standard_normal((N, hq, d))
    sel = np.ones((N, hq, len(off) - 1), dtype=bool)
    dQ, dK, dV = oracle.attention_backward_given_sets(Q, K, V, dO, off, n_vis, sel)
    q, k, v = (torch.from_numpy(a.copy()).requires_grad_() for a in (Q, K, V))
    causal = torch.ones(N, N, dtype=torch.bool).tril()
    o = Fn.scaled_dot_product_attention(
        q.permute(1, 0, 2)[None], k.repeat_interleave(g, dim=1).permute(1, 0, 2)[None],
        v.repeat_interleave(g, dim=1).permute(1, 0, 2)[None], attn_mask=causal)
    (o[0].permute(1, 0, 2) * torch.from_numpy(dO)).sum().backward()
    for got, t in ((dQ, q), (dK, k), (dV, v)):
        assert np.abs(got - t.grad.numpy()).max() < 1e-12


def test_attention_backward_sum_invariants():
    """Every row's probabilities sum to one and its dS sums to zero, so per KV
    head sum_j dV_j = sum of dO over the rows of its query heads and
    sum_j dK_j = 0, whatever the sets."""
    rng = np.random.default_rng(25)
    off = np.array([0, 4, 8, 12, 16, 20, 24])
    n_vis, n_text, hq, hkv, d = 24, 5, 4, 2, 8
    N = n_vis + n_text
    g = hq // hkv
    Q, K, V = _qkv(rng, N, hq, hkv, d)
    sel = rng.random((N, hq, len(off) - 1)) < 0.4
    dO = rng.standard_normal((N, hq, d))
    dQ, dK, dV = oracle.attention_backward_given_sets(Q, K, V, dO, off, n_vis, sel)
    for kv in range(hkv):
        assert np.abs(dV[:, kv].sum(0) - dO[:, kv * g:(kv + 1) * g].sum((0, 1))).max() < 1e-12
        assert np.abs(dK[:, kv].sum(0)).max() < 1e-12
    # the first token sees only itself: its dS is zero, so no query gradient
    assert np.abs(dQ[0]).max() < 1e-15
    # the magnitude sums bound the gradients, and equal them when every term is
    # positive (dV with dO > 0)
    *g, mags = oracle.attention_backward_given_sets(Q, K, V, dO, off, n_vis, sel,
                                                   with_magnitudes=True)
    for gg, mm in zip(g, mags):
        assert (np.abs(gg) <= mm + 1e-12).all()
    _, _, dVp, (_, _, mVp) = oracle.attention_backward_given_sets(
        Q, K, V, np.abs(dO), off, n_vis, sel, with_magnitudes=True)
    assert np.abs(dVp - mVp).max() < 1e-12


def test_backward_row_restrictions_agree_with_full():
    """Restricting the rows (cubes / text) gives the full result on those rows,
    and for the attention the full dK, dV on keys only those rows admit."""
    rng = np.random.default_rng(28)
    off = np.array([0, 4, 8, 12, 16, 20, 24])
    n_vis, n_text, hq, hkv, d = 24, 5, 4, 2, 8
    N = n_vis + n_text
    Q, K, V = _qkv(rng, N, hq, hkv, d)
    sel = rng.random((N, hq, len(off) - 1)) < 0.4
    dO = rng.standard_normal((N, hq, d))
    full = oracle.attention_backward_given_sets(Q, K, V, dO, off, n_vis, sel)
    part = oracle.attention_backward_given_sets(Q, K, V, dO, off, n_vis, sel, cubes=[5])
    rows = np.r_[20:24, n_vis:N]
    assert np.abs(part[0][rows] - full[0][rows]).max() < 1e-12
    assert not part[0][:20].any()
    for a, b in ((part[1], full[1]), (part[2], full[2])):
        assert np.abs(a[20:] - b[20:]).max() < 1e-12      # last cube's and text keys
    D, F = 6, 10
    x = rng.standard_normal((N, D))
    Wg, Wu, Wd = (rng.standard_normal(sh) * 0.5 for sh in ((F, D), (F, D), (D, F)))
    act = rng.random(N) < 0.6
    for c in range(len(off) - 1):
        act[off[c]] = True
    dy = rng.standard_normal((N, D))
    fdx = oracle.ffn_backward_given_sets(x, Wg, Wu, Wd, off, n_vis, act, dy)[0]
    pdx = oracle.ffn_backward_given_sets(x, Wg, Wu, Wd, off, n_vis, act, dy, cubes=[1, 3],
                                         text=False)[0]
    rows = np.r_[4:8, 12:16]
    assert np.abs(pdx[rows] - fdx[rows]).max() < 1e-12
    assert np.isnan(pdx[np.r_[0:4, 8:12, 16:N]]).all()


def test_ffn_backward_magnitudes_bound_the_gradients():
    """The rounding scales dominate the gradients they belong to (each is a sum
    of absolute values over the same terms, plus non-negative extras), and the
    dW_down scale is exactly twice |df|^T |h|."""
    off, n_vis, x, Wg, Wu, Wd, active, dy = _tiny_ffn_case(29)
    grads, mags = oracle.ffn_backward_given_sets(x, Wg, Wu, Wd, off, n_vis, active, dy,
                                                 with_magnitudes=True)
    plain = oracle.ffn_backward_given_sets(x, Wg, Wu, Wd, off, n_vis, active, dy)
    for g, p_, m in zip(grads, plain, mags):
        assert np.array_equal(g, p_)
    rows = active.copy()
    rows[n_vis:] = True
    assert (np.abs(grads[0] - dy)[rows] <= mags[0][rows] + 1e-12).all()
    for g, m in zip(grads[1:], mags[1:]):
        assert (np.abs(g) <= m + 1e-12).all()


def _tiny_ffn_case(seed):
    rng = np.random.default_rng(seed)
    D, F = 3, 4
    off = np.array([0, 3, 4, 7])
    n_vis, n_text = 7, 2
    N = n_vis + n_text
    x = rng.standard_normal((N, D))
    Wg, Wu, Wd = (rng.standard_normal(s) * 0.7 for s in ((F, D), (F, D), (D, F)))
    active = np.array([True, False, True, True, False, True, False, True, True])
    dy = rng.standard_normal((N, D))
    return off, n_vis, x, Wg, Wu, Wd, active, dy


def test_ffn_backward_equals_central_differences():
    off, n_vis, x, Wg, Wu, Wd, active, dy = _tiny_ffn_case(26)

    def loss(x, Wg, Wu, Wd):
        return float(np.sum(dy * oracle.ffn_given_sets(x, Wg, Wu, Wd, off, n_vis, active)))

    want = _central_diff(loss, [x.copy(), Wg.copy(), Wu.copy(), Wd.copy()])
    got = oracle.ffn_backward_given_sets(x, Wg, Wu, Wd, off, n_vis, active, dy)
    for g, w in zip(got, want):
        assert np.abs(g - w).max() < 1e-7


def test_ffn_backward_dense_equals_autograd_and_skipped_rows():
    rng = np.random.default_rng(27)
    D, F = 16, 24
    off = np.array([0, 6, 7, 15, 22])
    n_vis, n_text = 22, 3
    N = n_vis + n_text
    x = rng.standard_normal((N, D))
    Wg, Wu, Wd = (rng.standard_normal(s) * 0.3 for s in ((F, D), (F, D), (D, F)))
    dy = rng.standard_normal((N, D))
    got = oracle.ffn_backward_given_sets(x, Wg, Wu, Wd, off, n_vis, np.ones(N, bool), dy)
    t = [torch.from_numpy(a.copy()).requires_grad_() for a in (x, Wg, Wu, Wd)]
    y = t[0] + Fn.linear(Fn.silu(Fn.linear(t[0], t[1])) * Fn.linear(t[0], t[2]), t[3])
    (y * torch.from_numpy(dy)).sum().backward()
    for g, tt in zip(got, t):
        assert np.abs(g - tt.grad.numpy()).max() < 1e-11
    # sparse set: a skipped token's own gradient is dy; the cube's active tokens
    # share sum(dy_skipped) / |active| on top of their own dy
    active = rng.random(N) < 0.5
    active[[0, 6, 7, 15]] = True
    dx, _, _, _ = oracle.ffn_backward_given_sets(x, Wg, Wu, Wd, off, n_vis, active, dy)
    skipped = ~active
    skipped[n_vis:] = False
    assert np.array_equal(dx[skipped], dy[skipped])
    # W_down = 0: the FFN's input and gate gradients vanish
    Wd0 = np.zeros_like(Wd)
    dx0, dWg0, _, dWd0 = oracle.ffn_backward_given_sets(x, Wg, Wu, Wd0, off, n_vis, active, dy)
    assert np.array_equal(dx0, dy) and not dWg0.any()
    # dW_down collects h^T df: with the compensation term for cube 0 checked by hand
    a0 = np.nonzero(active[:6])[0]
    s0 = np.nonzero(~active[:6])[0]
    df0 = dy[a0] + dy[s0].sum(0) / len(a0)
    gate, up = x[a0] @ Wg.T, x[a0] @ Wu.T
    h = gate / (1 + np.exp(-gate)) * up
    _, _, _, dWd_c0 = oracle.ffn_backward_given_sets(x[:6], Wg, Wu, Wd, off[:2], 6, active[:6],
                                                     dy[:6])
    assert np.abs(dWd_c0 - df0.T @ h).max() < 1e-12


# ---------------------------------------------------------------- rounding scales, from above
# The rounding scales returned with ``with_magnitudes`` widen the GPU gradient
# bound, so an inflated scale would loosen the comparison. Above, they are
# pinned from below (they dominate the gradients). Here they are pinned from
# above: in cases where every term of a gradient element has one sign the
# scale must equal the gradient's magnitude (attention) or exactly twice it
# (FFN, where two roundings enter each term), so a scale inflated by any factor
# fails; and each attention scale is compared with its sum of absolute terms
# written out one term at a time.

def test_attention_magnitudes_equal_gradients_for_single_terms():
    """Query row 1 of cube 0 admits keys 0 and 1; with K_1 = 0 its dQ has the
    single term dS_10 K_0 / sqrt(d), so mQ = |dQ| there. The last key of the
    last cube (no text, one query head per KV head) is admitted by its own row
    only, so mK = |dK| there. With dO > 0 every P^T dO term is positive, so
    mV = dV everywhere."""
    rng = np.random.default_rng(31)
    off = np.array([0, 2, 4, 7])
    n_vis, hq, hkv, d = 7, 2, 2, 5
    Q, K, V = _qkv(rng, n_vis, hq, hkv, d)
    K[1] = 0.0                 # row 1 sees keys {0, 1}: only key 0 contributes to dQ
    K[4] = 0.0                 # row 5 (cube 2, second token) sees {4, 5} + selections
    sel = np.zeros((n_vis, hq, 3), dtype=bool)
    dO = rng.standard_normal((n_vis, hq, d))
    dQ, dK, dV, (mQ, mK, mV) = oracle.attention_backward_given_sets(
        Q, K, V, dO, off, n_vis, sel, with_magnitudes=True)
    for t in (1, 5):
        assert np.abs(dQ[t]).min() > 1e-6                 # the case is not degenerate
        np.testing.assert_allclose(mQ[t], np.abs(dQ[t]), rtol=1e-12, atol=0)
    np.testing.assert_allclose(mK[n_vis - 1], np.abs(dK[n_vis - 1]), rtol=1e-12, atol=0)
    assert np.abs(dK[n_vis - 1]).min() > 1e-6
    _, _, dVp, (_, _, mVp) = oracle.attention_backward_given_sets(
        Q, K, V, np.abs(dO) + 0.1, off, n_vis, sel, with_magnitudes=True)
    np.testing.assert_allclose(mVp, dVp, rtol=1e-12, atol=0)


def test_attention_magnitudes_term_by_term():
    """mQ, mK and mV equal their sums of absolute terms, taken one (row, key)
    term at a time; the row's probabilities are read from the pinned forward
    (one-hot values make the output the probability vector itself)."""
    rng = np.random.default_rng(32)
    off = np.array([0, 3, 5, 8])
    n_vis, n_text, hq, hkv, d = 8, 2, 4, 2, 3
    N = n_vis + n_text
    g = hq // hkv
    Q, K, V = _qkv(rng, N, hq, hkv, d)
    sel = rng.random((N, hq, 3)) < 0.5
    dO = rng.standard_normal((N, hq, d))
    *_, (mQ, mK, mV) = oracle.attention_backward_given_sets(Q, K, V, dO, off, n_vis, sel,
                                                            with_magnitudes=True)
    # P[t, h, u] from the forward with one-hot values (head dim N for V)
    onehot = np.zeros((N, hkv, N))
    for u in range(N):
        onehot[u, :, u] = 1.0
    Qp = np.zeros((N, hq, N))
    Kp = np.zeros((N, hkv, N))
    Qp[:, :, :d] = Q * math.sqrt(N / d)     # same logits at head dim N
    Kp[:, :, :d] = K
    P = oracle.attention_given_sets(Qp, Kp, onehot, off, n_vis, sel)
    wQ, wK, wV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    for t in range(N):
        for h in range(hq):
            kv = h // g
            dP = [float(dO[t, h] @ V[u, kv]) for u in range(N)]
            D = sum(P[t, h, u] * dP[u] for u in range(N))
            for u in range(N):
                if P[t, h, u] == 0.0:
                    continue
                dS = P[t, h, u] * (dP[u] - D)
                for c in range(d):
                    wQ[t, h, c] += abs(dS) * abs(K[u, kv, c]) / math.sqrt(d)
                    wK[u, kv, c] += abs(dS) * abs(Q[t, h, c]) / math.sqrt(d)
                    wV[u, kv, c] += P[t, h, u] * abs(dO[t, h, c])
    for m, w in ((mQ, wQ), (mK, wK), (mV, wV)):
        np.testing.assert_allclose(m, w, rtol=1e-9, atol=1e-12)


def test_ffn_magnitudes_twice_the_gradients_when_terms_are_positive():
    """With x, the three weights and dy all positive, every term of every
    gradient is positive, and each rounding scale counts each term twice (df and
    dg / du / h each rounded once): the scales equal exactly twice the
    gradients (dx without its dy part)."""
    rng = np.random.default_rng(33)
    D, F = 5, 7
    off = np.array([0, 3, 4, 8])
    n_vis, n_text = 8, 2
    N = n_vis + n_text
    x = rng.random((N, D)) + 0.1
    Wg, Wu, Wd = (rng.random(s) * 0.5 + 0.05 for s in ((F, D), (F, D), (D, F)))
    active = np.array([True, False, True, True, True, False, True, False, True, True])
    dy = rng.random((N, D)) + 0.1
    (dx, dWg, dWu, dWd), (mdx, mWg, mWu, mWd) = oracle.ffn_backward_given_sets(
        x, Wg, Wu, Wd, off, n_vis, active, dy, with_magnitudes=True)
    rows = active.copy()
    rows[n_vis:] = True
    np.testing.assert_allclose(mdx[rows], 2.0 * (dx - dy)[rows], rtol=1e-12, atol=0)
    assert not mdx[~rows].any()
    for m, gr in ((mWg, dWg), (mWu, dWu), (mWd, dWd)):
        assert gr.min() > 0.0
        np.testing.assert_allclose(m, 2.0 * gr, rtol=1e-12, atol=0)


def test_select_cubes_with_given_means_is_the_same_selection():
    """Passing the layer's cube means (computed once per layer) changes nothing."""
    rng = np.random.default_rng(34)
    off = np.array([0, 4, 8, 12, 16, 20])
    Q, K, _ = _qkv(rng, 24, 4, 2, 8)
    a, ma = oracle.select_cubes(Q, K, off, 20, 4, 2, 0.6, with_margin=True)
    b, mb = oracle.select_cubes(Q, K, off, 20, 4, 2, 0.6, with_margin=True,
                                kbar=oracle.cube_mean_keys(K, off))
    assert np.array_equal(a, b) and np.array_equal(ma, mb)


# ---------------------------------------------------------------- Uniform Sampling
def test_uniform_cubes_hand_values():
    """k of the i preceding cubes at even spacing from the first (floor(m i / k)),
    all of them when i <= k, none for the first cube."""
    assert oracle.uniform_cubes(10, 3).tolist() == [0, 3, 6]
    assert oracle.uniform_cubes(7, 7).tolist() == list(range(7))
    assert oracle.uniform_cubes(3, 5).tolist() == [0, 1, 2]
    assert oracle.uniform_cubes(0, 4).tolist() == []
    assert oracle.uniform_cubes(1000, 4).tolist() == [0, 250, 500, 750]
    with pytest.raises(ValueError):
        oracle.uniform_cubes(5, 0)


@pytest.mark.parametrize("i,k", [(i, k) for i in range(1, 40) for k in (1, 2, 3, 5, 8, 13)])
def test_uniform_cubes_even_spacing(i, k):
    """min(i, k) distinct ascending preceding cubes, starting at cube 0, whose gaps
    (including the one up to cube i) are floor(i/k) or ceil(i/k)."""
    j = oracle.uniform_cubes(i, k)
    assert len(j) == min(i, k) and len(set(j.tolist())) == len(j)
    assert (np.diff(j) > 0).all() and j[0] == 0 and j[-1] < i
    if i > k:
        gaps = np.diff(np.append(j, i))
        assert gaps.min() >= i // k and gaps.max() <= -(-i // k)


def test_select_cubes_uniform_shares_the_set_across_heads_and_tokens():
    off = np.array([0, 3, 5, 9, 12, 16])
    sel = oracle.select_cubes_uniform(off, 16, 4, 2)
    for t in range(16):
        c = int(np.searchsorted(off, t, side="right") - 1)
        want = np.zeros(5, bool)
        want[oracle.uniform_cubes(c, 2)] = True
        for h in range(4):
            assert np.array_equal(sel[t, h], want)
