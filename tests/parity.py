"""Helpers of the GPU parity tests: build a seeded layer on the device, run the
library through its C ABI, run the oracle on the same values, compare.

Comparison protocol:
* selection sets (cube sets of AdaS-Attn, active tokens of AdaS-FFN) must equal
  the oracle's bit for bit, except where the oracle's cut margin is below 1e-5;
  those cases are counted and reported, not required to match;
* outputs are compared with the oracle run on the library's own sets
  (``attention_given_sets`` / ``ffn_given_sets``), so arithmetic error and
  selection error are judged separately; bf16: max-abs 2e-2 and rel-L2 5e-3;
  fp32: max-abs 1e-4 and rel-L2 1e-5.  An output stored in bf16 (the
  attention output) cannot be closer to the exact value than its own rounding:
  where |ref| >= 8 half a bf16 ulp alone (1/32 and more) exceeds 2e-2, so
  there the bound is |err| <= 2e-2 + 1 ulp_bf16(|ref|); below 8 half an ulp is
  at most 1/64 and the plain 2e-2 applies.
"""
from __future__ import annotations

import numpy as np
import torch

import ffn_long_video_b200 as fb
import oracle
import workloads

MARGIN = 1e-5
TOL = {"bf16": (2e-2, 5e-3), "fp32": (1e-4, 1e-5)}

# One entry per selection check (rows or cubes compared, how many of them lie
# within MARGIN of a cut flip, and how many of those the library decided
# otherwise); tests/conftest.py writes the list to the file named by
# ADASPARK_PARITY_RECORD at the end of the session.
RECORD = []


def _record(kind, cfg, p, k, units, near, near_mismatch):
    RECORD.append({"kind": kind, "config": cfg.name, "p": None if k is not None else float(p),
                   "k": k, "units": int(units), "near_margin": int(near),
                   "near_margin_mismatch": int(near_mismatch)})


def near_cut_ok(P, chosen, p, k=None):
    """Whether a set that differs from the oracle's at a near-margin cut is still
    a valid near-cut of the probability vector P (float64, the oracle's):
    Top-p: its mass reaches p - MARGIN and its size is within one of the
    oracle's k*; Top-K: it has min(k, len(P)) entries whose mass is within
    MARGIN of the oracle's Top-K mass."""
    P = np.asarray(P, dtype=np.float64)
    chosen = np.asarray(chosen, dtype=bool)
    if k is not None:
        want = oracle.top_k(P, k)
        return chosen.sum() == want.sum() and P[chosen].sum() >= P[want].sum() - MARGIN
    kstar = int(oracle.top_p(P, p).sum())
    return P[chosen].sum() >= p - MARGIN and abs(int(chosen.sum()) - kstar) <= 1


def layout_tensors(cfg, device="cuda"):
    sizes = cfg.sizes
    ids = np.concatenate([np.repeat(np.arange(cfg.n_cubes, dtype=np.int32), sizes),
                          np.full(cfg.n_text, -1, np.int32)])
    off = cfg.offsets
    t_ids = torch.from_numpy(ids).to(device)
    t_off = torch.from_numpy(off).to(device)
    t_text = torch.from_numpy((ids == -1).astype(np.uint8)).to(device)
    return t_ids, t_off, t_text, off


def make_case(cfg, layer=0):
    dev = "cuda"
    lay = workloads.make_layer(cfg, layer=layer, project_on=dev)
    lay = {k: v.to(dev) for k, v in lay.items()}
    ids, off, text, off_np = layout_tensors(cfg, dev)
    return {"cfg": cfg, "t": lay, "ids": ids, "off": off, "text": text, "off_np": off_np}


def errors(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    diff = got - want
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(want), 1e-300))
    return max_abs, rel


def ulp_bf16(x):
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    a = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


BF16_ULP_FROM = 8.0   # |ref| from which half a bf16 ulp (>= 1/32) exceeds 2e-2


def excess_over_bf16(got, want):
    """max of |got - want| - allowance, where the allowance is one bf16 ulp of
    the reference for |want| >= 8 and zero below (half an ulp there is at most
    1/64, inside 2e-2): compared with the plain 2e-2 bound."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    if not got.size:
        return 0.0
    allow = np.where(np.abs(want) >= BF16_ULP_FROM, ulp_bf16(want), 0.0)
    return float((np.abs(got - want) - allow).max())


def run_attn(case, p=None, k=None, train=False, uniform=None):
    """Run AdaS-Attn (Top-p, or Top-K when k is given, or Uniform Sampling of
    ``uniform`` cubes; the training-mode call when ``train``) and export its
    sets."""
    cfg, t = case["cfg"], case["t"]
    p = cfg.p if p is None else p
    if uniform is not None:
        out, ws = fb.cube_attn_uniform(t["Q"], t["K"], t["V"], case["ids"], case["off"],
                                       cfg.n_vis, uniform)
    elif k is None:
        out, ws = fb.cube_attn(t["Q"], t["K"], t["V"], case["ids"], case["off"], cfg.n_vis, p,
                               train=train)
    else:
        out, ws = fb.cube_attn_topk(t["Q"], t["K"], t["V"], case["ids"], case["off"], cfg.n_vis,
                                    k)
    torch.cuda.synchronize()
    code, detail = fb.read_device_status(ws)
    assert code == fb.OK, (code, detail)
    sel = fb.attn_export_sets(ws, case["ids"], cfg.n_cubes, cfg.n_vis, cfg.n_tokens, cfg.hq,
                              cfg.hkv, cfg.d, fb.BF16 if cfg.dtype == "bf16" else fb.FP32)
    return out, sel, ws


def check_attn(case, p=None, tokens=None, report=None, k=None, train=False, uniform=None):
    """Selection parity + output parity of AdaS-Attn on ``tokens`` (default all);
    Top-K selection when ``k`` is given, Uniform Sampling of ``uniform`` cubes
    (integer sets, compared exactly) when that is given; the training-mode call
    when ``train``."""
    cfg, t = case["cfg"], case["t"]
    p = cfg.p if p is None else p
    out, gsel, ws = run_attn(case, p, k, train, uniform)
    Qc, Kc, Vc = (t[k].cpu() for k in ("Q", "K", "V"))
    off = case["off_np"]
    if tokens is None:
        tokens = np.arange(cfg.n_tokens)
    tokens = np.asarray(tokens)
    vis = tokens[tokens < cfg.n_vis]
    if uniform is not None:
        osel = oracle.select_cubes_uniform(off, cfg.n_vis, cfg.hq, uniform, tokens=vis)
        margin = np.full(osel.shape[:2], np.inf)
    else:
        osel, margin = oracle.select_cubes(Qc, Kc, off, cfg.n_vis, cfg.hq, cfg.hkv, p,
                                           tokens=vis, with_margin=True, k=k)
    g = gsel[vis]
    diff_rows = (osel != g).any(axis=2)
    near = margin < MARGIN
    bad = diff_rows & ~near
    n_near_mismatch = int((diff_rows & near).sum())
    assert not bad.any(), f"{int(bad.sum())} selection mismatches outside the margin " \
                          f"(first at {np.argwhere(bad)[:3].tolist()})"
    if n_near_mismatch:
        # the library's set on a near-margin row must still be a valid near-cut
        kbar = oracle.cube_mean_keys(Kc, off)
        g_of = cfg.hq // cfg.hkv
        Qf = Qc.double().numpy()
        for r, h in np.argwhere(diff_rows & near):
            tok = int(vis[r])
            c = int(np.searchsorted(off, tok, side="right") - 1)
            P = oracle.softmax(oracle.cube_scores(Qf[tok, h], kbar[:c, h // g_of], cfg.d))
            assert near_cut_ok(P, g[r, h, :c], p, k), (tok, int(h))
    if uniform is None:
        _record("attn", cfg, p, k, g.shape[0] * g.shape[1], near.sum(), n_near_mismatch)
    # outputs against the oracle on the library's own sets
    sel_full = np.zeros((len(tokens), cfg.hq, cfg.n_cubes), dtype=bool)
    is_vis = tokens < cfg.n_vis
    sel_full[is_vis] = gsel[tokens[is_vis]]
    want = oracle.attention_given_sets(Qc, Kc, Vc, off, cfg.n_vis, sel_full, tokens=tokens)
    got = out.float().cpu().numpy()[tokens]
    max_abs, rel = errors(got, want)
    tol_abs, tol_rel = TOL[cfg.dtype]
    # bf16 output: one ulp of the output format on top of the bound where
    # |ref| >= 8, the plain bound below
    worst = excess_over_bf16(got, want) if cfg.dtype == "bf16" else max_abs
    if report is not None:
        report.update(max_abs=max_abs, excess_over_ulp=worst, rel_l2=rel,
                      near_margin_rows=int(near.sum()), near_margin_mismatch=n_near_mismatch,
                      rows=int(g.shape[0] * g.shape[1]))
    assert worst <= tol_abs and rel <= tol_rel, (max_abs, worst, rel)
    return out, gsel, ws


IMPORTANCE_CODES = {"l2": fb.IMPORTANCE_L2_SHARE, "l2sq": fb.IMPORTANCE_L2SQ_SHARE,
                    "softmax": fb.IMPORTANCE_SOFTMAX}


def run_ffn(case, p=None, importance="l2"):
    cfg, t = case["cfg"], case["t"]
    p = cfg.p if p is None else p
    y, ws = fb.token_ffn(t["x"], t["W_gate"], t["W_up"], t["W_down"], case["ids"], case["off"],
                         case["text"], cfg.n_vis, p, importance=IMPORTANCE_CODES[importance])
    torch.cuda.synchronize()
    code, detail = fb.read_device_status(ws)
    assert code == fb.OK, (code, detail)
    act = fb.ffn_export_active(ws, cfg.n_tokens, cfg.n_vis, cfg.n_cubes, cfg.D, cfg.F,
                               fb.BF16 if cfg.dtype == "bf16" else fb.FP32)
    return y, act, ws


def check_ffn(case, p=None, cubes=None, text=True, report=None, importance="l2"):
    cfg, t = case["cfg"], case["t"]
    p = cfg.p if p is None else p
    y, gact, ws = run_ffn(case, p, importance)
    x = t["x"].cpu()
    off = case["off_np"]
    if cubes is None:
        cubes = np.arange(cfg.n_cubes)
    oact, margins = oracle.ffn_select(x, off, cfg.n_vis, p, cubes=cubes, with_margin=True,
                                      importance=importance)
    bad_cubes, near_mismatch = [], 0
    for c in cubes:
        a, b = off[c], off[c + 1]
        if not np.array_equal(oact[a:b], gact[a:b]):
            if margins[c] < MARGIN:
                near_mismatch += 1
                # the library's active set must still be a valid near-cut
                Xc = x[a:b].double().numpy()
                w = oracle.token_importance(np.sqrt((Xc * Xc).sum(axis=1)), importance)
                assert w is not None and near_cut_ok(w, gact[a:b], p), int(c)
            else:
                bad_cubes.append(int(c))
    assert not bad_cubes, f"active-set mismatch outside the margin in cubes {bad_cubes[:5]}"
    _record("ffn", cfg, p, None, len(cubes), (margins[cubes] < MARGIN).sum(), near_mismatch)
    assert gact[cfg.n_vis:].all()
    want = oracle.ffn_given_sets(x, t["W_gate"].cpu(), t["W_up"].cpu(), t["W_down"].cpu(), off,
                                 cfg.n_vis, gact, cubes=cubes, text=text)
    rows = np.isfinite(want[:, 0])
    got = y.cpu().numpy()
    max_abs, rel = errors(got[rows], want[rows])
    tol_abs, tol_rel = TOL[cfg.dtype]
    if report is not None:
        report.update(max_abs=max_abs, rel_l2=rel,
                      near_margin_cubes=int((margins[cubes] < MARGIN).sum()),
                      near_margin_mismatch=near_mismatch)
    assert max_abs <= tol_abs and rel <= tol_rel, (max_abs, rel)
    return y, gact, ws


# ----------------------------------------------------------------- backward
# Gradients have no unit scale of their own, so the bf16 bar is applied to the
# gradient measured in units of its own RMS, with the same one-ulp allowance as
# the bf16 outputs of the forward: per element |err| <= 2e-2 * rms(ref) +
# ulp_bf16(|ref|), and rel-L2 <= 5e-3. The ulp term covers sums whose terms
# share a sign (tokens of one cube are near-duplicates), where the bf16
# rounding of an operand (dS, P, df, dg, du, h) adds up in proportion to the
# sum itself instead of averaging out.
GRAD_TOL = (2e-2, 5e-3)


# For sums that round an operand to bf16 (dS or P in the attention gradients;
# df, dg, du, h in the FFN ones) a rigorous per-element bound also holds: RNE
# to 8 significant bits moves a value by at most 2^-9 of itself, so |err| <=
# 2^-9 times the oracle's rounding scale (sum |a| |b| over the element's terms,
# with an upstream rounding carried through, e.g. df's into dg); 2^-8 leaves
# room for the fp32 accumulation, the ex2 approximation and the recomputed
# softmax (the backward's P and dS are formed again from fp32 scores): over the
# whole GPU suite the largest error measured is 0.00348 of the scale (dQ) and
# 0.00337 (dV), about 1.8 times 2^-9, so 2^-9 alone would be too tight. It
# matters where the terms nearly cancel (each row's dS sums to zero; the rows
# of one cube are near-duplicates), which makes the gradient small next to its
# terms.
ROUND_BOUND = 2.0 ** -8


def check_grad(got, want, what, report=None, magnitude=None):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    rms = float(np.sqrt(np.mean(want * want))) if want.size else 0.0
    max_abs, rel = errors(got, want)
    bound = GRAD_TOL[0] * rms + ulp_bf16(want)
    scale_ratio = None
    if magnitude is not None:
        mag = np.asarray(magnitude, dtype=np.float64)
        bound = np.maximum(bound, ROUND_BOUND * mag)
        # the largest error in units of the rounding scale (the rounding alone
        # allows 2^-9 of it); elements with a zero scale are left out
        nz = mag > 0
        scale_ratio = float((np.abs(got - want)[nz] / mag[nz]).max()) if nz.any() else 0.0
    excess = (np.abs(got - want) - bound).max() if want.size else 0.0
    if report is not None:
        report[what] = {"max_abs": max_abs, "rms_ref": rms,
                        "max_over_rms": max_abs / rms if rms > 0 else max_abs,
                        "worst_excess": float(excess), "rel_l2": rel,
                        "max_err_over_scale": scale_ratio}
    assert excess <= 0.0 and rel <= GRAD_TOL[1], (what, max_abs, rms, float(excess), rel)


def run_ffn_backward(case, p=None):
    """Forward AdaS-FFN, then its backward for the case's seeded dy; returns the
    library's gradients, the forward's active set and dy."""
    cfg, t = case["cfg"], case["t"]
    _, act, fws = run_ffn(case, p)
    dy = workloads.make_upstream(cfg)["dy"].to(t["x"].device)
    dx, dWg, dWu, dWd, bws = fb.token_ffn_backward(t["W_gate"], t["W_up"], t["W_down"],
                                                   case["off"], cfg.n_vis, dy, fws)
    torch.cuda.synchronize()
    code, detail = fb.read_device_status(bws)
    assert code == fb.OK, (code, detail)
    return (dx, dWg, dWu, dWd), act, dy


def check_ffn_backward(case, p=None, report=None):
    cfg, t = case["cfg"], case["t"]
    grads, act, dy = run_ffn_backward(case, p)
    want, mags = oracle.ffn_backward_given_sets(t["x"].cpu(), t["W_gate"].cpu(),
                                                t["W_up"].cpu(), t["W_down"].cpu(),
                                                case["off_np"], cfg.n_vis, act, dy.cpu(),
                                                with_magnitudes=True)
    for g, w, m, nm in zip(grads, want, mags, ("dx", "dW_gate", "dW_up", "dW_down")):
        check_grad(g.cpu().numpy(), w, nm, report, magnitude=m)
    # a skipped token's gradient is its upstream gradient, bit for bit
    skipped = ~act
    skipped[cfg.n_vis:] = False
    assert torch.equal(grads[0].cpu()[torch.from_numpy(skipped)],
                       dy.cpu()[torch.from_numpy(skipped)])
    return grads, act


def run_attn_backward(case, p=None, k=None, train=False):
    """Forward AdaS-Attn (Top-p, or Top-K when k is given; training mode when
    ``train``), then its backward for the case's seeded dO; returns the
    library's gradients, the forward's sets [N, hq, C] (text rows False) and dO."""
    cfg, t = case["cfg"], case["t"]
    out, sel, fws = run_attn(case, p, k, train)
    dO = workloads.make_upstream(cfg)["dO"].to(t["Q"].device)
    dQ, dK, dV, bws = fb.cube_attn_backward(t["Q"], t["K"], t["V"], dO, case["ids"],
                                            case["off"], cfg.n_vis, fws)
    torch.cuda.synchronize()
    code, detail = fb.read_device_status(bws)
    assert code == fb.OK, (code, detail)
    sets = np.zeros((cfg.n_tokens, cfg.hq, cfg.n_cubes), dtype=bool)
    sets[:cfg.n_vis] = sel[:cfg.n_vis]
    return (dQ, dK, dV), sets, dO, (out, fws)


def check_attn_backward(case, p=None, k=None, report=None, train=False):
    cfg, t = case["cfg"], case["t"]
    grads, sets, dO, _ = run_attn_backward(case, p, k, train)
    *want, mags = oracle.attention_backward_given_sets(
        t["Q"].cpu(), t["K"].cpu(), t["V"].cpu(), dO.cpu(), case["off_np"], cfg.n_vis, sets,
        with_magnitudes=True)
    for g, w, m, nm in zip(grads, want, mags, ("dQ", "dK", "dV")):
        check_grad(g.cpu().numpy(), w, nm, report, magnitude=m)
    return grads, sets
