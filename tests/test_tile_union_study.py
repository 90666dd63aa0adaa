"""Why the attention tiles are 128 tokens of one query head, and why the
library keeps one cube set per (token, query head) rather than one per KV
group: measured on the oracle's own sets (CPU, float64) for a slice of a
16K-token grid of the 7B head shape (28 query / 4 KV heads, head_dim 128,
hidden 3584, 4x4x4 cubes, per-cube noise U(0.1, 1.0), p = 0.7).

A 128-row tile executes the union of its rows' cube sets: every key block
that any row takes runs for all 128 rows. Measured here:
* executed / useful work of the library's tiles (128 tokens x 1 head);
* the other row groupings of one KV group that keep 128 rows (64 tokens x 2
  heads, 32 x 4, 16 x 8), and 64-token single-head tiles, which would need
  M = 64 products;
* one set per KV group from the group's mean query (the GQA-shared variant):
  more selected pairs, and more executed blocks;
* the split walk: the cubes that at most 8 of a tile's rows chose, moved to
  gathered tiles, are many blocks but few pairs.
The numbers printed are the figures quoted in the design notes."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads

P = 0.7
CFG = workloads.LayerConfig(name="union-16k", grid=(16, 32, 32), cube=(4, 4, 4), n_text=0,
                            D=3584, hq=28, hkv=4, d=128, F=128, dtype="bf16", p=P,
                            sigma=None, sigma_range=(0.1, 1.0), seed=workloads.BASE_SEED + 3)
SLICE = (192, 208)      # cubes whose tokens are the query rows (late in the grid)


@pytest.fixture(scope="module")
def study():
    rng = workloads.layer_rng(CFG, 0)
    x = workloads.make_hidden(CFG, rng)
    w = workloads.make_weights(CFG, rng)     # W_q, W_k first: the same draws for any F
    xb = workloads._round(x, "bf16")
    qkv = workloads.project_qkv(CFG, xb, workloads._round(w["W_q"], "bf16"),
                                workloads._round(w["W_k"], "bf16"),
                                workloads._round(w["W_v"], "bf16"))
    off = CFG.offsets
    t0, t1 = off[SLICE[0]], off[SLICE[1]]
    tokens = np.arange(t0, t1)
    K = qkv["K"]
    kbar = oracle.cube_mean_keys(K, off)
    sel = oracle.select_cubes(qkv["Q"], K, off, CFG.n_vis, CFG.hq, CFG.hkv, P, tokens=tokens,
                              kbar=kbar)
    own = np.searchsorted(off, tokens, side="right") - 1
    sel[np.arange(len(tokens)), :, own] = True           # the own cube is always attended
    # one set per KV group from the group's mean query
    g = CFG.hq // CFG.hkv
    Qf = qkv["Q"].double().numpy()[tokens]
    shared = np.zeros_like(sel)
    for r, c in enumerate(own):
        for kv in range(CFG.hkv):
            qm = Qf[r, kv * g:(kv + 1) * g].mean(axis=0)
            Pm = oracle.softmax(oracle.cube_scores(qm, kbar[:c, kv], CFG.d))
            s = np.zeros(CFG.n_cubes, bool)
            s[:c] = oracle.top_p(Pm, P)
            s[c] = True
            shared[r, kv * g:(kv + 1) * g] = s
    return sel, shared


def _executed(sel, tok_per_tile, heads_per_tile):
    """128-row block-equivalents executed: per tile, the union of its rows'
    cubes, each weighted by the tile's rows / 128."""
    g = CFG.hq // CFG.hkv
    T = sel.shape[0]
    total = 0.0
    for kv in range(CFG.hkv):
        for h0 in range(kv * g, (kv + 1) * g, heads_per_tile):
            hs = list(range(h0, min(h0 + heads_per_tile, (kv + 1) * g)))
            for s0 in range(0, T, tok_per_tile):
                u = sel[s0:s0 + tok_per_tile][:, hs].any(axis=(0, 1))
                total += u.sum() * len(hs) * min(tok_per_tile, T - s0) / 128.0
    return total


def test_tile_unions(study):
    sel, shared = study
    useful = sel.sum() / 128.0                  # 64-key blocks x rows / 128
    t128 = _executed(sel, 128, 1)
    t64x2 = _executed(sel, 64, 2)
    t32x4 = _executed(sel, 32, 4)
    t16x8 = _executed(sel, 16, 8)
    t64 = _executed(sel, 64, 1)
    print(f"useful {useful:.0f}; 128x1 {t128:.0f}; 64x2 {t64x2:.0f}; 32x4 {t32x4:.0f}; "
          f"16x8 {t16x8:.0f}; 64x1 (M = 64) {t64:.0f}")
    # the union inflation is structural: rows of one cube select differently
    assert t128 / useful > 3.0
    # no 128-row grouping of one KV group does markedly better than 128 x 1
    assert min(t64x2, t32x4, t16x8) > 0.9 * t128
    # 64-row tiles would cut executed work, but only with M = 64 products
    assert t64 < 0.85 * t128


def test_group_shared_sets(study):
    sel, shared = study
    pairs, pairs_shared = sel.sum(), shared.sum()
    t128, t_shared = _executed(sel, 128, 1), _executed(shared, 128, 1)
    print(f"selected pairs per head {pairs}, group-shared {pairs_shared} "
          f"({pairs_shared / pairs:.2f}x); executed 128x1 {t128:.0f} vs {t_shared:.0f}")
    # the averaged query's softmax over cubes is flatter: many more pairs, and
    # no fewer executed blocks than per-head sets
    assert pairs_shared > 1.8 * pairs
    assert t_shared > 0.95 * t128


def test_split_walk_study(study):
    """The split walk on the oracle's sets: a tile's cubes below its lowest own
    cube that at most 8 of its 128 rows chose leave the tile's walk and run in
    gathered 128-row tiles per (KV head, cube). Most of the blocks such cubes
    cost move out, with only a small share of the selected pairs."""
    sel, _ = study
    T, hq, C = sel.shape
    off = CFG.offsets
    g = hq // CFG.hkv
    base = off[SLICE[0]]
    tiles = blocks = kept = moved_pairs = pairs = 0
    warps_all = warps_moved = 0
    groups = {}
    for h in range(hq):
        for s0 in range(0, T, 128):
            rows = sel[s0:s0 + 128, h]                    # [128, C]
            c_lo = int(np.searchsorted(off, base + s0, side="right") - 1)
            r = rows.sum(axis=0)
            w = np.array([rows[q:q + 32].any(axis=0) for q in range(0, rows.shape[0], 32)]).sum(0)
            tiles += 1
            for j in np.nonzero(r)[0]:
                blocks += 1
                pairs += int(r[j])
                warps_all += int(w[j])
                if j < c_lo and r[j] <= 8:
                    moved_pairs += int(r[j])
                    warps_moved += int(w[j])
                    key = (h // g, int(j))
                    groups[key] = groups.get(key, 0) + int(r[j])
                else:
                    kept += 1
    gathered = sum(math.ceil(n / 128) for n in groups.values())
    print(f"tiles {tiles}: blocks {blocks} -> kept {kept} + gathered {gathered}; "
          f"pairs moved {moved_pairs / pairs:.3f}; warp-blocks moved "
          f"{warps_moved / warps_all:.3f}")
    # the moved blocks are many, their pairs few, and the gathered tiles pack them
    assert kept + gathered < 0.8 * blocks
    assert moved_pairs < 0.15 * pairs
    assert warps_moved > 2.0 * moved_pairs / pairs * warps_all
