"""Hand-worked fixtures under tests/golden/ (each file states its source passage
and readings): cube partitions, Top-p cuts with ties and exact cumulative
masses, and AdaS-FFN token selection. They pin the oracle to values derived
from the definitions rather than from its own code, and the host partition of
the C ABI to the same values."""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.lstrip().startswith("#")]


def _partition_cases():
    cases, cur = [], None
    for ln in _lines("partition.txt"):
        key, _, rest = ln.partition(" ")
        if key == "case":
            cur = {k: int(v) for k, v in (kv.split("=") for kv in rest.split())}
            cases.append(cur)
        else:
            cur[key] = np.array([int(v) for v in rest.split()], np.int32)
    return cases


@pytest.mark.parametrize("case", _partition_cases(), ids=lambda c: f"T{c['T']}H{c['H']}W{c['W']}")
def test_partition_golden(case):
    args = [case[k] for k in ("T", "H", "W", "cube_h", "cube_w", "cube_t", "n_text")]
    perm, ids, off, C = oracle.cube_partition(*args)
    assert np.array_equal(perm, case["perm"])
    assert np.array_equal(ids, case["ids"])
    assert np.array_equal(off, case["offsets"])
    assert C == len(case["offsets"]) - 1
    import ffn_long_video_b200 as fb   # the library's host partition (no GPU needed)
    lperm, lids, loff = fb.cube_partition(*args)
    assert np.array_equal(lperm, case["perm"])
    assert np.array_equal(lids, case["ids"])
    assert np.array_equal(loff, case["offsets"])


def _top_p_cases():
    out = []
    for ln in _lines("top_p.txt"):
        p, P, kept = (s.strip() for s in ln.split("|"))
        out.append((float(p), [float(v) for v in P.split()], [int(v) for v in kept.split()]))
    return out


@pytest.mark.parametrize("p,P,kept", _top_p_cases())
def test_top_p_golden(p, P, kept):
    mask = oracle.top_p(np.array(P), p)
    assert sorted(np.flatnonzero(mask).tolist()) == kept


def _ffn_cases():
    out = []
    for ln in _lines("ffn_select.txt"):
        sizes, norms, n_text, p, active = (s.strip() for s in ln.split("|"))
        out.append(([int(v) for v in sizes.split()], [float(v) for v in norms.split()],
                    int(n_text), float(p), [int(v) for v in active.split()]))
    return out


@pytest.mark.parametrize("sizes,norms,n_text,p,active", _ffn_cases())
def test_ffn_select_golden(sizes, norms, n_text, p, active):
    n_vis = len(norms)
    D = 8
    e = np.zeros(D)
    e[3] = 1.0
    x = np.concatenate([np.outer(norms, e), np.ones((n_text, D))])
    off = np.concatenate([[0], np.cumsum(sizes)])
    got = oracle.ffn_select(x, off, n_vis, p)
    assert got.astype(int).tolist() == active
