"""Host-side arithmetic of bench.py (no GPU): the algorithmic work per launch,
the roofline entry built from it, the check that ties recorded DRAM counters
to the kernel source they were taken on, and the clock-sample filter."""
import hashlib
import os

import pytest

import bench
import workloads

CFG = workloads.CONFIGS[3]   # the 64K-token 7B-shaped layer
ATTN = {"key_blocks": 1000, "candidate_pairs": 5000}
FFN = {"active_visual": 300, "text_tokens": 20, "skipped_visual": 40}


def test_kernel_work_counts():
    d, D, F = CFG.d, CFG.D, CFG.F
    M = 320
    # attention: Q K^T and P V, 2 flops per multiply-add, 128 rows x 64 keys x d per block
    assert bench.kernel_work("attn_tc", CFG, ATTN, FFN) == (2 * 2 * 128 * 64 * d * 1000, "flop",
                                                             "tensor")
    assert bench.kernel_work("ffn_gemm1_tc", CFG, ATTN, FFN)[0] == 2 * 2 * M * D * F
    assert bench.kernel_work("ffn_gemm2_tc", CFG, ATTN, FFN)[0] == 2 * M * D * F
    # three bf16 parts of the cube means, two passes, 2 d flops per (row, cube) pair
    assert bench.kernel_work("select_tc", CFG, ATTN, FFN)[0] == 3 * 2 * 2 * d * 5000
    # backward: S, dP, dQ (three products) and S, dP, dV, dK (four) per block
    assert bench.kernel_work("attn_bwd_dq_tc", CFG, ATTN, FFN)[0] == 3 * 2 * 128 * 64 * d * 1000
    assert bench.kernel_work("attn_bwd_dkv_tc", CFG, ATTN, FFN)[0] == 4 * 2 * 128 * 64 * d * 1000
    # recompute gate and up plus dh = df W_down: three D x F products per row
    assert bench.kernel_work("ffn_bwd_gemm_hdg_tc", CFG, ATTN, FFN)[0] == 3 * 2 * M * D * F
    # HBM kernels: bytes moved
    assert bench.kernel_work("ffn_compensate", CFG, ATTN, FFN) == (40 * D * (2 + 4), "byte", "hbm")
    assert bench.kernel_work("ffn_select", CFG, ATTN, FFN)[0] == CFG.n_vis * D * 2
    assert bench.kernel_work("no_such_kernel", CFG, ATTN, FFN) == (None, None, None)


def test_roofline_fraction(monkeypatch):
    peaks = {"hbm_gbs": 5000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1000.0}
    monkeypatch.setattr(bench, "load_peaks", lambda: (dict(peaks), "measured"))
    attn = {"key_blocks": 5_000_000, "candidate_pairs": 0}   # about the 64K layer's
    work = bench.kernel_work("attn_tc", CFG, attn, FFN)[0]
    # two calls of 25 ms each, one launch per call
    r = bench.roofline_of("attn_tc", 2, 50.0, CFG, attn, FFN, traffic=123, launches=2)
    achieved = work / 25e-3 / 1e12
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(achieved, rel=1e-3)
    assert r["peak"] == 1000.0                       # the sustained figure
    assert r["frac"] == pytest.approx(achieved / 1000.0, rel=1e-3)
    assert r["traffic"] == 123 and r["ms_per_call"] == 25.0
    # the same calls as five launches each (one per KV head and the text
    # tiles): the work and time per call are unchanged; one launch's DRAM
    # counters no longer describe a call
    r5 = bench.roofline_of("attn_tc", 2, 50.0, CFG, attn, FFN, traffic=123, launches=10)
    assert r5["achieved"] == r["achieved"] and r5["traffic"] is None
    assert r5["launches_per_call"] == 5.0
    h = bench.roofline_of("ffn_select", 1, 2.0, CFG, ATTN, FFN, traffic=None)
    gbs = CFG.n_vis * CFG.D * 2 / 2e-3 / 1e9
    assert h["bound"] == "hbm" and h["achieved"] == pytest.approx(gbs, rel=1e-3)
    assert h["frac"] == pytest.approx(gbs / 5000.0, rel=1e-3)
    assert bench.roofline_of("no_such_kernel", 1, 1.0, CFG, ATTN, FFN, None) is None


def test_kernel_table_shares():
    # one call; the attention launched twice in it
    t = bench.kernel_table({"attn_tc": (2, 30.0), "ffn_select": (1, 10.0)}, 1, CFG, ATTN, FFN)
    assert list(t) == ["attn_tc", "ffn_select"]      # largest share first
    assert t["attn_tc"]["share"] == 0.75 and t["ffn_select"]["share"] == 0.25
    assert t["attn_tc"]["ms_per_call"] == 30.0 and t["attn_tc"]["launches_per_call"] == 2.0
    assert "tflops" in t["attn_tc"] and "gbs" in t["ffn_select"]


def _write_profile(root, kernel, workload, nbytes, sha):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    with open(os.path.join(root, "profiles", f"{kernel}_{workload}.md"), "w") as f:
        f.write(f"# summary\n\n- traffic-bytes-per-launch: `{nbytes}`\n- source-sha256: `{sha}`\n")


def test_traffic_tied_to_kernel_source(tmp_path, monkeypatch):
    root = str(tmp_path)
    csrc = os.path.join(root, "ffn_long_video_b200", "csrc")
    os.makedirs(csrc)
    src = b"// kernel source\n"
    with open(os.path.join(csrc, "attn_tc.cu"), "wb") as f:
        f.write(src)
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.load_traffic("attn_tc", "w") is None                     # no summary
    _write_profile(root, "attn_tc", "w", 4096, hashlib.sha256(src).hexdigest())
    assert bench.load_traffic("attn_tc", "w") == 4096                     # same source
    with open(os.path.join(csrc, "attn_tc.cu"), "ab") as f:
        f.write(b"// edited\n")
    assert bench.load_traffic("attn_tc", "w") is None                     # source changed
    _write_profile(root, "no_such_kernel", "w", 1, "0" * 64)
    assert bench.load_traffic("no_such_kernel", "w") is None              # unknown kernel


class _FakeProc:
    stdout = iter(())

    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0

    def kill(self):
        pass


def test_clock_samples_inside_the_region():
    s = bench.ClockSampler(0)
    s.proc = _FakeProc()
    s.t0, s.t1 = 100.0, 110.0

    def line(mhz, cap="Not Active", thermal="Not Active"):
        return f"0, {mhz}, 1965, 900.0, 0x4, Not Active, {thermal}, Not Active, {cap}"
    s.lines = [(99.0, line(500, thermal="Active")),      # before the region: dropped
               (101.0, line(1700, cap="Active")),
               (105.0, line(1800)),
               (110.05, line(1900)),                      # within one period after the end
               (111.0, line(600, thermal="Active")),      # after it: dropped
               (106.0, "garbled")]
    r = s.stop()
    assert r["samples"] == 3
    assert r["sm_mhz"] == 1800.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]


def test_clock_sampler_without_nvidia_smi():
    s = bench.ClockSampler(0)
    assert s.stop()["reasons"] == ["nvidia-smi unavailable"]


def test_popcount32_matches_python():
    import numpy as np
    import torch
    rng = np.random.default_rng(5)
    v = rng.integers(-2**31, 2**31, size=1000, dtype=np.int64).astype(np.int32)
    got = bench.popcount32(torch.from_numpy(v)).numpy()
    want = [bin(int(x) & 0xFFFFFFFF).count("1") for x in v]
    assert list(got) == want


def test_useful_pairs_count_every_admitted_key():
    """Selected cubes' keys + own-cube causal prefixes + text causal prefixes,
    over all heads, counted against a brute-force walk of a tiny layer."""
    cfg = workloads.small_config(name="pairs", grid=(2, 4, 4), cube=(2, 2, 2), n_text=5, D=64,
                                 hq=3, hkv=1, F=128)
    sizes, off = cfg.sizes, cfg.offsets
    selected_pairs = 17           # any count: each selected cube brings n_c keys
    brute = selected_pairs * int(sizes[0])
    for h in range(cfg.hq):
        for t in range(cfg.n_tokens):
            if t < cfg.n_vis:
                c = int((off <= t).sum()) - 1
                brute += t - int(off[c]) + 1
            else:
                brute += t + 1
    assert bench.useful_attention_pairs(cfg, selected_pairs) == brute


def test_oracle_sample_extrapolates_a_small_layer():
    """The CPU baseline on a tiny layer: every term of the extrapolation is
    there, the layer time is their sum and the value is tokens per second."""
    lay = workloads.make_layer(workloads.CONFIGS[1])
    r = bench.oracle_sample(workloads.CONFIGS[1], lay, budget_s=0.5)
    assert r["value"] > 0 and r["cores"] >= 1
    terms = r["extrapolation"].replace("setup", "").split("+")
    total = 0.0
    for term in terms:
        parts = term.replace("s", "").split("x")
        total += float(parts[0]) * float(parts[1]) if len(parts) == 2 else float(parts[0])
    assert abs(total - r["layer_s_extrapolated"]) <= 0.05 + 0.01 * total
    assert abs(r["value"] - workloads.CONFIGS[1].n_tokens / r["layer_s_extrapolated"]) \
        <= 0.05 * r["value"]


def test_rows_per_block_brute_force():
    """Per (128-row tile, cube) block: rows that chose the cube and active warps,
    against a plain loop over a random set tensor with a ragged last tile."""
    import numpy as np
    import torch
    rng = np.random.default_rng(5)
    n_vis, hq, C = 300, 2, 40
    sel = rng.random((n_vis, hq, C)) < 0.07
    W = (C + 31) // 32
    words = np.zeros((n_vis, hq, W), dtype=np.int64)
    for j in range(C):
        words[:, :, j // 32] |= sel[:, :, j].astype(np.int64) << (j % 32)
    bits = torch.from_numpy(words.astype(np.uint32).view(np.int32))
    got = bench.rows_per_block(bits, C, thresholds=(1, 3))
    hist = np.zeros(129, dtype=np.int64)
    pairs_le = {1: 0, 3: 0}
    warps_le = {1: 0, 3: 0}
    blocks_le = {1: 0, 3: 0}
    tot_pairs = tot_warps = 0
    for h in range(hq):
        for t0 in range(0, n_vis, 128):
            rows = sel[t0:t0 + 128, h, :]
            for j in range(C):
                r = int(rows[:, j].sum())
                if r == 0:
                    continue
                w = sum(int(rows[q:q + 32, j].any()) for q in range(0, rows.shape[0], 32))
                hist[r] += 1
                tot_pairs += r
                tot_warps += w
                for R in (1, 3):
                    if r <= R:
                        blocks_le[R] += 1
                        pairs_le[R] += r
                        warps_le[R] += w
    blocks = hist[1:].sum()
    assert got["blocks"] == blocks and got["pairs"] == tot_pairs
    assert got["active_warp_blocks"] == tot_warps
    assert got["histogram_r_1_to_128"] == hist[1:].tolist()
    for R in (1, 3):
        e = got["r_le"][str(R)]
        assert e["blocks"] == round(blocks_le[R] / blocks, 4)
        assert e["pairs"] == round(pairs_le[R] / tot_pairs, 4)
        assert e["active_warp_blocks"] == round(warps_le[R] / tot_warps, 4)
