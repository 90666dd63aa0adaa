"""Benchmark of the AdaSpark layer hot path (AdaS-Attn + AdaS-FFN) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--no-cpu-baseline] [--config 3]

One step = adaspark_cube_attn + adaspark_token_ffn over one layer of the
Qwen2.5-VL-7B-shaped 64K-token workload (65536 visual tokens in 4x4x4 cubes +
256 text tokens, 28/4 heads, head_dim 128, hidden 3584, SwiGLU 18944, p = 0.7),
inputs resident in HBM.  Prints one JSON line (rank 0).

* value: tokens/s over all ranks (each rank runs its own replica of the layer;
  the path has no exchange step), timed with CUDA events between barriers,
  max over ranks.
* e2e: the same metric through the C ABI with every step's inputs (Q, K, V, x)
  copied from pinned host memory and its outputs (out, y) copied back inside
  the timed region; the copies of neighbouring steps overlap the computation
  (copy-in, compute and copy-out streams, two device buffers of each).
* roofline: the kernel with the largest share of the step, its algorithmic
  FLOPs (or bytes) per launch over its event-timed average duration.
* cpu_baseline / --impl reference: the float64 oracle, timed on the host cores
  on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "AdaSpark layer tokens/s at 64K visual tokens (7B shape); % bf16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# kernel (timer name) -> source file whose build the DRAM counters were taken on
KERNEL_SOURCES = {"attn_tc": "attn_tc.cu", "select_tc": "select_tc.cu",
                  "ffn_gemm1_tc": "ffn_gemm_tc.cu", "ffn_gemm2_tc": "ffn_gemm_tc.cu",
                  "attn_bwd_dq_tc": "attn_bwd.cu", "attn_bwd_dkv_tc": "attn_bwd.cu"}


def load_traffic(kernel, workload):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of
    `kernel` on `workload`, from the ncu summary profiles/<kernel>_<workload>.md,
    which records the counters and the SHA-256 of the kernel's source file at
    capture time. None when there is no summary or the source has changed
    since (the counters then describe another kernel)."""
    import hashlib
    src = KERNEL_SOURCES.get(kernel)
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if src is None or not os.path.exists(path):
        return None
    fields = {}
    for line in open(path):
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    try:
        want = fields["source-sha256"]
        nbytes = int(fields["traffic-bytes-per-launch"])
    except (KeyError, ValueError):
        return None
    with open(os.path.join(ROOT, "ffn_long_video_b200", "csrc", src), "rb") as f:
        have = hashlib.sha256(f.read()).hexdigest()
    return nbytes if have == want else None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        """Start sampling every 100 ms and return once the first sample has
        arrived (nvidia-smi takes a moment to start), so that a short timed
        region that begins afterwards is sampled."""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        t_end = time.time() + 10.0
        while not self.lines and time.time() < t_end and self.proc.poll() is None:
            time.sleep(0.02)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, begin: bool):
        """Host time of the start / end of the timed region."""
        if begin:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        # one more period so that the last sample of the region has arrived
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        t0, t1 = getattr(self, "t0", 0.0), getattr(self, "t1", float("inf"))
        for ts, ln in self.lines:
            # a sample describes the period before it arrives: keep those that
            # arrived inside the region or within one period after its end
            if ts < t0 or ts > t1 + 0.1:
                continue
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------- workload
def build_workload(cfg, device):
    import torch
    import workloads
    lay = workloads.make_layer(cfg, project_on=device)
    lay = {k: v.to(device) for k, v in lay.items()}
    ids = np.concatenate([np.repeat(np.arange(cfg.n_cubes, dtype=np.int32), cfg.sizes),
                          np.full(cfg.n_text, -1, np.int32)])
    lay["cube_ids"] = torch.from_numpy(ids).to(device)
    lay["cube_offsets"] = torch.from_numpy(cfg.offsets).to(device)
    lay["text_mask"] = torch.from_numpy((ids == -1).astype(np.uint8)).to(device)
    return lay


def kernel_work(name, cfg, attn_stats, ffn_stats):
    """Algorithmic work of one launch: (amount, unit, bound)."""
    M = ffn_stats["active_visual"] + ffn_stats["text_tokens"]
    if name.startswith("ffn_gemm1"):
        return 4.0 * M * cfg.D * cfg.F, "flop", "tensor"
    if name.startswith("ffn_gemm2"):
        return 2.0 * M * cfg.D * cfg.F, "flop", "tensor"
    if name == "attn_tc_gather":
        # the split walk's gathered tiles: QK^T + PV per (gathered tile, 64-key block)
        return 4.0 * 128 * 64 * cfg.d * attn_stats.get("gathered_blocks", 0), "flop", "tensor"
    if name.startswith("attn_tc"):
        # QK^T + PV per executed (128-row tile, 64-key block)
        return 4.0 * 128 * 64 * cfg.d * attn_stats["key_blocks"], "flop", "tensor"
    if name.startswith("select_tc"):
        # executed score MMAs: 3 bf16 parts of kbar x 2 passes x 2*d per (row, cube) pair
        return 12.0 * cfg.d * attn_stats["candidate_pairs"], "flop", "tensor"
    if name.startswith("select"):
        return 2.0 * cfg.d * attn_stats["candidate_pairs"], "flop", "alu"
    # backward (selection straight-through); pairs = executed (tile, key block) pairs
    pairs = attn_stats["key_blocks"]
    if name == "attn_bwd_dq_tc":
        # after a training-mode forward (the way bench.py runs it): S = Q K^T,
        # dP = dO V^T and dQ += dS K once per block (an inference-mode forward
        # would add a first pass of S and dP: 10 instead of 6)
        return 6.0 * 128 * 64 * cfg.d * pairs, "flop", "tensor"
    if name == "attn_bwd_dkv_tc":
        # S, dP, dV^T += dO^T P, dK^T += Q^T dS
        return 8.0 * 128 * 64 * cfg.d * pairs, "flop", "tensor"
    if name == "ffn_bwd_gemm_hdg_tc":
        return 6.0 * M * cfg.D * cfg.F, "flop", "tensor"
    if name in ("ffn_bwd_gemm_dx_tc", "ffn_bwd_gemm_dwgu_tc"):
        return 4.0 * M * cfg.D * cfg.F, "flop", "tensor"
    if name == "ffn_bwd_gemm_dwd_tc":
        return 2.0 * M * cfg.D * cfg.F, "flop", "tensor"
    if name == "wdown_to_fp16":
        return float(cfg.D) * cfg.F * 4, "byte", "hbm"
    if name == "ffn_select":
        return float(cfg.n_vis) * cfg.D * 2, "byte", "hbm"
    if name == "ffn_compact":
        return float(M) * cfg.D * 2 * 2, "byte", "hbm"
    if name == "ffn_compensate":
        skipped = ffn_stats["skipped_visual"]
        return float(skipped) * cfg.D * (2 + 4), "byte", "hbm"
    if name == "cube_mean_keys":
        return float(cfg.n_vis) * cfg.hkv * cfg.d * 2, "byte", "hbm"
    return None, None, None


def kernel_table(ktimes, calls, cfg, attn_stats, ffn_stats):
    """Per kernel: ms per library call (a call may launch a kernel several
    times, e.g. the attention once per KV head), launches per call, share of
    the summed kernel time, and the achieved TFLOP/s or GB/s where its
    algorithmic work per call is known. `ktimes` covers `calls` calls."""
    total = sum(v[1] for v in ktimes.values()) or 1.0
    kernels = {}
    for k, (n, ms) in sorted(ktimes.items(), key=lambda kv: -kv[1][1]):
        w, u, b = kernel_work(k, cfg, attn_stats, ffn_stats)
        e = {"ms_per_call": round(ms / calls, 4), "launches_per_call": round(n / calls, 2),
             "share": round(ms / total, 4)}
        if w is not None:
            if b == "tensor":
                e["tflops"] = round(w / (ms / calls / 1e3) / 1e12, 1)
            else:
                e["gbs"] = round(w / (ms / calls / 1e3) / 1e9, 1)
        kernels[k] = e
    return kernels


def roofline_of(name, calls, ms, cfg, attn_stats, ffn_stats, traffic, launches=None):
    """Roofline entry of one kernel from its timer total `ms` over `calls`
    library calls (its algorithmic work is counted per call). `traffic` is the
    DRAM bytes of one launch; with several launches per call it is scaled to
    the call only when they are equal pieces of it (not known here), so it is
    reported per launch with the launch count beside it."""
    work, unit, bound = kernel_work(name, cfg, attn_stats, ffn_stats)
    if work is None:
        return None
    peaks, peak_src = load_peaks()
    per_launch_ms = ms / calls
    if bound == "tensor":
        achieved = work / (per_launch_ms / 1e3) / 1e12
        peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        return {"kernel": name, "bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a step)",
                "traffic": traffic if (launches or calls) == calls else None,
                "ms_per_call": round(per_launch_ms, 4),
                "launches_per_call": round((launches or calls) / calls, 2)}
    achieved = work / (per_launch_ms / 1e3) / 1e9
    peak = peaks["hbm_gbs"]
    return {"kernel": name, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
            "unit": "GB/s", "frac": round(achieved / peak, 4), "peak_source": f"{peak_src} hbm_gbs",
            "traffic": traffic if (launches or calls) == calls else None,
            "ms_per_call": round(per_launch_ms, 4),
            "launches_per_call": round((launches or calls) / calls, 2)}


def max_over_ranks(v, world, device="cpu"):
    """The largest of the ranks' values (all ranks get it): multi-GPU times are
    the slowest replica's, taken on the device by each rank."""
    if world <= 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(ms_total_local, steps, tokens_per_replica, world, device="cpu"):
    """Whole-job tokens/s of `world` independent replicas: every replica
    processes its own layer per step, the job's step time is the slowest
    replica's (max over ranks). Returns (ms_per_step, tokens/s)."""
    ms_step = max_over_ranks(ms_total_local, world, device) / steps
    return ms_step, world * tokens_per_replica / (ms_step / 1e3)


def popcount32(x):
    """Set bits of each int32 element (SWAR on int64), on the device."""
    x = x.to(torch_mod().int64) & 0xFFFFFFFF
    x = x - ((x >> 1) & 0x55555555)
    x = (x & 0x33333333) + ((x >> 2) & 0x33333333)
    x = (x + (x >> 4)) & 0x0F0F0F0F
    return ((x * 0x01010101) & 0xFFFFFFFF) >> 24


def torch_mod():
    import torch
    return torch


def _hist(values, n_bins, top):
    """Equal-width histogram of integer values in [0, top] as [[lo, hi, count], ...]
    (bins with zero count left out)."""
    torch = torch_mod()
    width = max(1, -(-(top + 1) // n_bins))
    idx = torch.clamp(values // width, max=n_bins - 1)
    counts = torch.bincount(idx, minlength=n_bins).cpu().tolist()
    return [[b * width, min(top, b * width + width - 1), int(c)]
            for b, c in enumerate(counts) if c]


def rows_per_block(bits, n_cubes, thresholds=(1, 2, 4, 8, 16, 32, 64)):
    """How the union walk spends its blocks. The attention runs one 128-row
    tile per (128 consecutive visual tokens, query head) and walks every cube
    that any of its rows selected; for each such (tile, cube) block, r = how
    many of the 128 rows selected the cube and w = how many of the tile's four
    32-row warps hold one of them (a warp with none skips its softmax work).
    `bits` is the exported set tensor int32 [n_vis, hq, ceil(C/32)] (own cube
    not marked). Returns the histogram of r, and for each R in `thresholds`
    the fractions of blocks, of selected (row, cube) pairs and of active
    warp-blocks that lie in blocks with r <= R."""
    torch = torch_mod()
    n_vis, hq, W = bits.shape
    T = -(-n_vis // 128)
    shifts = torch.arange(32, device=bits.device, dtype=torch.int32)
    hist = torch.zeros(129, dtype=torch.int64, device=bits.device)
    pairs_r = torch.zeros(129, dtype=torch.float64, device=bits.device)
    warps_r = torch.zeros(129, dtype=torch.float64, device=bits.device)
    for h in range(hq):
        b = bits[:, h, :]
        if T * 128 != n_vis:
            b = torch.cat([b, b.new_zeros(T * 128 - n_vis, W)])
        u = ((b.unsqueeze(-1) >> shifts) & 1).to(torch.uint8).reshape(T * 128, W * 32)[:, :n_cubes]
        r = u.reshape(T, 128, n_cubes).sum(1, dtype=torch.int64).flatten()
        w = u.reshape(T, 4, 32, n_cubes).amax(2).sum(1, dtype=torch.int64).flatten()
        hist += torch.bincount(r, minlength=129)
        pairs_r += torch.bincount(r, weights=r.double(), minlength=129)
        warps_r += torch.bincount(r, weights=w.double(), minlength=129)
    h_, p_, w_ = hist.cpu().numpy(), pairs_r.cpu().numpy(), warps_r.cpu().numpy()
    blocks, pairs, warps = h_[1:].sum(), p_[1:].sum(), w_[1:].sum()
    return {
        "blocks": int(blocks), "pairs": int(round(pairs)), "active_warp_blocks": int(round(warps)),
        "mean_rows": round(float(pairs / max(blocks, 1)), 2),
        "r_le": {str(R): {"blocks": round(float(h_[1:R + 1].sum() / max(blocks, 1)), 4),
                          "pairs": round(float(p_[1:R + 1].sum() / max(pairs, 1)), 4),
                          "active_warp_blocks": round(float(w_[1:R + 1].sum() / max(warps, 1)), 4)}
                 for R in thresholds},
        "histogram_r_1_to_128": [int(v) for v in h_[1:]],
    }


def useful_attention_pairs(cfg, selected_pairs):
    """(row, key) pairs the method itself computes in AdaS-Attn: the keys of
    every selected cube, the own cube's causal prefix of every visual row and
    the causal prefix of every text row, over all query heads (every bench
    workload has equal cubes)."""
    sizes = np.asarray(cfg.sizes)
    assert (sizes == sizes[0]).all(), "equal cubes expected"
    n_c = int(sizes[0])
    own = cfg.n_cubes * n_c * (n_c + 1) // 2
    text = sum(t + 1 for t in range(cfg.n_vis, cfg.n_tokens))
    return selected_pairs * n_c + cfg.hq * (own + text)


def realised_sparsity(cfg, lay, aws, fws, attn_stats, ffn_stats, ktimes, calls, dense_ktimes):
    """What the timed call selected and computed (read from the library after
    the timed region): cubes per row and keep ratio per cube as histograms,
    useful against executed attention FLOPs, the near-margin counters."""
    torch = torch_mod()
    import ffn_long_video_b200 as fb
    dt = fb.BF16 if cfg.dtype == "bf16" else fb.FP32
    C = cfg.n_cubes
    # cubes selected per (visual token, query head) row, own cube excluded
    bits = fb.attn_export_bits(aws, lay["cube_ids"], C, cfg.n_vis, cfg.n_tokens, cfg.hq, cfg.hkv,
                               cfg.d, dt)
    per_row = []
    for t0 in range(0, cfg.n_vis, 8192):
        per_row.append(popcount32(bits[t0:t0 + 8192]).sum(dim=-1).reshape(-1))
    per_row = torch.cat(per_row)
    per_block = rows_per_block(bits, C)
    del bits
    own = torch.repeat_interleave(torch.arange(C, device=per_row.device),
                                  torch.as_tensor(cfg.sizes, device=per_row.device))
    own_rows = own.repeat_interleave(cfg.hq)             # preceding cubes of each row
    has = own_rows > 0
    frac = per_row[has].double() / own_rows[has].double()
    q = torch.tensor([0.0, 0.1, 0.5, 0.9, 1.0], dtype=torch.float64, device=frac.device)
    frac_q = torch.quantile(frac[: 1 << 24], q).cpu().tolist() if frac.numel() else []
    # active tokens per cube
    act = torch.empty(cfg.n_tokens, dtype=torch.uint8, device=lay["x"].device)
    fb.lib().adaspark_ffn_export_active(fb._ptr(fws), cfg.n_tokens, cfg.n_vis, C, cfg.D, cfg.F,
                                        dt, fb._ptr(act), fb._stream(None))
    per_cube = torch.bincount(lay["cube_ids"][: cfg.n_vis].long(),
                              weights=act[: cfg.n_vis].double(), minlength=C).long()
    n_c = int(np.asarray(cfg.sizes).max())
    keep_hist = torch.bincount(per_cube, minlength=n_c + 1).cpu().tolist()
    useful_pairs = useful_attention_pairs(cfg, attn_stats["selected_pairs"])
    useful = 4.0 * cfg.d * useful_pairs
    # the tiles' own blocks and the split walk's gathered blocks
    executed = 4.0 * 128 * 64 * cfg.d * (attn_stats["key_blocks"] +
                                         attn_stats.get("gathered_blocks", 0))
    dense_attn = workloads_mod().dense_flops(cfg)["attn"]
    out = {
        "what": "read from the library after the timed region (exported sets, active flags, "
                "counters); attention FLOPs count QK^T and PV",
        "cubes_per_row": {
            "mean": attn_stats["selected_pairs"] / max(1, attn_stats["visual_rows"]),
            "histogram": _hist(per_row, 32, int(per_row.max().item()) if per_row.numel() else 0),
            "fraction_of_preceding_quantiles_0_10_50_90_100": [round(v, 4) for v in frac_q]},
        "selected_fraction": attn_stats["selected_pairs"] / max(1, attn_stats["candidate_pairs"]),
        "ffn_keep_ratio": ffn_stats["active_visual"] / max(1, cfg.n_vis),
        "active_tokens_per_cube": {"histogram": [[k, int(c)] for k, c in enumerate(keep_hist)
                                                 if c],
                                   "of": n_c},
        "attention_useful_tflop": round(useful / 1e12, 4),
        "attention_executed_tflop": round(executed / 1e12, 4),
        "attention_dense_tflop": round(dense_attn / 1e12, 4),
        "executed_over_useful": round(executed / max(useful, 1.0), 3),
        "useful_over_dense": round(useful / dense_attn, 4),
        "executed_key_blocks": attn_stats["key_blocks"],
        "split_walk": {"pairs_in_gathered_tiles": attn_stats.get("split_pairs", 0),
                       "gathered_blocks": attn_stats.get("gathered_blocks", 0),
                       "what": "selected (row, cube) pairs of cubes that few of a tile's rows "
                               "chose, run in gathered 128-row tiles and merged into their rows "
                               "(adaspark_set_split_rows)"},
        "rows_per_executed_block": dict(
            per_block, what="selected cubes of 128-row tiles (own cubes, which every tile "
                            "walks causally, not counted): r = rows of the tile that chose the "
                            "cube; fractions of blocks, pairs and active 32-row warp-blocks in "
                            "blocks with r <= R"),
        "overflow_rows": attn_stats["overflow_rows"],
        "near_margin": {
            "attn_rows": attn_stats["near_margin_rows"],
            "attn_rows_of": attn_stats["visual_rows"],
            "ffn_cubes": ffn_stats["near_margin_cubes"], "ffn_cubes_of": C,
            "how": "library counters: cuts within 1e-5 of flipping (min of C_k* - p, "
                   "p - C_k*-1, P_(k*) - P_(k*+1)) from the fp32 masses; the GPU tests check "
                   "them against the float64 oracle and check every near-margin row the "
                   "library decided differently for a valid near-cut"},
    }
    peaks, src = load_peaks()
    peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    attn = ktimes.get("attn_tc") or ktimes.get("attn_simt")
    gath = ktimes.get("attn_tc_gather")
    sel = [ktimes[k] for k in ("select_tc", "select_simt", "cube_mean_keys", "validate",
                               "split_prefix", "split_scatter") if k in ktimes]
    if attn:
        # per call: the tiles' walk plus the split walk's gathered tiles
        a_ms = attn[1] / calls + (gath[1] / calls if gath else 0.0)
        s_ms = sum(v[1] / calls for v in sel)
        out["attention_ms"] = round(a_ms, 4)
        out["selection_ms"] = round(s_ms, 4)
        out["useful_tflops"] = round(useful / (a_ms / 1e3) / 1e12, 1)
        out["useful_tflops_with_selection"] = round(useful / ((a_ms + s_ms) / 1e3) / 1e12, 1)
        out["roofline_useful"] = {"bound": "tensor", "achieved": out["useful_tflops"],
                                  "peak": peak, "unit": "TFLOP/s",
                                  "frac": round(out["useful_tflops"] / peak, 4),
                                  "peak_source": f"{src} bf16_tflops_sustained"}
        dattn = dense_ktimes.get("attn_tc") or dense_ktimes.get("attn_simt")
        if dattn:
            d_ms = dattn[1]                          # one call
            out["dense_attention_ms"] = round(d_ms, 4)
            out["sparse_attention_with_selection_over_dense"] = round((a_ms + s_ms) / d_ms, 4)
    return out


def workloads_mod():
    import workloads
    return workloads


def timed_steps(step, n, stream, ktimer=False):
    """Run `step` n times between two events on `stream`; returns (ms, kernel
    times or None)."""
    torch = torch_mod()
    import ffn_long_video_b200 as fb
    if ktimer:
        fb.timer_enable(True)
        fb.timer_read()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    kt = None
    if ktimer:
        kt = fb.timer_read()
        fb.timer_enable(False)
    return e0.elapsed_time(e1), kt


def run_ours(args, rank, world, device):
    import torch
    import ffn_long_video_b200 as fb

    cfg = resolve_config(args)
    if fb.device_check(torch.cuda.current_device()) != fb.OK:
        raise RuntimeError("not an sm_100 device")
    if args.only:
        return run_only(args, cfg, device)
    if cfg.n_layers > 1:
        return run_stack(args, cfg, world, device)
    dt = fb.BF16 if cfg.dtype == "bf16" else fb.FP32
    lay = build_workload(cfg, device)
    N, n_vis = cfg.n_tokens, cfg.n_vis
    out = torch.empty_like(lay["Q"])
    y = torch.empty((N, cfg.D), dtype=torch.float32, device=device)
    aws = torch.empty(fb.cube_attn_workspace_bytes(N, n_vis, cfg.n_cubes, cfg.hq, cfg.hkv, cfg.d,
                                                   dt), dtype=torch.uint8, device=device)
    fws = torch.empty(fb.token_ffn_workspace_bytes(N, n_vis, cfg.n_cubes, cfg.D, cfg.F, dt),
                      dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def step(p=cfg.p, Q=None, K=None, V=None, x=None):
        fb.cube_attn(Q if Q is not None else lay["Q"], K if K is not None else lay["K"],
                     V if V is not None else lay["V"], lay["cube_ids"], lay["cube_offsets"],
                     n_vis, p, out=out, workspace=aws)
        fb.token_ffn(x if x is not None else lay["x"], lay["W_gate"], lay["W_up"], lay["W_down"],
                     lay["cube_ids"], lay["cube_offsets"], lay["text_mask"], n_vis, p, y=y,
                     workspace=fws)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    def reduce_max(v):
        return max_over_ranks(v, world, device)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    for ws in (aws, fws):
        code, det = fb.read_device_status(ws)
        if code != fb.OK:
            raise RuntimeError(f"device status {code} detail {det:#x}")

    # ---------------- timed region (device events, inputs resident in HBM)
    clocks = ClockSampler(torch.cuda.current_device())
    fb.timer_enable(True)
    fb.timer_read()
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    l0 = fb.launch_count()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.mark(True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    clocks.mark(False)
    launches = fb.launch_count() - l0
    ms_total = ev0.elapsed_time(ev1)
    clk = clocks.stop()
    barrier()
    ktimes = fb.timer_read()
    fb.timer_enable(False)
    ms_step, value = replica_throughput(ms_total, args.steps, N, world, device)

    attn_stats = fb.attn_read_stats(aws)
    ffn_stats = fb.ffn_read_stats(fws)

    # ---------------- roofline of the dominant kernel
    dname, (dn, dms) = max(ktimes.items(), key=lambda kv: kv[1][1])
    roof = roofline_of(dname, args.steps, dms, cfg, attn_stats, ffn_stats,
                       load_traffic(dname, cfg.name), launches=dn)
    kernels = kernel_table(ktimes, args.steps, cfg, attn_stats, ffn_stats)

    # ---------------- e2e through the C ABI with host buffers
    e2e = measure_e2e(args, cfg, lay, out, y, aws, fws, world, device)

    # ---------------- dense contrast (p = 1, same kernels, selection skipped)
    for _ in range(2):
        step(p=1.0)
    dense_total, _ = timed_steps(lambda: step(p=1.0), 2, stream)
    _, dense_kt = timed_steps(lambda: step(p=1.0), 1, stream, ktimer=True)
    dense_ms = reduce_max(dense_total) / 2

    # ---------------- the timed workload's sets back in the workspaces
    step()
    torch.cuda.synchronize()
    sparsity = realised_sparsity(cfg, lay, aws, fws, attn_stats, ffn_stats, ktimes, args.steps,
                                 dense_kt)

    # ---------------- backward (fine-tuning step), the forward's sets held fixed
    backward = None
    if not args.no_backward and cfg.dtype == "bf16":
        backward = measure_backward(args, cfg, lay, fws, attn_stats, ffn_stats, world, device,
                                    ms_step)

    dense = workloads_mod().dense_flops(cfg)
    return {
        "value": value, "ms_per_step": ms_step, "launches": launches // args.steps,
        "clocks": clk, "roofline": roof, "kernels": kernels, "e2e": e2e,
        "dense_contrast": {"ms_per_step": round(dense_ms, 3),
                           "value": world * N / (dense_ms / 1e3),
                           "dense_tflop": round((dense["attn"] + dense["ffn"]) / 1e12, 2),
                           "sparse_over_dense": round(ms_step / dense_ms, 4),
                           "kernels": kernel_table(dense_kt, 1, cfg, attn_stats, ffn_stats)},
        "sparsity": sparsity, "backward": backward, "cfg": cfg, "lay": lay,
    }


def run_only(args, cfg, device):
    """Profiling mode: one of the two calls alone, with only its own inputs,
    output and workspace on the device (about 1.3 GB for AdaS-Attn at 64K), so
    that a profiler capture of one launch moves little memory; or ("step") the
    step's two calls with nothing else, for a list of its launches. Prints the
    time per step; not a bench line."""
    import torch
    import ffn_long_video_b200 as fb
    import workloads
    dt = fb.BF16 if cfg.dtype == "bf16" else fb.FP32
    lay = workloads.make_layer(cfg, project_on=device)
    ids = np.concatenate([np.repeat(np.arange(cfg.n_cubes, dtype=np.int32), cfg.sizes),
                          np.full(cfg.n_text, -1, np.int32)])
    t_ids = torch.from_numpy(ids).to(device)
    t_off = torch.from_numpy(cfg.offsets).to(device)
    if args.only == "step":
        lay = {k: v.to(device) for k, v in lay.items()}
        text = torch.from_numpy((ids == -1).astype(np.uint8)).to(device)
        out = torch.empty_like(lay["Q"])
        y = torch.empty((cfg.n_tokens, cfg.D), dtype=torch.float32, device=device)
        aws = torch.empty(fb.cube_attn_workspace_bytes(cfg.n_tokens, cfg.n_vis, cfg.n_cubes,
                                                       cfg.hq, cfg.hkv, cfg.d, dt),
                          dtype=torch.uint8, device=device)
        ws = torch.empty(fb.token_ffn_workspace_bytes(cfg.n_tokens, cfg.n_vis, cfg.n_cubes, cfg.D,
                                                      cfg.F, dt), dtype=torch.uint8, device=device)

        def step():
            fb.cube_attn(lay["Q"], lay["K"], lay["V"], t_ids, t_off, cfg.n_vis, cfg.p, out=out,
                         workspace=aws)
            fb.token_ffn(lay["x"], lay["W_gate"], lay["W_up"], lay["W_down"], t_ids, t_off, text,
                         cfg.n_vis, cfg.p, y=y, workspace=ws)
    elif args.only == "attn":
        Q, K, V = (lay[k].to(device) for k in ("Q", "K", "V"))
        del lay
        torch.cuda.empty_cache()
        out = torch.empty_like(Q)
        ws = torch.empty(fb.cube_attn_workspace_bytes(cfg.n_tokens, cfg.n_vis, cfg.n_cubes, cfg.hq,
                                                      cfg.hkv, cfg.d, dt), dtype=torch.uint8,
                         device=device)
        step = lambda: fb.cube_attn(Q, K, V, t_ids, t_off, cfg.n_vis, cfg.p, out=out,
                                    workspace=ws)
    else:
        x, Wg, Wu, Wd = (lay[k].to(device) for k in ("x", "W_gate", "W_up", "W_down"))
        del lay
        torch.cuda.empty_cache()
        text = torch.from_numpy((ids == -1).astype(np.uint8)).to(device)
        y = torch.empty((cfg.n_tokens, cfg.D), dtype=torch.float32, device=device)
        ws = torch.empty(fb.token_ffn_workspace_bytes(cfg.n_tokens, cfg.n_vis, cfg.n_cubes, cfg.D,
                                                      cfg.F, dt), dtype=torch.uint8, device=device)
        step = lambda: fb.token_ffn(x, Wg, Wu, Wd, t_ids, t_off, text, cfg.n_vis, cfg.p, y=y,
                                    workspace=ws)
    for _ in range(args.warmup):
        step()
    ms, kt = timed_steps(step, args.steps, torch.cuda.current_stream(), ktimer=True)
    code, det = fb.read_device_status(ws)
    if code != fb.OK:
        raise RuntimeError(f"device status {code} detail {det:#x}")
    print(json.dumps({"only": args.only, "workload": cfg.name, "ms_per_call": ms / args.steps,
                      "kernels": {k: round(v[1] / v[0], 4) for k, v in kt.items()},
                      "device_bytes": torch.cuda.memory_reserved()}))
    raise SystemExit(0)


def measure_e2e(args, cfg, lay, out, y, aws, fws, world, device):
    """The step through the C ABI with host buffers. Every step copies its
    inputs (Q, K, V, x) from pinned host memory and its outputs (out, y) back,
    as a serving loop would: on a copy-in stream, the compute stream and a
    copy-out stream, with two device buffers of each kind. Q, K and V go first,
    so that AdaS-Attn starts while x is still on its way (AdaS-FFN waits for
    it), and the attention output leaves while AdaS-FFN runs; step k's outputs
    leave and step k+1's inputs arrive while step k+1 computes. The timed
    region runs from before the first input copy to the end of the last output
    copy."""
    import torch
    import ffn_long_video_b200 as fb
    N, n_vis = cfg.n_tokens, cfg.n_vis
    pinned = {k: torch.empty(lay[k].shape, dtype=lay[k].dtype, pin_memory=True)
              for k in ("Q", "K", "V", "x")}
    for k in pinned:
        pinned[k].copy_(lay[k])
    dev_in = [{k: torch.empty_like(lay[k]) for k in pinned} for _ in range(2)]
    dev_out = [torch.empty_like(out) for _ in range(2)]
    dev_y = [torch.empty_like(y) for _ in range(2)]
    host_out = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    host_y = [torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = host_out[0].numel() * host_out[0].element_size() + \
        host_y[0].numel() * host_y[0].element_size()
    e2e_steps = max(2, args.steps)
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    mk = lambda: [torch.cuda.Event() for _ in range(e2e_steps)]
    ev_qkv, ev_x, ev_attn, ev_cmp, ev_out_a, ev_out_y = mk(), mk(), mk(), mk(), mk(), mk()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for k in range(e2e_steps):
        b = k % 2
        if k >= 2:
            s_in.wait_event(ev_cmp[k - 2])           # inputs of buffer b consumed
        with torch.cuda.stream(s_in):
            for name in ("Q", "K", "V"):
                dev_in[b][name].copy_(pinned[name], non_blocking=True)
            ev_qkv[k].record(s_in)
            dev_in[b]["x"].copy_(pinned["x"], non_blocking=True)
            ev_x[k].record(s_in)
        d = dev_in[b]
        s_cmp.wait_event(ev_qkv[k])
        if k >= 2:
            s_cmp.wait_event(ev_out_a[k - 2])        # attention output of buffer b copied out
        with torch.cuda.stream(s_cmp):
            fb.cube_attn(d["Q"], d["K"], d["V"], lay["cube_ids"], lay["cube_offsets"], n_vis,
                         cfg.p, out=dev_out[b], workspace=aws, stream=s_cmp)
            ev_attn[k].record(s_cmp)
        s_cmp.wait_event(ev_x[k])
        if k >= 2:
            s_cmp.wait_event(ev_out_y[k - 2])        # y of buffer b copied out
        with torch.cuda.stream(s_cmp):
            fb.token_ffn(d["x"], lay["W_gate"], lay["W_up"], lay["W_down"], lay["cube_ids"],
                         lay["cube_offsets"], lay["text_mask"], n_vis, cfg.p, y=dev_y[b],
                         workspace=fws, stream=s_cmp)
            ev_cmp[k].record(s_cmp)
        s_out.wait_event(ev_attn[k])
        with torch.cuda.stream(s_out):
            host_out[b].copy_(dev_out[b], non_blocking=True)
            ev_out_a[k].record(s_out)
        s_out.wait_event(ev_cmp[k])
        with torch.cuda.stream(s_out):
            host_y[b].copy_(dev_y[b], non_blocking=True)
            ev_out_y[k].record(s_out)
    e1.record(s_out)
    torch.cuda.synchronize()
    for ws in (aws, fws):
        code, det = fb.read_device_status(ws)
        if code != fb.OK:
            raise RuntimeError(f"device status {code} detail {det:#x} in the e2e steps")
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device) / e2e_steps
    del dev_in, dev_out, dev_y, host_out, host_y, pinned
    torch.cuda.empty_cache()
    return {"value": world * N / (e2e_ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(e2e_ms, 3)}


def stack_inputs(cfg, device):
    """Per-layer inputs of the four-layer stack, made once by the harness
    outside the timed region: Q/K/V = x W (torch), h = x + out W_o with the
    library's AdaS-Attn output, the next layer's x = that layer's y scaled to
    unit RMS per token (in place of the RMSNorm of a decoder); the same wiring
    as the stack's parity test."""
    import torch
    import ffn_long_video_b200 as fb
    import workloads
    ids = np.concatenate([np.repeat(np.arange(cfg.n_cubes, dtype=np.int32), cfg.sizes),
                          np.full(cfg.n_text, -1, np.int32)])
    common = {"cube_ids": torch.from_numpy(ids).to(device),
              "cube_offsets": torch.from_numpy(cfg.offsets).to(device),
              "text_mask": torch.from_numpy((ids == -1).astype(np.uint8)).to(device)}
    layers, x = [], None
    for layer in range(cfg.n_layers):
        w = {k: v.to(device) for k, v in workloads.make_stack(cfg, layer).items()}
        if layer == 0:
            x = w.pop("x")
        qkv = workloads.project_qkv(cfg, x, w["W_q"], w["W_k"], w["W_v"], project_on=device)
        L = {k: v.to(device) for k, v in qkv.items()}
        out, _ = fb.cube_attn(L["Q"], L["K"], L["V"], common["cube_ids"],
                              common["cube_offsets"], cfg.n_vis, cfg.p)
        h = (x.float() + (out.reshape(cfg.n_tokens, -1).float() @ w["W_o"].float())).to(x.dtype)
        del out
        y, _ = fb.token_ffn(h, w["W_gate"], w["W_up"], w["W_down"], common["cube_ids"],
                            common["cube_offsets"], common["text_mask"], cfg.n_vis, cfg.p)
        L.update(x=x, h=h, **{k: w[k] for k in ("W_q", "W_k", "W_v", "W_o", "W_gate", "W_up",
                                                 "W_down")})
        layers.append(L)
        x = (y * torch.rsqrt(y.pow(2).mean(dim=1, keepdim=True) + 1e-6)).to(x.dtype)
        del y
        torch.cuda.empty_cache()
    return layers, common


def stack_layer0(cfg, device):
    """The first layer's inputs of the stack (x and its Q/K/V projections, the
    FFN weights), made without the library: what the reference arm times."""
    import workloads
    w = workloads.make_stack(cfg, 0)
    lay = {k: w[k] for k in ("x", "W_gate", "W_up", "W_down")}
    lay.update(workloads.project_qkv(cfg, w["x"], w["W_q"], w["W_k"], w["W_v"],
                                     project_on=device))
    return lay


def run_stack(args, cfg, world, device):
    """The four-layer 262K-token stack: one step runs AdaS-Attn and AdaS-FFN of
    all four layers on their inputs (resident in HBM). The layer wrapper with
    its Q/K/V/O projections (adaspark_layer, the library's tensor-core GEMM)
    is timed beside it, and the projections reported as the difference."""
    import torch
    import ffn_long_video_b200 as fb
    layers, common = stack_inputs(cfg, device)
    N, n_vis, C = cfg.n_tokens, cfg.n_vis, cfg.n_cubes
    out = torch.empty_like(layers[0]["Q"])
    y = torch.empty((N, cfg.D), dtype=torch.float32, device=device)
    aws = torch.empty(fb.cube_attn_workspace_bytes(N, n_vis, C, cfg.hq, cfg.hkv, cfg.d, fb.BF16),
                      dtype=torch.uint8, device=device)
    fws = torch.empty(fb.token_ffn_workspace_bytes(N, n_vis, C, cfg.D, cfg.F, fb.BF16),
                      dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    stats = []

    def step(collect=False):
        for L in layers:
            fb.cube_attn(L["Q"], L["K"], L["V"], common["cube_ids"], common["cube_offsets"],
                         n_vis, cfg.p, out=out, workspace=aws)
            fb.token_ffn(L["h"], L["W_gate"], L["W_up"], L["W_down"], common["cube_ids"],
                         common["cube_offsets"], common["text_mask"], n_vis, cfg.p, y=y,
                         workspace=fws)
            if collect:
                stats.append((fb.attn_read_stats(aws), fb.ffn_read_stats(fws)))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    for ws in (aws, fws):
        code, det = fb.read_device_status(ws)
        if code != fb.OK:
            raise RuntimeError(f"device status {code} detail {det:#x}")
    clocks = ClockSampler(torch.cuda.current_device())
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    l0 = fb.launch_count()
    clocks.mark(True)
    ms_total, ktimes = timed_steps(step, args.steps, stream, ktimer=True)
    clocks.mark(False)
    launches = fb.launch_count() - l0
    clk = clocks.stop()
    ms_step, value = replica_throughput(ms_total, args.steps, N, world, device)
    step(collect=True)      # per-layer counters (untimed)
    # the layer wrapper, projections included
    lws = torch.empty(fb.layer_workspace_bytes(N, n_vis, C, cfg.hq, cfg.hkv, cfg.d, cfg.D, cfg.F),
                      dtype=torch.uint8, device=device)

    def full_step():
        for L in layers:
            fb.layer(L["x"], L["Wt_q"], L["Wt_k"], L["Wt_v"], L["Wt_o"], L["W_gate"], L["W_up"],
                     L["W_down"], common["cube_ids"], common["cube_offsets"],
                     common["text_mask"], n_vis, cfg.hq, cfg.hkv, cfg.p, cfg.p, y=y,
                     workspace=lws)

    for L in layers:     # [in, out] draws -> the [out, in] layout of the layer call
        for k in ("q", "k", "v", "o"):
            L["Wt_" + k] = L["W_" + k].t().contiguous()
    full_step()
    full_ms, _ = timed_steps(full_step, max(1, min(args.steps, 3)), stream)
    full_ms /= max(1, min(args.steps, 3))
    code, det = fb.read_device_status(lws)
    if code != fb.OK:
        raise RuntimeError(f"layer wrapper device status {code} detail {det:#x}")
    att0, ffn0 = stats[0]
    dname, (dn, dms) = max(ktimes.items(), key=lambda kv: kv[1][1])
    # kernel work of layer 0's counters (the layers differ a little)
    calls = args.steps * cfg.n_layers
    roof = roofline_of(dname, calls, dms, cfg, att0, ffn0, load_traffic(dname, cfg.name),
                       launches=dn)
    per_layer = []
    for att, ffn in stats:
        useful = 4.0 * cfg.d * useful_attention_pairs(cfg, att["selected_pairs"])
        executed = 4.0 * 128 * 64 * cfg.d * (att["key_blocks"] + att.get("gathered_blocks", 0))
        per_layer.append({
            "mean_cubes_per_row": round(att["selected_pairs"] / max(1, att["visual_rows"]), 2),
            "selected_fraction": round(att["selected_pairs"] / max(1, att["candidate_pairs"]), 4),
            "ffn_keep_ratio": round(ffn["active_visual"] / max(1, n_vis), 4),
            "attention_useful_tflop": round(useful / 1e12, 3),
            "attention_executed_tflop": round(executed / 1e12, 3),
            "executed_over_useful": round(executed / useful, 3),
            "near_margin_attn_rows": att["near_margin_rows"],
            "near_margin_ffn_cubes": ffn["near_margin_cubes"]})
    return {
        "value": value, "ms_per_step": ms_step, "launches": launches // args.steps,
        "clocks": clk, "roofline": roof,
        "kernels": kernel_table(ktimes, calls, cfg, att0, ffn0), "e2e": None,
        "e2e_note": "not measured for the stack (every step would copy four layers' inputs)",
        "stack": {"layers": cfg.n_layers, "core_ms_per_layer": round(ms_step / cfg.n_layers, 3),
                  "with_projections_ms_per_step": round(full_ms, 3),
                  "projections_ms_per_step": round(full_ms - ms_step, 3),
                  "per_layer": per_layer},
        "dense_contrast": None, "sparsity": None, "backward": None, "cfg": cfg,
        "lay": layers[0],
    }


def measure_backward(args, cfg, lay, fws, attn_stats, ffn_stats, world, device, forward_ms):
    """One backward step = adaspark_cube_attn_backward + adaspark_token_ffn_backward
    on the sets the forward left in its workspaces, for seeded upstream
    gradients (dO bf16, dy fp32) resident in HBM; device-timed like the forward.
    The attention forward of a training step is adaspark_cube_attn_train (same
    sets; it keeps the fp32 output the backward takes D_r from); its time is
    reported beside the inference call's."""
    import torch
    import ffn_long_video_b200 as fb
    import workloads
    N, n_vis = cfg.n_tokens, cfg.n_vis
    up = workloads.make_upstream(cfg)
    dO, dy = up["dO"].to(device), up["dy"].to(device)
    out_t = torch.empty_like(lay["Q"])
    aws = torch.empty(fb.cube_attn_train_workspace_bytes(N, n_vis, cfg.n_cubes, cfg.hq, cfg.hkv,
                                                         cfg.d), dtype=torch.uint8,
                      device=device)

    def attn_train():
        fb.cube_attn(lay["Q"], lay["K"], lay["V"], lay["cube_ids"], lay["cube_offsets"], n_vis,
                     cfg.p, out=out_t, workspace=aws, train=True)

    for _ in range(2):
        attn_train()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for _ in range(3):
        attn_train()
    f1.record()
    torch.cuda.synchronize()
    attn_train_ms = max_over_ranks(f0.elapsed_time(f1), world, device) / 3
    code, det = fb.read_device_status(aws)
    if code != fb.OK:
        raise RuntimeError(f"training forward device status {code} detail {det:#x}")
    # the training-mode forward walks each tile's whole list (no split walk):
    # its counters give the blocks the backward executes
    attn_stats = dict(attn_stats, **{k: v for k, v in fb.attn_read_stats(aws).items()
                                     if k in ("key_blocks", "tiles")})
    bufs = {"a": {}, "f": {}}

    def bwd():
        ga = fb.cube_attn_backward(lay["Q"], lay["K"], lay["V"], dO, lay["cube_ids"],
                                   lay["cube_offsets"], n_vis, aws, **bufs["a"])
        gf = fb.token_ffn_backward(lay["W_gate"], lay["W_up"], lay["W_down"], lay["cube_offsets"],
                                   n_vis, dy, fws, **bufs["f"])
        bufs["a"] = dict(dQ=ga[0], dK=ga[1], dV=ga[2], workspace=ga[3])
        bufs["f"] = dict(dx=gf[0], dW_gate=gf[1], dW_up=gf[2], dW_down=gf[3], workspace=gf[4])

    steps = max(1, min(args.steps, 5))
    for _ in range(max(1, args.warmup)):
        bwd()
    torch.cuda.synchronize()
    for ws in (bufs["a"]["workspace"], bufs["f"]["workspace"]):
        code, det = fb.read_device_status(ws)
        if code != fb.OK:
            raise RuntimeError(f"backward device status {code} detail {det:#x}")
    fb.timer_enable(True)
    fb.timer_read()
    torch.cuda.synchronize()
    l0 = fb.launch_count()
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b0.record()
    for _ in range(steps):
        bwd()
    b1.record()
    torch.cuda.synchronize()
    launches = fb.launch_count() - l0
    ktimes = fb.timer_read()
    fb.timer_enable(False)
    ms = max_over_ranks(b0.elapsed_time(b1), world, device) / steps
    dname, (dn, dms) = max(ktimes.items(), key=lambda kv: kv[1][1])
    return {
        "what": "attention + FFN backward of the timed layer, cube and token sets of its "
                "forward held fixed (straight-through selection), attention forward in "
                "training mode; gradients fp32",
        "ms_per_step": round(ms, 3), "value": world * N / (ms / 1e3), "unit": "tokens/s",
        "steps": steps, "forward_plus_backward_ms": round(forward_ms + ms, 3),
        "attention_train_forward_ms": round(attn_train_ms, 3),
        "gpu_launches": launches,
        "roofline": roofline_of(dname, steps, dms, cfg, attn_stats, ffn_stats,
                                load_traffic(dname, cfg.name), launches=dn),
        "kernels": kernel_table(ktimes, steps, cfg, attn_stats, ffn_stats),
    }


# --------------------------------------------------------------------- CPU oracle
def oracle_sample(cfg, lay, budget_s=20.0, seed=0):
    """Time the float64 oracle, as it stands, on a bounded sample of the layer.

    The work the oracle does once per layer (float64 copies of Q, K, V, x and the
    three FFN weights; the cube mean keys) is timed once. Then, one at a time
    and timed each: AdaS-Attn rows of random visual tokens (all query heads:
    selection with the layer's cube means, then the attention), of random text
    tokens, and AdaS-FFN of random whole cubes; the text tokens' dense FFN once.
    The layer time is extrapolated as
        setup + n_vis * t(visual token) + n_text * t(text token)
              + C * t(cube) + t(text FFN).
    Returns a dict with the tokens/s of that extrapolated layer, the seconds
    actually spent, the extrapolation and the sample."""
    import torch
    import oracle
    rng = np.random.default_rng(seed)
    cores = len(os.sched_getaffinity(0))
    t_all = time.perf_counter()
    host = {k: lay[k].cpu() for k in ("Q", "K", "V", "x", "W_gate", "W_up", "W_down")}
    off = cfg.offsets
    a = time.perf_counter()
    f64 = {k: v.to(torch.float64).numpy() for k, v in host.items()}
    kbar = oracle.cube_mean_keys(f64["K"], off)
    setup_s = time.perf_counter() - a

    def attn_row(t):
        if t < cfg.n_vis:
            sel = oracle.select_cubes(f64["Q"], f64["K"], off, cfg.n_vis, cfg.hq, cfg.hkv, cfg.p,
                                      tokens=np.array([t]), kbar=kbar)
        else:
            sel = np.zeros((1, cfg.hq, cfg.n_cubes), bool)
        oracle.attention_given_sets(f64["Q"], f64["K"], f64["V"], off, cfg.n_vis, sel,
                                    tokens=np.array([t]))

    def timed_until(fn, draw, share, cap):
        spent, n = 0.0, 0
        while n < 1 or (spent < budget_s * share and n < cap):
            b = time.perf_counter()
            fn(draw())
            spent += time.perf_counter() - b
            n += 1
        return spent / n, n

    t_vis, n_vis_s = timed_until(attn_row, lambda: int(rng.integers(0, cfg.n_vis)), 0.35, 64)
    t_txt, n_txt_s = (0.0, 0)
    if cfg.n_text:
        t_txt, n_txt_s = timed_until(attn_row,
                                     lambda: int(rng.integers(cfg.n_vis, cfg.n_tokens)), 0.1, 16)
    t_cube, n_cube_s = timed_until(
        lambda c: oracle.token_ffn(f64["x"], f64["W_gate"], f64["W_up"], f64["W_down"], off,
                                   cfg.n_vis, cfg.p, cubes=[c], text=False),
        lambda: int(rng.integers(0, cfg.n_cubes)), 0.35, 16)
    b = time.perf_counter()
    if cfg.n_text:
        oracle.ffn_given_sets(f64["x"], f64["W_gate"], f64["W_up"], f64["W_down"], off,
                              cfg.n_vis, np.ones(cfg.n_tokens, bool), cubes=[], text=True)
    t_text_ffn = time.perf_counter() - b
    layer_s = (setup_s + cfg.n_vis * t_vis + cfg.n_text * t_txt + cfg.n_cubes * t_cube +
               t_text_ffn)
    spent = time.perf_counter() - t_all
    return {
        "value": cfg.n_tokens / layer_s, "cores": cores, "seconds": round(spent, 1),
        "layer_s_extrapolated": float(f"{layer_s:.4g}"),
        "extrapolation": f"setup {setup_s:.2f} s + {cfg.n_vis} x {t_vis:.4f} s + "
                         f"{cfg.n_text} x {t_txt:.4f} s + {cfg.n_cubes} x {t_cube:.4f} s + "
                         f"{t_text_ffn:.2f} s",
        "sample": (f"float64 oracle: per-layer setup (float64 copies, cube means) once; "
                   f"AdaS-Attn rows of {n_vis_s} random visual and {n_txt_s} random text tokens "
                   f"(all {cfg.hq} heads), AdaS-FFN of {n_cube_s} random cubes and the "
                   f"{cfg.n_text} text tokens; extrapolated to the {cfg.n_tokens}-token layer "
                   f"(not a timed layer)"),
    }


def resolve_config(args):
    """The workload of a run: configs 1-5, or point `--sweep i` of the 128K
    sweep (p x cube shape) of config 4."""
    import workloads
    if args.sweep is not None:
        if args.config != 4:
            raise SystemExit("--sweep applies to --config 4")
        return workloads.sweep_config(args.sweep)
    return workloads.CONFIGS[args.config]


def describe(cfg):
    layers = f"{cfg.n_layers} independent " if cfg.n_layers > 1 else "one "
    return (f"{cfg.name}: {layers}AdaSpark layer{'s' if cfg.n_layers > 1 else ''}, "
            f"{cfg.n_vis} visual tokens "
            f"({cfg.grid[0]}x{cfg.grid[1]}x{cfg.grid[2]} grid, {cfg.cube[0]}x{cfg.cube[1]}x"
            f"{cfg.cube[2]} cubes) + {cfg.n_text} text tokens, {cfg.hq}/{cfg.hkv} heads, "
            f"head_dim {cfg.d}, hidden {cfg.D}, SwiGLU {cfg.F}, p={cfg.p}, {cfg.dtype}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=3)
    ap.add_argument("--sweep", type=int, default=None,
                    help="point 0-7 of the 128K sweep of --config 4 (p x cube shape)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the backward-pass measurement")
    ap.add_argument("--only", choices=["attn", "ffn", "step"], default=None,
                    help="profiling mode: one call alone (small device footprint), or the "
                         "step's two calls without the extra measurements")
    args = ap.parse_args()

    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    cfg = resolve_config(args)
    workload = describe(cfg)
    dtype = "f32" if cfg.dtype == "fp32" else "bf16"

    if args.impl == "reference":
        if rank != 0:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
            return
        lay = build_workload(cfg, device) if cfg.n_layers == 1 else stack_layer0(cfg, device)
        budget = max(5.0, 150.0 / max(1, args.steps + args.warmup))
        runs = [oracle_sample(cfg, lay, budget_s=budget, seed=i)
                for i in range(args.warmup + args.steps)][args.warmup:]
        value = float(np.median([r["value"] for r in runs])) / cfg.n_layers
        mid = sorted(runs, key=lambda r: r["value"])[len(runs) // 2]
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
                "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(float(np.median([r["seconds"] for r in runs])) * 1e3, 1),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic",
                "config": {"workload": workload, "parallelism": "none (host cores)"},
                "timing": {"what": "each step times one bounded sample of the oracle on the "
                                   "layer (ms_per_step: the sample's own seconds); value: "
                                   "tokens/s of the extrapolated layer"
                                   + (f", divided by the {cfg.n_layers} layers"
                                      if cfg.n_layers > 1 else ""),
                           "layer_s_extrapolated": mid["layer_s_extrapolated"],
                           "extrapolation": mid["extrapolation"]},
                "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": mid["cores"],
                                 "kind": "oracle", "sample": mid["sample"]},
                "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    res = run_ours(args, rank, world, device)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r = oracle_sample(cfg, res["lay"], budget_s=20.0)
        cpu = {"value": r["value"] / cfg.n_layers, "unit": "tokens/s", "cores": r["cores"],
               "kind": "oracle", "sample": r["sample"], "seconds": r["seconds"],
               "layer_s_extrapolated": r["layer_s_extrapolated"],
               "extrapolation": r["extrapolation"]}
    if rank == 0:
        big = cfg.n_tokens * cfg.D * (2 if cfg.dtype == "bf16" else 4) > 126e6
        line = {
            "metric": METRIC, "value": res["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype,
            "data": "synthetic (seeded cube-structured inputs, random-init weights)",
            "config": {"workload": workload, "global_batch": world, "seq_len": cfg.n_tokens,
                       "parallelism": "replicas" if world > 1 else "single GPU",
                       "l2": ("inputs larger than L2 (x is "
                              f"{cfg.n_tokens * cfg.D * (2 if cfg.dtype == 'bf16' else 4) / 1e6:.0f}"
                              " MB)") if big else
                             "inputs fit in L2 (a small workload; not an L2-flushed figure)"},
            "roofline": res["roofline"], "cpu_baseline": cpu, "e2e": res["e2e"],
            "gpu_launches": res["launches"] * args.steps, "clocks": res["clocks"],
            "kernels": res["kernels"], "dense_contrast": res["dense_contrast"],
            "sparsity": res["sparsity"], "backward": res["backward"],
            "tensor_pct_of_peak": res["roofline"]["frac"] if res["roofline"] else None,
        }
        if "stack" in res:
            line["stack"] = res["stack"]
            line["e2e_note"] = res["e2e_note"]
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
