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


def kernel_table(ktimes, cfg, attn_stats, ffn_stats):
    """Per kernel: ms per launch, share of the summed kernel time, and the
    achieved TFLOP/s or GB/s where its algorithmic work is known."""
    total = sum(v[1] for v in ktimes.values()) or 1.0
    kernels = {}
    for k, (n, ms) in sorted(ktimes.items(), key=lambda kv: -kv[1][1]):
        w, u, b = kernel_work(k, cfg, attn_stats, ffn_stats)
        e = {"ms_per_launch": round(ms / n, 4), "share": round(ms / total, 4)}
        if w is not None:
            if b == "tensor":
                e["tflops"] = round(w / (ms / n / 1e3) / 1e12, 1)
            else:
                e["gbs"] = round(w / (ms / n / 1e3) / 1e9, 1)
        kernels[k] = e
    return kernels


def roofline_of(name, n, ms, cfg, attn_stats, ffn_stats, traffic):
    """Roofline entry of one kernel from its timer totals (n launches, ms)."""
    work, unit, bound = kernel_work(name, cfg, attn_stats, ffn_stats)
    if work is None:
        return None
    peaks, peak_src = load_peaks()
    per_launch_ms = ms / n
    if bound == "tensor":
        achieved = work / (per_launch_ms / 1e3) / 1e12
        peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        return {"kernel": name, "bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a step)",
                "traffic": traffic, "ms_per_launch": round(per_launch_ms, 4)}
    achieved = work / (per_launch_ms / 1e3) / 1e9
    peak = peaks["hbm_gbs"]
    return {"kernel": name, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
            "unit": "GB/s", "frac": round(achieved / peak, 4), "peak_source": f"{peak_src} hbm_gbs",
            "traffic": traffic, "ms_per_launch": round(per_launch_ms, 4)}


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


def run_ours(args, rank, world, device):
    import torch
    import ffn_long_video_b200 as fb
    import workloads

    cfg = workloads.CONFIGS[args.config]
    if fb.device_check(torch.cuda.current_device()) != fb.OK:
        raise RuntimeError("not an sm_100 device")
    lay = build_workload(cfg, device)
    N, n_vis = cfg.n_tokens, cfg.n_vis
    out = torch.empty_like(lay["Q"])
    y = torch.empty((N, cfg.D), dtype=torch.float32, device=device)
    aws = torch.empty(fb.cube_attn_workspace_bytes(N, n_vis, cfg.n_cubes, cfg.hq, cfg.hkv, cfg.d,
                                                   fb.BF16), dtype=torch.uint8, device=device)
    fws = torch.empty(fb.token_ffn_workspace_bytes(N, n_vis, cfg.n_cubes, cfg.D, cfg.F, fb.BF16),
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
    roof = roofline_of(dname, dn, dms, cfg, attn_stats, ffn_stats, load_traffic(dname, cfg.name))
    kernels = kernel_table(ktimes, cfg, attn_stats, ffn_stats)

    # ---------------- e2e through the C ABI with host buffers
    # Every step copies its inputs (Q, K, V, x) from pinned host memory and its
    # outputs (out, y) back, as a serving loop would: on a copy-in stream, the
    # compute stream and a copy-out stream, with two device buffers of each
    # kind. Q, K and V go first, so that AdaS-Attn starts while x is still on
    # its way (AdaS-FFN waits for it), and the attention output leaves while
    # AdaS-FFN runs; step k's outputs leave and step k+1's inputs arrive while
    # step k+1 computes. The timed region runs from before the first input
    # copy to the end of the last output copy.
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
    barrier()
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
    e2e_ms = reduce_max(e0.elapsed_time(e1)) / e2e_steps
    e2e = {"value": world * N / (e2e_ms / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
           "ms_per_step": round(e2e_ms, 3)}

    # ---------------- dense contrast (p = 1, same kernels, selection skipped)
    for _ in range(2):
        step(p=1.0)
    torch.cuda.synchronize()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for _ in range(2):
        step(p=1.0)
    d1.record(stream)
    torch.cuda.synchronize()
    dense_ms = d0.elapsed_time(d1) / 2

    # ---------------- backward (fine-tuning step), the forward's sets held fixed
    backward = None
    if not args.no_backward:
        step()  # the sets of the timed workload (p = cfg.p) back in the FFN workspace
        backward = measure_backward(args, cfg, lay, fws, attn_stats, ffn_stats, world, device,
                                    ms_step)

    dense = workloads.dense_flops(cfg)
    sparsity = {
        "mean_selected_cubes_per_row": attn_stats["selected_pairs"] / max(1,
                                                                          attn_stats["visual_rows"]),
        "selected_fraction": attn_stats["selected_pairs"] / max(1, attn_stats["candidate_pairs"]),
        "executed_key_blocks": attn_stats["key_blocks"],
        "overflow_rows": attn_stats["overflow_rows"],
        "ffn_keep_ratio": ffn_stats["active_visual"] / max(1, n_vis),
    }
    return {
        "value": value, "ms_per_step": ms_step, "launches": launches // args.steps,
        "clocks": clk, "roofline": roof, "kernels": kernels, "e2e": e2e,
        "dense_contrast": {"ms_per_step": round(dense_ms, 3),
                           "value": world * N / (dense_ms / 1e3),
                           "dense_tflop": round((dense["attn"] + dense["ffn"]) / 1e12, 2)},
        "sparsity": sparsity, "backward": backward, "cfg": cfg, "lay": lay,
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
        "roofline": roofline_of(dname, dn, dms, cfg, attn_stats, ffn_stats,
                                load_traffic(dname, cfg.name)),
        "kernels": kernel_table(ktimes, cfg, attn_stats, ffn_stats),
    }


# --------------------------------------------------------------------- CPU oracle
def oracle_sample(cfg, lay, budget_s=20.0, seed=0):
    """Time the float64 oracle on a bounded sample: attention rows (all heads) of
    tokens spread over the sequence, and the FFN of whole cubes.  Returns
    (tokens/s extrapolated, description, cores)."""
    import torch
    import oracle
    rng = np.random.default_rng(seed)
    cores = len(os.sched_getaffinity(0))
    Q, K, V, x = (lay[k].cpu() for k in ("Q", "K", "V", "x"))
    Wg, Wu, Wd = (lay[k].cpu() for k in ("W_gate", "W_up", "W_down"))
    off = cfg.offsets
    t0 = time.perf_counter()
    n_att = 0
    att_time = 0.0
    toks = []
    while att_time < budget_s * 0.5 and n_att < 64:
        t = int(rng.integers(0, cfg.n_tokens))
        a = time.perf_counter()
        sel = oracle.select_cubes(Q, K, off, cfg.n_vis, cfg.hq, cfg.hkv, cfg.p,
                                  tokens=np.array([t]) if t < cfg.n_vis else np.array([], int))
        full = np.zeros((1, cfg.hq, cfg.n_cubes), bool)
        if t < cfg.n_vis:
            full[0] = sel[0]
        oracle.attention_given_sets(Q, K, V, off, cfg.n_vis, full, tokens=np.array([t]))
        att_time += time.perf_counter() - a
        n_att += 1
        toks.append(t)
    n_cubes = 0
    ffn_time = 0.0
    while ffn_time < budget_s * 0.5 and n_cubes < 16:
        c = int(rng.integers(0, cfg.n_cubes))
        a = time.perf_counter()
        oracle.token_ffn(x, Wg, Wu, Wd, off, cfg.n_vis, cfg.p, cubes=[c], text=False)
        ffn_time += time.perf_counter() - a
        n_cubes += 1
    per_tok = att_time / n_att + ffn_time / (n_cubes * cfg.n_c)
    desc = (f"{n_att} random tokens' AdaS-Attn rows (all {cfg.hq} heads, incl. cube means and "
            f"selection) + AdaS-FFN of {n_cubes} random cubes; per-token times extrapolated to "
            f"the {cfg.n_tokens}-token layer")
    return 1.0 / per_tok, desc, cores, time.perf_counter() - t0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the backward-pass measurement")
    args = ap.parse_args()

    import torch
    import workloads
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
    cfg = workloads.CONFIGS[args.config]
    workload = (f"{cfg.name}: one AdaSpark layer, {cfg.n_vis} visual tokens "
                f"({cfg.grid[0]}x{cfg.grid[1]}x{cfg.grid[2]} grid, {cfg.cube[0]}x{cfg.cube[1]}x"
                f"{cfg.cube[2]} cubes) + {cfg.n_text} text tokens, {cfg.hq}/{cfg.hkv} heads, "
                f"head_dim {cfg.d}, hidden {cfg.D}, SwiGLU {cfg.F}, p={cfg.p}")

    if args.impl == "reference":
        if rank != 0:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
            return
        lay = build_workload(cfg, device)
        vals = []
        descs = None
        cores = len(os.sched_getaffinity(0))
        budget = max(5.0, 150.0 / max(1, args.steps + args.warmup))
        for i in range(args.warmup + args.steps):
            v, descs, cores, _ = oracle_sample(cfg, lay, budget_s=budget, seed=i)
            if i >= args.warmup:
                vals.append(v)
        value = float(np.median(vals))
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
                "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": cfg.n_tokens / value * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": workload, "parallelism": "none (host cores)"},
                "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                                 "kind": "oracle", "sample": descs},
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
        v, desc, cores, spent = oracle_sample(cfg, res["lay"], budget_s=20.0)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": desc, "seconds": round(spent, 1)}
    if rank == 0:
        line = {
            "metric": METRIC, "value": res["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded cube-structured inputs, random-init weights)",
            "config": {"workload": workload, "global_batch": world, "seq_len": cfg.n_tokens,
                       "parallelism": "replicas" if world > 1 else "single GPU",
                       "l2": "inputs larger than L2 (Q and x are 472 MB each)"},
            "roofline": res["roofline"], "cpu_baseline": cpu, "e2e": res["e2e"],
            "gpu_launches": res["launches"] * args.steps, "clocks": res["clocks"],
            "kernels": res["kernels"], "dense_contrast": res["dense_contrast"],
            "sparsity": res["sparsity"], "backward": res["backward"],
            "tensor_pct_of_peak": res["roofline"]["frac"] if res["roofline"] else None,
        }
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
