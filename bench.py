"""Benchmark of the Parallax attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--sweep]

Headline (`value`): split-KV decode throughput in GB/s of KV cache streamed,
on the decode workload B=64, H=16, L=4096, d=128 bf16 (all sequences full),
one plx_decode launch per step, inputs resident in HBM (2.1 GB of KV, larger
than the 126 MB L2, so no flush is needed).  The same run measures the causal
prefill B=8, H=16, N=4096, d=128 bf16 in TFLOP/s (the metric's second half)
under "prefill", a layer step (projections, RMSNorm+RoPE, attention) under
"layer", and the grouped-KV decode B=64, H=32, Hkv=8, L=4096, d=128 in GB/s
under "decode_gqa", the training forward plus backward pass of the
prefill workload under "prefill.backward", and sliding windows of 1024 keys on
the prefill and decode workloads under "window", the decode over an e4m3 KV
cache (the decode workload's shape and groups of 4) under "decode_fp8kv", and
five cells of the decode sweep under "decode_sweep".  For N > 1 GPUs (launched by torchrun) every rank runs the
same per-GPU workload on its own seeded inputs with no data-path collective
(weak scaling); time is the max over ranks.

`--only NAME` runs one workload four times and exits (what the profiler
captures under profiles/ run).  `--impl reference` times the float64 CPU oracle (the only reference this
method has) on bounded samples of the same workload.  `--sweep` prints one
line per decode sweep cell instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode KV GB/s (% HBM peak); causal prefill TFLOP/s (% BF16 peak)"
DECODE = dict(B=64, H=16, L=4096, d=128)
PREFILL = dict(B=8, H=16, N=4096, d=128)
# The compute-matched variant (head dim halved, twice the heads, same width).
PREFILL_D64 = dict(B=8, H=32, N=4096, d=64)
WINDOW = 1024  # sliding-window length of the window lines
# Grouped KV heads: 32 query heads over 8 KV heads (groups of 4, the grouping of the
# Llama-3-8B lineage), 1.07 GB of KV.
DECODE_GQA = dict(B=64, H=32, Hkv=8, L=4096, d=128)
L2_BYTES = 126 * 1024 * 1024  # B200 L2
LAYER = dict(B=4, N=8192, D=2048, H=16)
SWEEP_B = [1, 8, 64, 256, 1024, 2048]
SWEEP_L = [128, 1024, 4096, 16384, 32768]
SWEEP_MAX_BYTES = 150e9
# Sweep cells in the default line: few long sequences, mid-size and large batches, short contexts.
SWEEP_SUBSET = [(1, 32768), (8, 4096), (64, 1024), (256, 16384), (2048, 128)]

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "of measured"
    return dict(FALLBACK_PEAKS), "of fallback"


def decode_bytes(seqlens, H, d):
    kv = int(np.sum(seqlens.astype(np.int64))) * H * d * 2 * 2
    return kv, kv + 3 * len(seqlens) * H * d * 2


def prefill_flops(B, H, N, d, causal=True):
    pairs = N * (N + 1) // 2 if causal else N * N
    return 8.0 * d * pairs * B * H


def lib_ws_window(plx, B, H, Hkv, L, d, W):
    return int(plx.lib.plx_decode_window_workspace_bytes(B, H, Hkv, L, d, W))


def backward_flops(B, H, N, d, causal=True):
    """Algorithmic flops of the backward pass: eight GEMMs per visible pair
    (S, T, dA = dO V^T, dV, dK from dl and from dt, dQ, dR), 2 d flops each."""
    pairs = N * (N + 1) // 2 if causal else N * N
    return 16.0 * d * pairs * B * H


def backward_bytes(B, H, N, d):
    """Bytes the backward pass must move once: Q, K, V, R, dO, out (bf16), vbar
    (fp32), lse and tbar read; dQ, dK, dV, dR written; the statistics
    workspace (16 B per row) written and read."""
    rows = B * H * N
    return rows * d * (6 * 2 + 4 + 4 * 2) + rows * (2 * 4 + 2 * 16)


def prefill_bytes(B, H, N, d):
    return 5 * B * H * N * d * 2


def kernel_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "local_linear_attention_streamed_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profile_field(name, src_hash, key):
    """A field of a committed ncu summary under profiles/, if the summary is
    still current (its kernel sources hash to src_hash), else None."""
    path = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(path):
        return None
    with open(path) as f:
        p = json.load(f)
    if p.get("kernel_source_hash") != src_hash:
        return None
    return p.get(key)


def traffic_from_profile(name, src_hash, units_scale=1.0):
    """dram read+write bytes per launch from a committed ncu summary, if still current."""
    v = profile_field(name, src_hash, "dram_bytes_per_launch")
    return None if v is None else float(v) * units_scale


# ---------------------------------------------------------------------------
# Clock sampling during the timed region.
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.dev = device_index

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.dev)], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                self.out = ""
        return False

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 7:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[3:]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        return {"sm_mhz": float(np.median([r[0] for r in rows])), "sm_max_mhz": rows[0][1],
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# GPU arm.
# ---------------------------------------------------------------------------

def timed(fn, steps, warmup, stream, dist=None):
    """Warm up, then time `steps` calls; returns (total ms of the region, [ms per call])."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(steps):
        ev[i][0].record(stream)
        fn()
        ev[i][1].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    per = [a.elapsed_time(b) for a, b in ev]
    return start.elapsed_time(end), per


def _reduce_scalar(x, dist, op):
    if dist is None:
        return x
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(x, dist):
    """Slowest rank's time: the whole job is done only when every rank is."""
    return _reduce_scalar(x, dist, None if dist is None else dist.ReduceOp.MAX)


def sum_over_ranks(x, dist):
    """Units processed by all ranks together (weak scaling: each rank has its own)."""
    return _reduce_scalar(x, dist, None if dist is None else dist.ReduceOp.SUM)


def rank_seed(base, rank):
    """Each rank draws its own synthetic inputs."""
    return base + 1000 * rank


def whole_job_rate(units_per_rank, ms_per_rank, dist):
    """Units per second of the whole job: all ranks' units over the slowest rank's time."""
    return sum_over_ranks(units_per_rank, dist) / (max_over_ranks(ms_per_rank, dist) * 1e-3)


def run_gpu(args, rank, world, dist):
    import torch
    from local_linear_attention_streamed_b200 import plx, synth

    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    peaks, peak_src = load_peaks()
    seed = rank_seed(1002, rank)

    # ---- Decode (headline).
    B, H, L, d = args.decode_batch, DECODE["H"], DECODE["L"], DECODE["d"]
    specs = synth.decode_specs(B, H, L, d)
    t = {}
    for name, spec in specs.items():
        t[name] = torch.empty(spec.shape, dtype=torch.bfloat16, device=dev)
        synth.device_fill(t[name].data_ptr(), synth.BF16, seed, spec)
    sl_host = synth.seqlens(seed, B, L, ragged=False)
    sl = torch.from_numpy(sl_host).to(dev)
    out = torch.empty_like(t["q"])
    kv_bytes, alg_bytes = decode_bytes(sl_host, H, d)

    def dec():
        plx.decode(t["q"], t["r"], t["K"], t["V"], sl, out=out)

    clk = ClockSampler(torch.cuda.current_device()).__enter__()
    total_ms, per = timed(dec, args.steps, args.warmup, stream, dist)
    status = plx.get_device_status()
    if status != 0:
        raise RuntimeError(f"decode reported {plx.status_string(status)}")
    total_ms = max_over_ranks(total_ms, dist)
    ms_step = total_ms / args.steps
    kernel_ms = float(np.mean(per))
    value = sum_over_ranks(kv_bytes * args.steps, dist) / (total_ms * 1e-3) / 1e9
    achieved = alg_bytes / (kernel_ms * 1e-3) / 1e9
    src_hash = kernel_hash("decode_gqa_tc.cu", "decode_tc_common.cuh", "sm100.cuh")
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                # The committed capture is of the default workload; other sizes report none.
                "traffic": (traffic_from_profile("decode_bf16_B64_H16_L4096.json", src_hash)
                            if B == DECODE["B"] else None),
                "peak_source": peak_src, "kernel": "decode_gqa_tc_kernel<128, 1>",
                "algorithmic_bytes_per_launch": alg_bytes,
                "frac_of_spec_8000": round(achieved / 8000.0, 4)}

    # ---- e2e: host buffers in pinned memory, copies inside the timed region.
    e2e = None
    if not args.no_e2e:
        host = {n: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for n, v in t.items()}
        for n in host:
            host[n].copy_(t[n])
        sl_pinned = torch.from_numpy(sl_host.copy()).pin_memory()
        out_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        d_in = {n: torch.empty_like(v) for n, v in t.items()}
        d_sl = torch.empty_like(sl)
        d_out = torch.empty_like(out)

        def e2e_step():
            for n in d_in:
                d_in[n].copy_(host[n], non_blocking=True)
            d_sl.copy_(sl_pinned, non_blocking=True)
            plx.decode(d_in["q"], d_in["r"], d_in["K"], d_in["V"], d_sl, out=d_out)
            out_host.copy_(d_out, non_blocking=True)

        e_steps = max(1, min(args.steps, 5))
        e_ms, _ = timed(e2e_step, e_steps, 1, stream, dist)
        e_ms = max_over_ranks(e_ms, dist)
        h2d = sum(v.numel() * v.element_size() for v in host.values()) + sl_pinned.numel() * 4
        d2h = out_host.numel() * out_host.element_size()
        e2e = {"value": round(sum_over_ranks(kv_bytes * e_steps, dist) / (e_ms * 1e-3) / 1e9, 2),
               "unit": "GB/s", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(e_ms / e_steps, 3)}
        del host, d_in
    del t
    torch.cuda.empty_cache()

    # ---- Prefill.
    prefill = None
    if not args.no_prefill:
        pB, pH, pN, pd = args.prefill_batch, PREFILL["H"], PREFILL["N"], PREFILL["d"]
        pspecs = synth.prefill_specs(pB, pH, pN, pd)
        pt = {}
        for name, spec in pspecs.items():
            pt[name] = torch.empty(spec.shape, dtype=torch.bfloat16, device=dev)
            synth.device_fill(pt[name].data_ptr(), synth.BF16, seed + 2, spec)
        pout = torch.empty_like(pt["Q"])

        def pre():
            plx.prefill(pt["Q"], pt["K"], pt["V"], pt["R"], causal=True, out=pout)

        psteps = max(1, args.steps // 2)
        p_total, p_per = timed(pre, psteps, max(3, args.warmup // 2), stream, dist)
        if plx.get_device_status() != 0:
            raise RuntimeError("prefill reported a device error")
        p_total = max_over_ranks(p_total, dist)
        flops = prefill_flops(pB, pH, pN, pd)
        p_kernel_ms = float(np.mean(p_per))
        p_ach = flops / (p_kernel_ms * 1e-3) / 1e12
        prefill = {
            "metric": "causal prefill TFLOP/s", "unit": "TFLOP/s",
            "value": round(sum_over_ranks(flops * psteps, dist) / (p_total * 1e-3) / 1e12, 2),
            "ms_per_step": round(p_total / psteps, 3), "steps": psteps,
            "config": {"workload": f"causal prefill B={pB} H=16 N=4096 d=128 bf16",
                       "l2": f"inputs {4 * pB * 16 * 4096 * 128 * 2 >> 20} MB"
                             + (", larger than L2" if 4 * pB * 16 * 4096 * 128 * 2 > L2_BYTES else "")},
            "roofline": {"bound": "tensor", "achieved": round(p_ach, 1), "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": round(p_ach / peaks["bf16_tflops"], 4),
                         "frac_of_sustained": round(p_ach / peaks["bf16_tflops_sustained"], 4),
                         "traffic": (traffic_from_profile("prefill_B8_H16_N4096.json",
                                                          kernel_hash("prefill_tc.cu", "sm100.cuh"))
                                     if pB == PREFILL["B"] else None),
                         # ncu: sm__pipe_tensor_cycles_active (% of peak, elapsed) of one full-size launch
                         "tensor_pipe_active_pct": (profile_field("prefill_B8_H16_N4096.json",
                                                                  kernel_hash("prefill_tc.cu", "sm100.cuh"),
                                                                  "tensor_pipe_active_pct")
                                                    if pB == PREFILL["B"] else None),
                         "peak_source": peak_src, "algorithmic_flops_per_launch": flops},
            "gpu_launches": psteps,
        }
        del pt
        torch.cuda.empty_cache()
        # Head dim 64 at the same width (same Q, K, V, R bytes).
        qB, qH, qN, qd = (PREFILL_D64[k] for k in ("B", "H", "N", "d"))
        qspecs = synth.prefill_specs(qB, qH, qN, qd)
        qt = {}
        for name, spec in qspecs.items():
            qt[name] = torch.empty(spec.shape, dtype=torch.bfloat16, device=dev)
            synth.device_fill(qt[name].data_ptr(), synth.BF16, seed + 6, spec)
        qout = torch.empty_like(qt["Q"])

        def pre64():
            plx.prefill(qt["Q"], qt["K"], qt["V"], qt["R"], causal=True, out=qout)

        q_total, q_per = timed(pre64, psteps, max(3, args.warmup // 2), stream, dist)
        if plx.get_device_status() != 0:
            raise RuntimeError("prefill (d = 64) reported a device error")
        q_total = max_over_ranks(q_total, dist)
        qflops = prefill_flops(qB, qH, qN, qd)
        q_ach = qflops / (float(np.mean(q_per)) * 1e-3) / 1e12
        prefill["d64"] = {
            "workload": f"causal prefill B={qB} H={qH} N={qN} d={qd} bf16 (head dim halved, same width)",
            "value": round(sum_over_ranks(qflops * psteps, dist) / (q_total * 1e-3) / 1e12, 2),
            "unit": "TFLOP/s", "ms_per_step": round(q_total / psteps, 3),
            "kernel_tflops": round(q_ach, 1), "frac": round(q_ach / peaks["bf16_tflops"], 4),
        }
        del qt
        torch.cuda.empty_cache()

        # Training: forward that saves the backward's inputs, then the backward
        # pass (three launches: statistics, dK/dV, dQ/dR) on the same workload.
        if not args.no_backward:
            bspecs = synth.backward_specs(pB, pH, pN, pd)
            bt = {}
            for name, spec in bspecs.items():
                bt[name] = torch.empty(spec.shape, dtype=torch.bfloat16, device=dev)
                synth.device_fill(bt[name].data_ptr(), synth.BF16, seed + 7, spec)
            saved = plx.prefill_train(bt["Q"], bt["K"], bt["V"], bt["R"], True)
            grads = tuple(torch.empty_like(bt["Q"]) for _ in range(4))
            bws = torch.empty(plx.prefill_bwd_workspace_bytes(pB, pH, pN, pd) // 4, dtype=torch.float32,
                              device=dev)

            def trn():
                plx.prefill_train(bt["Q"], bt["K"], bt["V"], bt["R"], True)

            def bwd():
                plx.prefill_backward(bt["Q"], bt["K"], bt["V"], bt["R"], *saved, bt["dO"], True, grads=grads,
                                     workspace=bws)

            t_total, t_per = timed(trn, psteps, max(3, args.warmup // 2), stream, dist)
            b_total, b_per = timed(bwd, psteps, max(3, args.warmup // 2), stream, dist)
            if plx.get_device_status() != 0:
                raise RuntimeError("backward reported a device error")
            b_total = max_over_ranks(b_total, dist)
            bflops = backward_flops(pB, pH, pN, pd)
            b_ach = bflops / (float(np.mean(b_per)) * 1e-3) / 1e12
            t_ms = float(np.mean(t_per))
            prefill["backward"] = {
                "workload": f"causal prefill backward B={pB} H={pH} N={pN} d={pd} bf16 "
                            "(dQ, dK, dV, dR from dO and the training forward's out, vbar, lse, tbar)",
                "metric": "backward TFLOP/s", "unit": "TFLOP/s",
                "value": round(sum_over_ranks(bflops * psteps, dist) / (b_total * 1e-3) / 1e12, 2),
                "ms_per_step": round(b_total / psteps, 3), "steps": psteps,
                "achieved": round(b_ach, 1), "frac": round(b_ach / peaks["bf16_tflops"], 4),
                "frac_of_sustained": round(b_ach / peaks["bf16_tflops_sustained"], 4),
                "algorithmic_flops_per_step": bflops,
                "executed_mma_flops_per_step": bflops * 11.0 / 8.0,
                "flops_note": "algorithmic = 8 GEMMs per visible pair; the two kernels issue 11 "
                              "(the scores are recomputed in the dQ/dR kernel)",
                "gpu_launches_per_step": 3,
                "traffic_per_step": (traffic_from_profile("backward_B8_H16_N4096.json",
                                                          kernel_hash("backward_tc.cu", "sm100.cuh"))
                                     if pB == PREFILL["B"] else None),
                "algorithmic_bytes_per_step": backward_bytes(pB, pH, pN, pd),
                "train_forward_ms": round(t_ms, 3),
                "train_forward_tflops": round(flops / (t_ms * 1e-3) / 1e12, 1),
                "train_step_ms": round(t_ms + float(np.mean(b_per)), 3),
            }
            del bt, saved, grads, bws
            torch.cuda.empty_cache()

        # Grouped KV heads on the same query workload (G = 4): forward, and
        # the training forward plus backward.
        if not args.no_gqa:
            gHkv = pH // 4
            gspecs = synth.backward_specs(pB, pH, pN, pd)
            for n, tid in (("K", synth.TID_K), ("V", synth.TID_V)):
                gspecs[n] = synth.TensorSpec(tid, (pB, gHkv, pN, pd), gspecs[n].dist, gspecs[n].sigma)
            gt = {}
            for name, spec in gspecs.items():
                gt[name] = torch.empty(spec.shape, dtype=torch.bfloat16, device=dev)
                synth.device_fill(gt[name].data_ptr(), synth.BF16, seed + 8, spec)
            gout = torch.empty_like(gt["Q"])

            def gfwd():
                plx.prefill_gqa(gt["Q"], gt["K"], gt["V"], gt["R"], True, out=gout)

            gf_total, gf_per = timed(gfwd, psteps, max(3, args.warmup // 2), stream, dist)
            gf_total = max_over_ranks(gf_total, dist)
            entry = {
                "workload": f"causal prefill B={pB} H={pH} Hkv={gHkv} N={pN} d={pd} bf16 (grouped KV heads, G=4)",
                "value": round(sum_over_ranks(flops * psteps, dist) / (gf_total * 1e-3) / 1e12, 2),
                "unit": "TFLOP/s", "ms_per_step": round(gf_total / psteps, 3),
                "kernel_tflops": round(flops / (float(np.mean(gf_per)) * 1e-3) / 1e12, 1),
            }
            if not args.no_backward:
                gsaved = plx.prefill_train(gt["Q"], gt["K"], gt["V"], gt["R"], True)
                ggrads = (torch.empty_like(gt["Q"]), torch.empty_like(gt["K"]), torch.empty_like(gt["V"]),
                          torch.empty_like(gt["Q"]))
                gws = torch.empty(plx.prefill_bwd_workspace_bytes(pB, pH, pN, pd) // 4, dtype=torch.float32,
                                  device=dev)

                def gbwd():
                    plx.prefill_backward(gt["Q"], gt["K"], gt["V"], gt["R"], *gsaved, gt["dO"], True,
                                         grads=ggrads, workspace=gws)

                gb_total, gb_per = timed(gbwd, psteps, max(3, args.warmup // 2), stream, dist)
                gb_total = max_over_ranks(gb_total, dist)
                gbflops = backward_flops(pB, pH, pN, pd)
                entry["backward"] = {
                    "value": round(sum_over_ranks(gbflops * psteps, dist) / (gb_total * 1e-3) / 1e12, 2),
                    "unit": "TFLOP/s", "ms_per_step": round(gb_total / psteps, 3),
                    "kernel_tflops": round(gbflops / (float(np.mean(gb_per)) * 1e-3) / 1e12, 1),
                    "gpu_launches_per_step": 3,
                }
                del gsaved, ggrads, gws
            if plx.get_device_status() != 0:
                raise RuntimeError("grouped-KV prefill reported a device error")
            prefill["gqa"] = entry
            del gt, gout
            torch.cuda.empty_cache()

    # ---- Decode with grouped KV heads (the next row of the scope: one KV stream per group).
    # ---- Sliding-window variants (a window of 1024 keys on the prefill and decode workloads).
    win = None
    if not args.no_window:
        W = WINDOW
        wB, wH, wN, wd = args.prefill_batch, PREFILL["H"], PREFILL["N"], PREFILL["d"]
        wspecs = synth.prefill_specs(wB, wH, wN, wd)
        wt = {}
        for name, spec in wspecs.items():
            wt[name] = torch.empty(spec.shape, dtype=torch.bfloat16, device=dev)
            synth.device_fill(wt[name].data_ptr(), synth.BF16, seed + 8, spec)
        wout = torch.empty_like(wt["Q"])

        def wpre():
            plx.prefill_window(wt["Q"], wt["K"], wt["V"], wt["R"], W, out=wout)

        wsteps = max(1, args.steps // 2)
        w_total, w_per = timed(wpre, wsteps, max(3, args.warmup // 2), stream, dist)
        pairs = (W * (W + 1) // 2 + (wN - W) * W) * wB * wH
        wflops = 8.0 * wd * pairs
        w_ach = wflops / (float(np.mean(w_per)) * 1e-3) / 1e12
        del wt, wout
        dB, dH, dL, dd = args.decode_batch, DECODE["H"], DECODE["L"], DECODE["d"]
        dspecs = synth.decode_specs(dB, dH, dL, dd)
        dt_ = {}
        for name, spec in dspecs.items():
            dt_[name] = torch.empty(spec.shape, dtype=torch.bfloat16, device=dev)
            synth.device_fill(dt_[name].data_ptr(), synth.BF16, seed + 9, spec)
        dsl = torch.full((dB,), dL, dtype=torch.int32, device=dev)
        dout = torch.empty_like(dt_["q"])
        dws = torch.empty(max(16, lib_ws_window(plx, dB, dH, dH, dL, dd, W)), dtype=torch.uint8, device=dev)

        def wdec():
            plx.decode_window(dt_["q"], dt_["r"], dt_["K"], dt_["V"], dsl, W, out=dout, workspace=dws)

        # Block-sparse prefill on the same inputs shape: every 128-query tile sees
        # its diagonal blocks, the 16 key blocks (1024 keys) before them and the
        # first 2 blocks.
        nt, nkb = (wN + 127) // 128, (wN + 63) // 64
        bmask = np.array([[kb < 2 or 2 * t - 16 <= kb or kb // 2 == t for kb in range(nkb)] for t in range(nt)])
        wt2 = {}
        for name, spec in wspecs.items():
            wt2[name] = torch.empty(spec.shape, dtype=torch.bfloat16, device=dev)
            synth.device_fill(wt2[name].data_ptr(), synth.BF16, seed + 10, spec)
        sout = torch.empty_like(wt2["Q"])

        def spre():
            plx.prefill_block_sparse(wt2["Q"], wt2["K"], wt2["V"], wt2["R"], bmask, out=sout)

        s_total, s_per = timed(spre, wsteps, max(3, args.warmup // 2), stream, dist)
        spairs = 0
        for i in range(wN):
            t = i // 128
            full = i // 64  # blocks strictly before key block of i are whole; i's own block is partial
            spairs += int(np.sum(bmask[t, :full])) * 64 + (i % 64 + 1)
        sflops = 8.0 * wd * spairs * wB * wH
        s_ach = sflops / (float(np.mean(s_per)) * 1e-3) / 1e12

        # Dilated prefill (dilation 4, the whole residue class: query i sees
        # keys i, i - 4, i - 8, ...) on the same inputs.
        DIL = 4

        def dpre():
            plx.prefill_dilated(wt2["Q"], wt2["K"], wt2["V"], wt2["R"], DIL, 0, out=sout)

        g_total, g_per = timed(dpre, wsteps, max(3, args.warmup // 2), stream, dist)
        n_cls = wN // DIL
        gflops = 8.0 * wd * DIL * n_cls * (n_cls + 1) / 2 * wB * wH
        g_ach = gflops / (float(np.mean(g_per)) * 1e-3) / 1e12
        del wt2, sout
        d_total, d_per = timed(wdec, args.steps, args.warmup, stream, dist)
        dbytes = dB * dH * min(W, dL) * dd * 2 * 2 + 3 * dB * dH * dd * 2
        if plx.get_device_status() != 0:
            raise RuntimeError("window kernels reported a device error")
        win = {
            "window": W,
            "prefill": {
                "workload": f"sliding-window prefill W={W} B={wB} H={wH} N={wN} d={wd} bf16",
                "value": round(sum_over_ranks(wflops * wsteps, dist) / (max_over_ranks(w_total, dist) * 1e-3) / 1e12, 2),
                "unit": "TFLOP/s", "kernel_tflops": round(w_ach, 1), "frac": round(w_ach / peaks["bf16_tflops"], 4),
                "algorithmic_flops_per_launch": wflops,
                "traffic": (traffic_from_profile("prefill_window_B8_H16_N4096_W1024.json",
                                                 kernel_hash("prefill_tc.cu", "sm100.cuh"))
                            if wB == PREFILL["B"] else None),
            },
            "block_sparse_prefill": {
                "workload": f"block-sparse prefill B={wB} H={wH} N={wN} d={wd} bf16: per 128-query tile its "
                            "diagonal blocks, the 16 64-key blocks before them and the first 2 blocks",
                "value": round(sum_over_ranks(sflops * wsteps, dist) / (max_over_ranks(s_total, dist) * 1e-3) / 1e12, 2),
                "unit": "TFLOP/s", "kernel_tflops": round(s_ach, 1), "frac": round(s_ach / peaks["bf16_tflops"], 4),
                "algorithmic_flops_per_launch": sflops,
            },
            "dilated_prefill": {
                "workload": f"dilated prefill B={wB} H={wH} N={wN} d={wd} bf16, dilation {DIL} (query i sees keys "
                            f"i, i - {DIL}, i - {2 * DIL}, ...)",
                "value": round(sum_over_ranks(gflops * wsteps, dist) / (max_over_ranks(g_total, dist) * 1e-3) / 1e12, 2),
                "unit": "TFLOP/s", "kernel_tflops": round(g_ach, 1), "frac": round(g_ach / peaks["bf16_tflops"], 4),
                "algorithmic_flops_per_launch": gflops,
            },
            "decode": {
                "workload": f"sliding-window decode W={W} B={dB} H={dH} L={dL} d={dd} bf16 (all lengths {dL})",
                "value": round(sum_over_ranks(dbytes * args.steps, dist) / (max_over_ranks(d_total, dist) * 1e-3) / 1e9, 1),
                "unit": "GB/s", "kernel_gbs": round(dbytes / (float(np.mean(d_per)) * 1e-3) / 1e9, 1),
                "frac": round(dbytes / (float(np.mean(d_per)) * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                "algorithmic_bytes_per_launch": dbytes,
                "traffic": (traffic_from_profile("decode_window_B64_H16_L4096_W1024.json",
                                                kernel_hash("decode_gqa_tc.cu", "decode_tc_common.cuh", "sm100.cuh"))
                            if dB == DECODE["B"] else None),
            },
        }
        del dt_, dout, dws
        torch.cuda.empty_cache()

    gqa = None
    if not args.no_gqa:
        gB, gH, gHkv, gL, gd = (DECODE_GQA[k] for k in ("B", "H", "Hkv", "L", "d"))
        gspecs = synth.decode_gqa_specs(gB, gH, gHkv, gL, gd)
        gt = {}
        for name, spec in gspecs.items():
            gt[name] = torch.empty(spec.shape, dtype=torch.bfloat16, device=dev)
            synth.device_fill(gt[name].data_ptr(), synth.BF16, seed + 5, spec)
        gsl = torch.full((gB,), gL, dtype=torch.int32, device=dev)
        gout = torch.empty_like(gt["q"])

        def gdec():
            plx.decode_gqa(gt["q"], gt["r"], gt["K"], gt["V"], gsl, out=gout)

        gsteps = max(1, args.steps // 2)
        g_total, g_per = timed(gdec, gsteps, max(3, args.warmup // 2), stream, dist)
        if plx.get_device_status() != 0:
            raise RuntimeError("grouped decode reported a device error")
        g_total = max_over_ranks(g_total, dist)
        g_kv = gB * gHkv * gL * gd * 2 * 2
        g_alg = g_kv + 3 * gB * gH * gd * 2
        g_kernel_ms = float(np.mean(g_per))
        g_ach = g_alg / (g_kernel_ms * 1e-3) / 1e9
        gqa = {
            "metric": "grouped-KV decode KV GB/s", "unit": "GB/s",
            "value": round(sum_over_ranks(g_kv * gsteps, dist) / (g_total * 1e-3) / 1e9, 2),
            "ms_per_step": round(g_total / gsteps, 4), "steps": gsteps,
            "config": {"workload": f"decode B={gB} H={gH} Hkv={gHkv} (groups of {gH // gHkv}) "
                                   f"L={gL} d={gd} bf16, all seqlens {gL}",
                       "l2": f"inputs larger than L2 ({g_kv / 1e9:.2f} GB KV); no flush"},
            "roofline": {"bound": "hbm", "achieved": round(g_ach, 1), "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": round(g_ach / peaks["hbm_gbs"], 4),
                         "traffic": (traffic_from_profile("decode_gqa_B64_H32_Hkv8_L4096.json",
                                                          kernel_hash("decode_gqa_tc.cu", "decode_tc_common.cuh", "sm100.cuh"))
                                     if (gB, gH, gHkv, gL, gd) == (64, 32, 8, 4096, 128) else None),
                         "peak_source": peak_src, "kernel": (f"decode_gqa_tc_kernel<{gd}, {gH // gHkv}>" if gd == 128 or gHkv % 2 == 0
                                    else f"decode_gqa_kernel<{gd}, {gH // gHkv}>"),
                         "algorithmic_bytes_per_launch": g_alg},
            "gpu_launches": gsteps,
        }
        del gt
        torch.cuda.empty_cache()
        # Head dim halved at the same width (64 x 32 heads): the tensor-core
        # decode takes two heads a unit.
        hB, hH, hL, hd = DECODE["B"], 32, DECODE["L"], 64
        hspecs = synth.decode_specs(hB, hH, hL, hd)
        ht = {}
        for name, spec in hspecs.items():
            ht[name] = torch.empty(spec.shape, dtype=torch.bfloat16, device=dev)
            synth.device_fill(ht[name].data_ptr(), synth.BF16, seed + 8, spec)
        hsl = torch.full((hB,), hL, dtype=torch.int32, device=dev)
        hout = torch.empty_like(ht["q"])

        def hdec():
            plx.decode(ht["q"], ht["r"], ht["K"], ht["V"], hsl, out=hout)

        h_total, h_per = timed(hdec, gsteps, max(3, args.warmup // 2), stream, dist)
        if plx.get_device_status() != 0:
            raise RuntimeError("d = 64 decode reported a device error")
        h_kv = hB * hH * hL * hd * 2 * 2
        h_alg = h_kv + 3 * hB * hH * hd * 2
        h_ach = h_alg / (float(np.mean(h_per)) * 1e-3) / 1e9
        gqa["d64"] = {
            "workload": f"decode B={hB} H={hH} L={hL} d={hd} bf16, all lengths {hL} (head dim halved, same width)",
            "value": round(sum_over_ranks(h_kv * gsteps, dist) / (max_over_ranks(h_total, dist) * 1e-3) / 1e9, 2),
            "unit": "GB/s", "kernel_gbs": round(h_ach, 1), "frac": round(h_ach / peaks["hbm_gbs"], 4),
            "kernel": ("decode_gqa_tc_kernel<64, 1> (two heads a unit)" if plx.lib.plx_decode_uses_tc(hB, hH, hL, hd)
                       else "decode_bf16_kernel<64>"),
            "algorithmic_bytes_per_launch": h_alg,
        }
        del ht
        torch.cuda.empty_cache()
        # Grouped cells at B=64, Hkv=8, L=4096: groups of 8 at d = 128 and the
        # head-pair form at d = 64 (two KV heads a unit) for groups of 2, 4, 8.
        cells = []
        for (cd, cG) in [(128, 8), (64, 2), (64, 4), (64, 8)]:
            cB, cHkv, cL = 64, 8, 4096
            cH = cG * cHkv
            cspecs = synth.decode_gqa_specs(cB, cH, cHkv, cL, cd)
            ct = {}
            for name, spec in cspecs.items():
                ct[name] = torch.empty(spec.shape, dtype=torch.bfloat16, device=dev)
                synth.device_fill(ct[name].data_ptr(), synth.BF16, seed + 9, spec)
            csl = torch.full((cB,), cL, dtype=torch.int32, device=dev)
            cout = torch.empty_like(ct["q"])

            def cdec():
                plx.decode_gqa(ct["q"], ct["r"], ct["K"], ct["V"], csl, out=cout)

            c_total, c_per = timed(cdec, gsteps, max(3, args.warmup // 2), stream, dist)
            if plx.get_device_status() != 0:
                raise RuntimeError("grouped decode reported a device error")
            c_alg = cB * cHkv * cL * cd * 2 * 2 + 3 * cB * cH * cd * 2
            c_ach = c_alg / (float(np.mean(c_per)) * 1e-3) / 1e9
            cells.append({"d": cd, "groups": cG, "workload": f"decode B={cB} H={cH} Hkv={cHkv} L={cL} d={cd} bf16",
                          "kernel_gbs": round(c_ach, 1), "frac": round(c_ach / peaks["hbm_gbs"], 4),
                          "kernel": f"decode_gqa_tc_kernel<{cd}, {cG}>", "algorithmic_bytes_per_launch": c_alg})
            del ct
            torch.cuda.empty_cache()
        gqa["cells"] = cells

    # ---- Decode over an e4m3 KV cache: the decode workload's shape, and groups of 4.
    fp8kv = None
    if not args.no_fp8kv:
        fp8kv = {}
        for (fB, fH, fHkv, fL, fd) in [(DECODE["B"], DECODE["H"], DECODE["H"], DECODE["L"], DECODE["d"]),
                                       tuple(DECODE_GQA[k] for k in ("B", "H", "Hkv", "L", "d"))]:
            fspecs = synth.decode_gqa_specs(fB, fH, fHkv, fL, fd)
            ft = {}
            for name, spec in fspecs.items():
                ft[name] = torch.empty(spec.shape, dtype=torch.bfloat16, device=dev)
                synth.device_fill(ft[name].data_ptr(), synth.BF16, seed + 6, spec)
            Kc, Ks = plx.kv_quantize_fp8(ft["K"])
            Vc, Vs = plx.kv_quantize_fp8(ft["V"])
            del ft["K"], ft["V"]
            fsl = torch.full((fB,), fL, dtype=torch.int32, device=dev)
            fout = torch.empty_like(ft["q"])

            def fdec():
                plx.decode_fp8kv(ft["q"], ft["r"], Kc, Ks, Vc, Vs, fsl, out=fout)

            fsteps = max(1, args.steps // 2)
            f_total, f_per = timed(fdec, fsteps, max(3, args.warmup // 2), stream, dist)
            if plx.get_device_status() != 0:
                raise RuntimeError("fp8-cache decode reported a device error")
            f_total = max_over_ranks(f_total, dist)
            f_kv = fB * fHkv * fL * (fd + 4) * 2          # codes and scales of K and V
            f_alg = f_kv + 3 * fB * fH * fd * 2           # + q, r, out
            f_ms = float(np.mean(f_per))
            f_ach = f_alg / (f_ms * 1e-3) / 1e9
            keys = fB * fHkv * fL
            entry = {
                "metric": "fp8-cache decode KV GB/s", "unit": "GB/s",
                "value": round(sum_over_ranks(f_kv * fsteps, dist) / (f_total * 1e-3) / 1e9, 2),
                "ms_per_step": round(f_total / fsteps, 4), "steps": fsteps,
                "cached_rows_per_s": round(sum_over_ranks(keys * fsteps, dist) / (f_total * 1e-3), 1),
                "config": {"workload": f"decode B={fB} H={fH} Hkv={fHkv} L={fL} d={fd}, e4m3 cache with "
                                       f"per-row fp32 scales ({f_kv / 1e9:.2f} GB), bf16 q, rho, out",
                           "l2": "inputs larger than L2; no flush"},
                "roofline": {"bound": "hbm", "achieved": round(f_ach, 1), "peak": peaks["hbm_gbs"],
                             "unit": "GB/s", "frac": round(f_ach / peaks["hbm_gbs"], 4),
                             "traffic": (traffic_from_profile("decode_fp8kv_B64_H16_L4096.json",
                                                              kernel_hash("decode_fp8kv.cu", "decode_tc_common.cuh",
                                                                          "sm100.cuh"))
                                         if (fB, fH, fHkv) == (DECODE["B"], DECODE["H"], DECODE["H"]) else None),
                             "peak_source": peak_src, "kernel": f"decode_fp8kv_kernel<{fH // fHkv}>",
                             "algorithmic_bytes_per_launch": f_alg},
                "gpu_launches": fsteps,
            }
            fp8kv["groups_of_%d" % (fH // fHkv)] = entry
            del ft, Kc, Vc, Ks, Vs
            torch.cuda.empty_cache()

    # ---- A fixed subset of the decode sweep (batch x context, ragged lengths).
    sweep = None
    if not args.no_sweep and dist is None:
        sweep = [sweep_cell(sB, sL, max(5, args.steps // 5), 3, peaks) for (sB, sL) in SWEEP_SUBSET]

    # ---- Full layer (x [4, 8192, 2048], 16 heads of 128).
    layer = None
    if not args.no_layer:
        LB, LN, LD, LH = LAYER["B"], LAYER["N"], LAYER["D"], LAYER["H"]
        lspecs = synth.layer_specs(LB, LN, LD)
        lt = {}
        for name, spec in lspecs.items():
            lt[name] = torch.empty(spec.shape, dtype=torch.bfloat16, device=dev)
            synth.device_fill(lt[name].data_ptr(), synth.BF16, seed + 3, spec)
        y = torch.empty_like(lt["x"])

        def lay():
            plx.layer_forward(lt["x"], lt["WQ"], lt["WK"], lt["WV"], lt["WR"], lt["WO"], LH, out=y)

        lsteps = max(1, args.steps // 4)
        l_total, l_per = timed(lay, lsteps, 3, stream, dist)
        if plx.get_device_status() != 0:
            raise RuntimeError("layer reported a device error")
        # The attention inside the layer on inputs of the same shape.
        ad = LD // LH
        aspecs = synth.prefill_specs(LB, LH, LN, ad)
        at = {}
        for name, spec in aspecs.items():
            at[name] = torch.empty(spec.shape, dtype=torch.bfloat16, device=dev)
            synth.device_fill(at[name].data_ptr(), synth.BF16, seed + 4, spec)
        aout = torch.empty_like(at["Q"])

        def att():
            plx.prefill(at["Q"], at["K"], at["V"], at["R"], causal=True, out=aout)

        a_total, a_per = timed(att, lsteps, 3, stream, dist)
        l_ms, a_ms = float(np.mean(l_per)), float(np.mean(a_per))
        aflops = prefill_flops(LB, LH, LN, ad)
        pflops = 5 * 2.0 * LB * LN * LD * LD  # q, k, v, rho and output projections
        layer = {
            "config": {"workload": "layer x[4, 8192, 2048] bf16, 16 heads of 128, causal"},
            "layer_ms": round(l_ms, 3),
            "attention_ms": round(a_ms, 3),
            "attention_tflops": round(aflops / (a_ms * 1e-3) / 1e12, 1),
            "attention_flops": aflops,
            "rest_ms": round(l_ms - a_ms, 3),
            "rest_note": "projections (cuBLAS bf16, 1.37e12 flops), RMSNorm+RoPE, head split/merge",
            "projection_flops": pflops,
            "layer_tflops_all": round((aflops + pflops) / (l_ms * 1e-3) / 1e12, 1),
            "gpu_launches_per_step": {"own_kernels": 6, "cublas_gemms": 5},
        }

        # The same layer with its five linears in dynamic fp8 (per-tensor e4m3).
        def lay8():
            plx.layer_forward_fp8(lt["x"], lt["WQ"], lt["WK"], lt["WV"], lt["WR"], lt["WO"], LH, out=y)

        f_total, f_per = timed(lay8, lsteps, 3, stream, dist)
        if plx.get_device_status() != 0:
            raise RuntimeError("fp8 layer reported a device error")
        f_ms = float(np.mean(f_per))
        layer["fp8_linears"] = {
            "layer_ms": round(f_ms, 3),
            "rest_ms": round(f_ms - a_ms, 3),
            "note": "x, the weights and the attention output quantised per tensor to e4m3 every call "
                    "(|max| reductions and quantisers: own kernels), e4m3 GEMMs through cuBLASLt",
            "gpu_launches_per_step": {"own_kernels": 6 + 6, "cublaslt_gemms": 5},
        }
        del lt, at
        torch.cuda.empty_cache()

    clk.__exit__(None, None, None)
    return {
        "value": round(value, 2), "ms_per_step": round(ms_step, 4), "roofline": roofline,
        "e2e": e2e, "clocks": clk.summary(), "prefill": prefill, "layer": layer, "decode_gqa": gqa,
        "window": win, "decode_fp8kv": fp8kv, "decode_sweep": sweep,
        "gpu_launches": args.steps,
        "kernel_ms": kernel_ms,
    }


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm).
# ---------------------------------------------------------------------------

def oracle_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        if info:
            return max(i.get("num_threads", 1) for i in info)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


_POOLS = {}


def _decode_pool(seed=1002, units=4):
    """A few whole (b, h) decode units generated once on the host (not timed)."""
    key = ("decode", seed, units)
    if key not in _POOLS:
        from local_linear_attention_streamed_b200 import synth
        B, H, L, d = DECODE["B"], DECODE["H"], DECODE["L"], DECODE["d"]
        specs = synth.decode_specs(B, H, L, d)
        rng = np.random.default_rng(0)
        pool = []
        for _ in range(units):
            b, h = int(rng.integers(B)), int(rng.integers(H))
            r0 = (b * H + h) * L
            pool.append((synth.host_rows_f64(seed, specs["q"], synth.BF16, b * H + h, 1)[0],
                         synth.host_rows_f64(seed, specs["r"], synth.BF16, b * H + h, 1)[0],
                         synth.host_rows_f64(seed, specs["K"], synth.BF16, r0, L),
                         synth.host_rows_f64(seed, specs["V"], synth.BF16, r0, L)))
        _POOLS[key] = pool
    return _POOLS[key]


def _prefill_pool(seed=1004, rows=8):
    """A few causal rows of the prefill workload generated once on the host (not timed)."""
    key = ("prefill", seed, rows)
    if key not in _POOLS:
        from local_linear_attention_streamed_b200 import synth
        B, H, N, d = PREFILL["B"], PREFILL["H"], PREFILL["N"], PREFILL["d"]
        specs = synth.prefill_specs(B, H, N, d)
        rng = np.random.default_rng(1)
        pool = []
        for _ in range(rows):
            b, h, i = int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(N))
            r0 = (b * H + h) * N
            pool.append((synth.host_rows_f64(seed, specs["Q"], synth.BF16, r0 + i, 1)[0],
                         synth.host_rows_f64(seed, specs["R"], synth.BF16, r0 + i, 1)[0],
                         synth.host_rows_f64(seed, specs["K"], synth.BF16, r0, i + 1),
                         synth.host_rows_f64(seed, specs["V"], synth.BF16, r0, i + 1)))
        _POOLS[key] = pool
    return _POOLS[key]


def oracle_decode_sample(budget_s):
    """Times the oracle on whole (b, h) units of the decode workload; returns (GB/s, units, s)."""
    import oracle
    pool = _decode_pool()
    done, secs, nbytes = 0, 0.0, 0
    while secs < budget_s or done == 0:
        q, r, K, V = pool[done % len(pool)]
        t0 = time.perf_counter()
        oracle.parallax_row(q, r, K, V)
        secs += time.perf_counter() - t0
        nbytes += K.shape[0] * K.shape[1] * 2 * 2
        done += 1
    return nbytes / secs / 1e9, done, secs


def oracle_prefill_sample(budget_s):
    """Times the oracle on causal rows of the prefill workload; returns (TFLOP/s, rows, s)."""
    import oracle
    pool = _prefill_pool()
    done, secs, flops = 0, 0.0, 0.0
    while secs < budget_s or done == 0:
        q, r, K, V = pool[done % len(pool)]
        t0 = time.perf_counter()
        oracle.parallax_row(q, r, K, V)
        secs += time.perf_counter() - t0
        flops += 8.0 * K.shape[1] * K.shape[0]
        done += 1
    return flops / secs / 1e12, done, secs


# ---------------------------------------------------------------------------
# Sweep.
# ---------------------------------------------------------------------------

def sweep_cell(B, L, steps, warmup, peaks, dist=None, seed=1003):
    """One decode sweep cell (H=16, d=128 bf16, lengths uniform on [L/2, L]):
    GB/s of algorithmic bytes per launch, CUDA events on the launching stream."""
    import torch
    from local_linear_attention_streamed_b200 import plx, synth
    H, d = 16, 128
    stream = torch.cuda.current_stream()
    alloc = B * H * L * d * 2 * 2
    specs = synth.decode_specs(B, H, L, d)
    t = {}
    for name, spec in specs.items():
        t[name] = torch.empty(spec.shape, dtype=torch.bfloat16, device="cuda")
        synth.device_fill(t[name].data_ptr(), synth.BF16, seed, spec)
    sl_host = synth.seqlens(seed, B, L, ragged=True)
    sl = torch.from_numpy(sl_host).cuda()
    out = torch.empty_like(t["q"])
    kv, alg = decode_bytes(sl_host, H, d)
    # Cells that fit in L2 rotate through enough copies to defeat it.
    copies = 1 if alloc > 4 * L2_BYTES else int(math.ceil(4 * L2_BYTES / alloc))
    extra = [{n: v.clone() for n, v in t.items()} for _ in range(copies - 1)]
    sets = [t] + extra
    idx = [0]

    def fn():
        s = sets[idx[0] % len(sets)]
        idx[0] += 1
        plx.decode(s["q"], s["r"], s["K"], s["V"], sl, out=out)

    total, per = timed(fn, steps, warmup, stream, dist)
    if plx.get_device_status() != 0:
        raise RuntimeError(f"decode sweep cell {(B, L)} reported a device error")
    ms = float(np.mean(per))
    cell = {"cell": [B, L], "kv_gb": round(kv / 1e9, 4), "us_per_launch": round(ms * 1e3, 2),
            "GBps": round(alg / (ms * 1e-3) / 1e9, 1),
            "frac_hbm": round(alg / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "splits": plx.lib.plx_decode_num_splits(B, H, L, d),
            "kernel": "tensor-core" if plx.lib.plx_decode_uses_tc(B, H, L, d) else "warp-mma",
            "l2_copies": copies}
    del t, extra, sets
    torch.cuda.empty_cache()
    return cell


def run_sweep(args):
    peaks, peak_src = load_peaks()
    H, d = 16, 128
    for B in SWEEP_B:
        for L in SWEEP_L:
            alloc = B * H * L * d * 2 * 2
            if alloc > SWEEP_MAX_BYTES:
                print(json.dumps({"cell": [B, L], "skipped": f"KV cache {alloc / 1e9:.1f} GB > 150 GB"}))
                continue
            print(json.dumps(sweep_cell(B, L, args.steps, args.warmup, peaks)), flush=True)


# ---------------------------------------------------------------------------
# One workload, a few launches (what profiler captures run: one kernel, a few
# launches, a few GB on the device).
# ---------------------------------------------------------------------------

ONLY = ("decode", "decode_gqa", "decode_window", "decode_fp8kv", "prefill", "prefill_window", "backward")


def run_only(name, launches=4):
    import torch
    from local_linear_attention_streamed_b200 import plx, synth
    dev = torch.device("cuda", torch.cuda.current_device())

    def fill(specs, seed):
        t = {}
        for n, spec in specs.items():
            t[n] = torch.empty(spec.shape, dtype=torch.bfloat16, device=dev)
            synth.device_fill(t[n].data_ptr(), synth.BF16, seed, spec)
        return t

    if name in ("decode", "decode_window"):
        B, H, L, d = (DECODE[k] for k in ("B", "H", "L", "d"))
        t = fill(synth.decode_specs(B, H, L, d), 1002)
        sl = torch.full((B,), L, dtype=torch.int32, device=dev)
        if name == "decode":
            def f():
                plx.decode(t["q"], t["r"], t["K"], t["V"], sl)
        else:
            def f():
                plx.decode_window(t["q"], t["r"], t["K"], t["V"], sl, WINDOW)
    elif name in ("decode_gqa", "decode_fp8kv"):
        B, H, Hkv, L, d = ((DECODE_GQA[k] for k in ("B", "H", "Hkv", "L", "d")) if name == "decode_gqa"
                           else (DECODE["B"], DECODE["H"], DECODE["H"], DECODE["L"], DECODE["d"]))
        t = fill(synth.decode_gqa_specs(B, H, Hkv, L, d), 1007)
        sl = torch.full((B,), L, dtype=torch.int32, device=dev)
        if name == "decode_gqa":
            def f():
                plx.decode_gqa(t["q"], t["r"], t["K"], t["V"], sl)
        else:
            Kc, Ks = plx.kv_quantize_fp8(t.pop("K"))
            Vc, Vs = plx.kv_quantize_fp8(t.pop("V"))

            def f():
                plx.decode_fp8kv(t["q"], t["r"], Kc, Ks, Vc, Vs, sl)
    else:
        B, H, N, d = (PREFILL[k] for k in ("B", "H", "N", "d"))
        t = fill(synth.backward_specs(B, H, N, d), 1004)
        if name == "prefill":
            def f():
                plx.prefill(t["Q"], t["K"], t["V"], t["R"], causal=True)
        elif name == "prefill_window":
            def f():
                plx.prefill_window(t["Q"], t["K"], t["V"], t["R"], WINDOW)
        else:
            saved = plx.prefill_train(t["Q"], t["K"], t["V"], t["R"], True)

            def f():
                plx.prefill_backward(t["Q"], t["K"], t["V"], t["R"], *saved, t["dO"], True)
    for _ in range(launches):
        f()
    torch.cuda.synchronize()
    status = plx.get_device_status()
    if status != 0:
        raise RuntimeError(f"{name} reported {plx.status_string(status)}")
    print(json.dumps({"only": name, "launches": launches, "status": "ok"}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--sweep", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-gqa", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-window", action="store_true")
    ap.add_argument("--no-layer", action="store_true")
    ap.add_argument("--no-fp8kv", action="store_true")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--only", choices=ONLY, default=None,
                    help="run one workload a few times and exit (for profiler captures)")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work per leg")
    ap.add_argument("--decode-batch", type=int, default=DECODE["B"],
                    help="decode batch (smaller values for profiler captures only)")
    ap.add_argument("--prefill-batch", type=int, default=PREFILL["B"],
                    help="prefill batch (smaller values for profiler captures only)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = {"workload": f"decode B={args.decode_batch} H=16 L=4096 d=128 bf16, all seqlens 4096",
           "global_batch": args.decode_batch * world, "seq_len": DECODE["L"],
           "parallelism": f"replicas{world}" if world > 1 else "single",
           "l2": f"inputs larger than L2 ({args.decode_batch * 16 * 4096 * 128 * 4 / 1e9:.2f} GB KV "
                 "per GPU); no flush"}

    if args.impl == "reference":
        if rank != 0:
            return
        threads = oracle_threads()
        per_step = []
        for s in range(args.warmup + args.steps):
            gbps, units, secs = oracle_decode_sample(min(args.cpu_budget, 1.0))
            if s >= args.warmup:
                per_step.append((gbps, units, secs))
        value = float(np.mean([p[0] for p in per_step]))
        line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(1e3 * float(np.mean([p[2] for p in per_step])), 2),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": cfg,
                "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                                 "sample": f"{int(np.mean([p[1] for p in per_step]))} whole (b,h) units of "
                                           "4096 keys per step (a pool of 4), float64 oracle"},
                "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    else:
        torch.cuda.set_device(0)

    if args.only is not None:
        if rank == 0:
            run_only(args.only)
        if dist is not None:
            dist.destroy_process_group()
        return

    if args.sweep:
        if rank == 0:
            run_sweep(args)
        if dist is not None:
            dist.destroy_process_group()
        return

    res = run_gpu(args, rank, world, dist)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    cpu = None
    if world == 1:
        gbps, units, secs = oracle_decode_sample(args.cpu_budget)
        cpu = {"value": round(gbps, 4), "unit": "GB/s", "cores": oracle_threads(), "kind": "oracle",
               "sample": f"{units} passes over 4 whole (b,h) decode units of 4096 keys "
                         f"({secs:.1f} s of oracle time), float64"}
        if res["prefill"] is not None:
            tf, rows, psecs = oracle_prefill_sample(args.cpu_budget / 2)
            res["prefill"]["cpu_baseline"] = {
                "value": round(tf, 6), "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
                "sample": f"{rows} passes over 8 random causal rows ({psecs:.1f} s), float64"}
    line = {"metric": METRIC, "value": res["value"], "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": cfg, "roofline": res["roofline"], "cpu_baseline": cpu,
            "e2e": res["e2e"], "gpu_launches": res["gpu_launches"], "clocks": res["clocks"],
            "prefill": res["prefill"], "layer": res["layer"], "decode_gqa": res["decode_gqa"],
            "window": res["window"], "decode_fp8kv": res["decode_fp8kv"], "decode_sweep": res["decode_sweep"]}
    print(json.dumps(line))


if __name__ == "__main__":
    main()
