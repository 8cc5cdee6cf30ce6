"""Benchmark of the activation-sparse gated FFN (TwELL) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload ffn_2b] [--impl ours|reference]

One step = one pass of the inference hot path over one synthetic batch:
twell_gate_gemm (tcgen05 gate GEMM + TwELL epilogue) then twell_fused_updown
(gather up/down over the active units).  Inputs are resident in HBM; x,
Wg, Wu, Wd total 160 MB at the 2B shape, more than the 126 MB L2, so no flush
is done between steps.  Rank 0 prints ONE JSON line.  Under torchrun every
rank runs an independent replica on its own GPU (weak scaling: no data-path
collective; only the timing is max-reduced).

--impl reference times the CPU oracle (single-threaded fp64 C) on a bounded
token sample per step, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from activation_sparse_transformer_tma_b200 import synth  # noqa: E402

METRIC = "FFN tokens/sec on 1 B200 (2B-shaped, ~99% sparse) + % HBM/tensor roofline"
UNIT = "tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="ffn_2b")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extras", action="store_true", help="skip comparator/training/decode legs")
    ap.add_argument("--legs", default="dense,tiles,energy,decode,training",
                    help="comma-separated extra legs to run after the timed step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p["bf16_tflops_sustained"], "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local_rank):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        self.gpu = vis.split(",")[local_rank] if vis else str(local_rank)
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------- reference --
def run_reference(args, rank):
    """CPU oracle arm: a bounded token sample per step, rank 0 only."""
    if rank != 0:
        return
    import oracle
    w = synth.make_workload(args.workload)
    dt = w["dtype"]
    x = synth.widen(w["x"], dt)
    Wg, Wu, Wd = (synth.widen(w[k], dt) for k in ("Wg_t", "Wu_t", "Wd"))

    def one(rows):
        g = oracle.gate_rows(x, Wg, rows, g_round=dt)
        enc = oracle.twell_encode(g, w["W"], w["C"])
        return oracle.twell_ffn(x[rows], enc, Wu, Wd)

    t0 = time.perf_counter()
    one(synth.subsample_rows(w["T"], 2, seed=99))
    per_tok = (time.perf_counter() - t0) / 2
    total_steps = args.steps + args.warmup
    n = int(max(1, min(256, 150.0 / max(total_steps, 1) / per_tok)))
    for s in range(args.warmup):
        one(synth.subsample_rows(w["T"], n, seed=1000 + s))
    t0 = time.perf_counter()
    for s in range(args.steps):
        one(synth.subsample_rows(w["T"], n, seed=2000 + s))
    el = time.perf_counter() - t0
    v = n * args.steps / el
    sample = (f"{n} seeded tokens of {args.workload} per step (gate + TwELL encode + sparse "
              f"FFN, fp64), 1 thread of {os.cpu_count()} host cores")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, args),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(w, args):
    return {"workload": w["name"], "T": w["T"], "d": w["d"], "F": w["F"], "W": w["W"],
            "C": w["C"], "dtype": w["dtype"], "global_batch_tokens": w["T"] * args.gpus,
            "parallelism": f"replicas{args.gpus}", "seed": 0,
            "l2": "inputs (x, Wg, Wu, Wd) exceed the 126 MB L2; no flush between steps"}


# --------------------------------------------------------------------- ours --
def src_sha(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "activation_sparse_transformer_tma_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(profile_md, sha):
    """DRAM bytes per launch from a committed ncu summary, if it matches the source."""
    try:
        text = open(os.path.join(ROOT, "profiles", profile_md)).read()
    except OSError:
        return None
    m_sha = re.search(r"source_sha256_16:\s*([0-9a-f]+)", text)
    m_b = re.search(r"dram_bytes_per_launch_full_size:\s*([0-9.eE+]+)", text)
    if not (m_sha and m_b) or m_sha.group(1) != sha:
        return None
    return float(m_b.group(1))


def run_ours(args, rank, world, local_rank):
    import torch
    from activation_sparse_transformer_tma_b200 import twell as tw

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))

    w = synth.make_workload(args.workload)
    T, d, F, C = w["T"], w["d"], w["F"], w["C"]
    dt = torch.bfloat16 if w["dtype"] == synth.BF16 else torch.float32

    def dev(a):
        if w["dtype"] == synth.BF16:
            return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
        return torch.from_numpy(a).cuda()

    x, Wg, Wu, Wd = (dev(w[k]) for k in ("x", "Wg_t", "Wu_t", "Wd"))
    g = tw.Twell(T, F, C, dtype=dt, spill_cap=max(4096, (F // 128) * T // 8))
    # y is accumulated and stored in fp32 (the residual-stream precision)
    y = torch.empty((T, d), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = tw.fused_workspace(T, d)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        tw.twell_gate_gemm(x, Wg, g, None, status)
        if ev is not None:
            ev[1].record(stream)
        tw.twell_fused_updown(x, g, Wu, Wd, y, ws, status)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for k in range(K):
        step(evs[k])
    t_end.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    ms_total = t_start.elapsed_time(t_end)
    ms_gate = sum(e[0].elapsed_time(e[1]) for e in evs) / K
    ms_fused = sum(e[1].elapsed_time(e[2]) for e in evs) / K
    st = int(status.item())
    if dist:
        tt = torch.tensor([ms_total], device="cuda")
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms_total = float(tt.item())
    ms_step = ms_total / K
    value = world * T * K / (ms_total / 1e3)

    # ------------------------------------------------------------- e2e leg --
    # Through the public API with host buffers: every step copies its x from
    # pinned host memory and reads its y back.  Steps are pipelined over three
    # streams with double-buffered device x and y, so the copy-in of step k+1
    # and the copy-out of step k-1 overlap the kernels of step k.
    xh = torch.empty((T, d), dtype=dt, pin_memory=True)
    xh.copy_(x.cpu())
    E = max(3, min(K, 30))

    def e2e_rate(y_dtype):
        yh = torch.empty((T, d), dtype=y_dtype, pin_memory=True)
        s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        xd = [torch.empty_like(x) for _ in range(2)]
        yd = [torch.empty((T, d), dtype=y_dtype, device="cuda") for _ in range(2)]
        ev = {n: [torch.cuda.Event() for _ in range(2)]
              for n in ("x_ready", "x_free", "y_ready", "y_free")}
        for b in range(2):  # every buffer starts free
            ev["x_free"][b].record(s_cmp)
            ev["y_free"][b].record(s_out)

        def e2e_step(k):
            b = k & 1
            s_in.wait_event(ev["x_free"][b])
            with torch.cuda.stream(s_in):
                xd[b].copy_(xh, non_blocking=True)
            ev["x_ready"][b].record(s_in)
            s_cmp.wait_event(ev["x_ready"][b])
            s_cmp.wait_event(ev["y_free"][b])
            tw.twell_gate_gemm(xd[b], Wg, g, None, status, stream=s_cmp)
            tw.twell_fused_updown(xd[b], g, Wu, Wd, yd[b], ws, status, stream=s_cmp)
            ev["x_free"][b].record(s_cmp)
            ev["y_ready"][b].record(s_cmp)
            s_out.wait_event(ev["y_ready"][b])
            with torch.cuda.stream(s_out):
                yh.copy_(yd[b], non_blocking=True)
            ev["y_free"][b].record(s_out)

        for k in range(3):
            e2e_step(k)
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        s_cmp.wait_event(e0)
        s_out.wait_event(e0)
        for k in range(E):
            e2e_step(k)
        e1.record(s_out)
        torch.cuda.synchronize()
        ms_e2e = e0.elapsed_time(e1)
        if dist:
            tt = torch.tensor([ms_e2e], device="cuda")
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            ms_e2e = float(tt.item())
        return {"value": world * T * E / (ms_e2e / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": xh.numel() * xh.element_size(),
                "d2h_bytes_per_step": yh.numel() * yh.element_size(),
                "pipeline": "3 streams (copy-in, kernels, copy-out), double-buffered x and y"}

    # y in fp32, the accumulator's precision (the headline); then the same
    # path writing y rounded once to bf16, which halves the read-back that
    # bounds this pipeline
    e2e = e2e_rate(torch.float32)
    e2e_bf16 = e2e_rate(torch.bfloat16)
    e2e_bf16["what"] = "as e2e, with y returned in bf16 (the fp32 sums rounded once)"

    hbm, tf_burst, tf_sust, src = peaks()
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    fp32_peak = n_sm * 128 * 2 * sm_max_mhz() * 1e6 / 1e12  # TFLOP/s, FMA = 2 FLOP
    flops_gate = 2.0 * T * d * F
    tflops_gate = flops_gate / (ms_gate * 1e-3) / 1e12
    nnz = int(g.cnt.to(torch.int64).sum().item())
    flops_fused = 2.0 * 2 * d * nnz          # one dot and one axpy of length d per entry
    tflops_fused = flops_fused / (ms_fused * 1e-3) / 1e12
    Kt = F // 128
    live = live_units(torch, g)
    # x, fp32 y, TwELL, and one Wu and one Wd row of every unit active in the batch
    unique_bytes = 2 * T * d + 4 * T * d + Kt * T * (3 * C + 1) + live * 2 * d * 2
    roof_gate = {"kernel": "twell_gate_gemm (tcgen05 + TwELL epilogue)", "bound": "tensor",
                 "achieved": tflops_gate, "peak": tf_burst, "unit": "TFLOP/s",
                 "frac": tflops_gate / tf_burst,
                 "peak_source": f"{src} bf16 burst (the timed region is well under a second)",
                 "frac_of_sustained_peak": tflops_gate / tf_sust,
                 "traffic": profiled_traffic("gate_twell_gemm_ffn_2b.md",
                                             src_sha("gemm_tc.cu", "pdl.cuh", "tw_common.cuh")),
                 "algorithmic": f"2*T*d*F = {flops_gate:.4g} FLOP per launch"}
    roof_fused = {"kernel": "twell_fused_updown (gather dot + axpy on CUDA cores)", "bound": "alu",
                  "achieved": tflops_fused, "peak": fp32_peak, "unit": "TFLOP/s",
                  "frac": tflops_fused / fp32_peak,
                  "peak_source": f"derived: {n_sm} SMs x 128 fp32 FMA lanes x 2 x {sm_max_mhz():.0f} MHz",
                  "traffic": profiled_traffic("fused_updown_ffn_2b.md",
                                              src_sha("fused_updown.cu", "pdl.cuh", "tw_common.cuh")),
                  "algorithmic": f"4*d*nnz = {flops_fused:.4g} FLOP per launch (nnz = {nnz})",
                  "gathered_GBps": nnz * 4 * d / (ms_fused * 1e-3) / 1e9,
                  "unique_hbm_bytes": unique_bytes, "live_units": live,
                  "unique_hbm_GBps": unique_bytes / (ms_fused * 1e-3) / 1e9,
                  "unique_hbm_frac": unique_bytes / (ms_fused * 1e-3) / 1e9 / hbm}
    # The three bounds of the fused kernel (unique HBM bytes, fp32 FMA, gathered
    # rows through L2), the last against a live measurement of scattered
    # whole-row gathers from an L2-resident 33.5 MB matrix (tw_measure_row_gather).
    l2_rate = row_gather_rate(torch, tw, Wu if dt == torch.bfloat16 else None)
    gathered = nnz * 4 * d * (2 if dt == torch.bfloat16 else 4) // 2
    bounds_us = {"hbm_unique": unique_bytes / (hbm * 1e9) * 1e6,
                 "fp32_fma": flops_fused / (fp32_peak * 1e12) * 1e6}
    if l2_rate:
        bounds_us["l2_gather"] = gathered / l2_rate * 1e6
        roof_fused["l2_gather"] = {
            "what": "scattered whole-row 16-byte gathers of an L2-resident 33.5 MB bf16 matrix, "
                    "16 warps per SM, measured in this run",
            "peak_GBps": l2_rate / 1e9, "gathered_bytes": gathered,
            "bound_us": bounds_us["l2_gather"],
            "frac": bounds_us["l2_gather"] / (ms_fused * 1e3)}
    binding = max(bounds_us, key=bounds_us.get)
    roof_fused["bounds_us"] = bounds_us
    roof_fused["binding_bound"] = binding
    roof_fused["frac_of_binding_bound"] = bounds_us[binding] / (ms_fused * 1e3)
    dominant = roof_fused if ms_fused >= ms_gate else roof_gate
    kernels = {"gate_twell_gemm": {"ms": ms_gate, **roof_gate},
               "fused_updown": {"ms": ms_fused, "nnz_per_token": nnz / T, **roof_fused},
               "spills_per_step": int(g.spill_n.item())}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if dt == torch.bfloat16 else "f32",
            "data": "synthetic (seeded generator: Zipf(1.1) units, lognormal token skew, "
                    "mean 29 active units per token)",
            "config": config_of(w, args), "roofline": dominant, "e2e": e2e,
            "e2e_bf16_y": e2e_bf16,
            "gpu_launches": KERNELS_PER_STEP * K, "clocks": clk, "kernels": kernels,
            "device_status": st}

    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_leg(w, y)
    legs = set() if args.no_extras else {s.strip() for s in args.legs.split(",") if s.strip()}
    if legs:
        if rank == 0 and "dense" in legs:
            line["dense_comparator"] = dense_leg(torch, tw, x, Wg, Wu, Wd, T, d, F, ms_step, args)
        if rank == 0 and "tiles" in legs:
            line["tile_sweep"] = tile_sweep_leg(torch, tw, x, Wg, Wu, Wd, T, d, F)
        if rank == 0 and "energy" in legs:
            line["energy"] = energy_leg(torch, tw, x, Wg, Wu, Wd, g, y, ws, status, T, d, F,
                                        local_rank)
        del x, Wg, Wu, Wd, g, y, ws, xh
        torch.cuda.empty_cache()
        if rank == 0 and "decode" in legs:
            line["decode"] = decode_leg(torch, tw, hbm)
        if "training" in legs:  # every rank: data-parallel, one gradient all-reduce per step
            tr = training_leg(torch, tw, dist, world)
            if rank == 0:
                line["training"] = tr
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# kernels of one inference step: gate GEMM; plan count, plan scan, plan write,
# fused kernel (the two workspace clears are memsets, not kernels)
KERNELS_PER_STEP = 5


def live_units(torch, g):
    """Number of units active anywhere in the batch, read from the TwELL
    (slots below each tile's count, and the non-zeros of spilled segments)."""
    K = g.F // g.W
    used = torch.zeros(g.F, dtype=torch.bool, device="cuda")
    base = (torch.arange(K, device="cuda") * g.W).view(K, 1, 1)
    if g.C:
        slot = torch.arange(g.C, device="cuda").view(1, 1, g.C)
        valid = slot < g.cnt.long().unsqueeze(2)
        used[(g.idx.long() + base)[valid]] = True
    n = min(int(g.spill_n.item()), g.spill_cap)
    if n:
        tk = g.spill_tk[:n].long()
        nz = g.spill_val[:n] != 0
        cols = torch.arange(g.W, device="cuda").view(1, g.W)
        used[(tk[:, 1:2] * g.W + cols)[nz]] = True
    return int(used.sum().item())


def tile_sweep_leg(torch, tw, x, Wg, Wu, Wd, T, d, F):
    """The same 2B-shaped step with other TwELL tile widths W and capacities C:
    spilled (token, tile) pairs per step and the step time (gate + fused)."""
    out = []
    for W, C in ((128, 4), (128, 8), (128, 16), (128, 32), (64, 8), (256, 16), (256, 32)):
        g = tw.Twell(T, F, C, dtype=torch.bfloat16, spill_cap=(F // W) * T // 4, W=W)
        y = torch.empty((T, d), dtype=torch.float32, device="cuda")
        ws = tw.fused_workspace(T, d)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        for _ in range(3):
            tw.twell_gate_gemm(x, Wg, g, None, st)
            tw.twell_fused_updown(x, g, Wu, Wd, y, ws, st)
        torch.cuda.synchronize()
        # steps queued back to back (no host sync inside), as in the timed loop
        n = 20
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
        for i in range(n):
            ev[i][0].record()
            tw.twell_gate_gemm(x, Wg, g, None, st)
            ev[i][1].record()
            tw.twell_fused_updown(x, g, Wu, Wd, y, ws, st)
            ev[i][2].record()
        torch.cuda.synchronize()
        tg = sum(e[0].elapsed_time(e[1]) for e in ev)
        tf = sum(e[1].elapsed_time(e[2]) for e in ev)
        twell_bytes = (F // W) * T * (3 * C + 1)
        out.append({"W": W, "C": C, "spills_per_step": int(g.spill_n.item()),
                    "gate_ms": tg / n, "fused_ms": tf / n, "step_ms": (tg + tf) / n,
                    "tokens_per_s": T / ((tg + tf) / n * 1e-3), "twell_bytes": twell_bytes,
                    "device_status": int(st.item())})
        del g, y, ws
    torch.cuda.empty_cache()
    return out


def nvml_handle(torch, local_rank):
    """NVML handle of this process's GPU (matched by UUID), or None."""
    try:
        import pynvml
        pynvml.nvmlInit()
        u = str(torch.cuda.get_device_properties(local_rank).uuid)
        for cand in (u, "GPU-" + u):
            try:
                return pynvml.nvmlDeviceGetHandleByUUID(cand)
            except Exception:
                pass
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        idx = int(vis.split(",")[local_rank]) if vis else local_rank
        return pynvml.nvmlDeviceGetHandleByIndex(idx)
    except Exception:
        return None


def energy_leg(torch, tw, x, Wg, Wu, Wd, g, y, ws, status, T, d, F, local_rank):
    """Energy per token of the sparse step and of the in-library dense FFN of
    the same shape.  NVML's cumulative energy counter (read-only, mJ) is read
    around a loop of about two seconds of each; the ratio is dense / sparse."""
    h = nvml_handle(torch, local_rank)
    if h is None:
        return {"unavailable": "NVML energy counter not readable"}
    import pynvml
    Wd_dense = Wd.t().contiguous()
    hbuf = torch.empty((T, F), dtype=torch.bfloat16, device="cuda")
    yd = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")

    def sparse():
        tw.twell_gate_gemm(x, Wg, g, None, status)
        tw.twell_fused_updown(x, g, Wu, Wd, y, ws, status)

    def dense():
        tw.dense_ffn_forward(x, Wg, Wu, Wd_dense, hbuf, yd)

    def measure(fn, seconds=2.0):
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(20):
            fn()
        torch.cuda.synchronize()
        n = max(50, int(seconds / ((time.perf_counter() - t0) / 20)))
        e0 = pynvml.nvmlDeviceGetTotalEnergyConsumption(h)
        t0 = time.perf_counter()
        for _ in range(n):
            fn()
        torch.cuda.synchronize()
        el = time.perf_counter() - t0
        joules = (pynvml.nvmlDeviceGetTotalEnergyConsumption(h) - e0) / 1e3
        return {"steps": n, "seconds": el, "joules": joules, "avg_watts": joules / el,
                "j_per_token": joules / (n * T)}

    sp = measure(sparse)
    dn = measure(dense)
    del hbuf, yd, Wd_dense
    return {"sparse": sp, "dense": dn,
            "dense_over_sparse_j_per_token": dn["j_per_token"] / sp["j_per_token"],
            "method": "NVML total-energy counter around each loop (whole-GPU energy, "
                      "idle power included); wall clock for the loop length"}


def sm_max_mhz():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["sm_max_mhz"])
    except Exception:
        return 1965.0


def decode_leg(torch, tw, hbm):
    """Small batches (T = 1, 8, 16, 64) of the 2B shape with a cold L2: a 512 MB
    buffer is READ between iterations, which leaves L2 full of clean lines of
    that buffer (a write flush would leave ~126 MB of dirty lines whose
    write-back the next kernel would pay for).  Two paths: the gate and fused
    calls (twell_gate_gemm + twell_fused_updown), and the whole FFN in one
    cooperative launch (twell_ffn_small_batch, also timed with a warm L2);
    and the in-library dense FFN of the same tokens for comparison.  The
    sparse step streams Wg (33.5 MB) and gathers one Wu and one Wd row per
    active entry; the dense one streams all three weights (100.7 MB)."""
    flush = torch.ones(128 * 1024 * 1024, dtype=torch.float32, device="cuda")
    sink = torch.empty((), dtype=torch.float32, device="cuda")
    # Between the flush and the start event a one-element kernel runs (L2
    # stays cold), so the flush's own completion is not in the interval.
    # CUDA events still read about 6 us for an empty kernel timed this way;
    # that figure is reported beside the timings.
    tiny = torch.zeros(1, dtype=torch.float32, device="cuda")

    def cold():
        torch.sum(flush, dim=0, out=sink)
        tiny.add_(1.0)

    def cold_us(fn, n=15, skip=5):
        ts = []
        for it in range(n):
            cold()
            e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            e[0].record()
            fn()
            e[1].record()
            torch.cuda.synchronize()
            if it >= skip:
                ts.append(e[0].elapsed_time(e[1]))
        return float(np.median(ts)) * 1e3

    out = {"empty_launch_us": cold_us(lambda: tiny.add_(1.0))}
    # The floor for a launch that streams the gate's weights: one read of a
    # 33.5 MB buffer (the bytes of Wg at the 2B shape) by the library's
    # stream-read aid, timed the same way.
    wg_floor = torch.empty(8192 * 2048, dtype=torch.bfloat16, device="cuda")
    wg_floor.view(torch.int16).random_(-32768, 32767)
    chk = torch.zeros(1, dtype=torch.int32, device="cuda")
    out["stream_read_floor"] = {
        "bytes": wg_floor.numel() * 2,
        "us": cold_us(lambda: tw.measure_stream_read(wg_floor, chk)),
        "what": "tw_measure_stream_read of the Wg bytes, cold L2, one launch"}
    floor_us = out["stream_read_floor"]["us"]
    del wg_floor
    for T in (1, 8, 16, 64):
        w = synth.make_workload("decode_2b", T=T)
        d, F, C = w["d"], w["F"], w["C"]
        dev = {k: torch.from_numpy(w[k].view(np.int16)).cuda().view(torch.bfloat16)
               for k in ("x", "Wg_t", "Wu_t", "Wd")}
        g = tw.Twell(T, F, C, dtype=torch.bfloat16, spill_cap=4096)
        y = torch.empty((T, d), dtype=torch.float32, device="cuda")
        ws = tw.fused_workspace(T, d)
        sws = tw.small_batch_workspace(T, d, F) if T <= 64 else None
        if T == 1:
            Wd_dense = dev["Wd"].t().contiguous()  # the comparator's [d][F] down weight
        hd = torch.empty((T, F), dtype=torch.bfloat16, device="cuda")
        yd = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
        td, tw_warm = [], []
        tg, tf, ts = [], [], []
        for it in range(25):
            cold()
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            e[0].record()
            tw.twell_gate_gemm(dev["x"], dev["Wg_t"], g)
            e[1].record()
            tw.twell_fused_updown(dev["x"], g, dev["Wu_t"], dev["Wd"], y, ws)
            e[2].record()
            if sws is not None:
                cold()
                e1 = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                e1[0].record()
                tw.twell_ffn_small_batch(dev["x"], dev["Wg_t"], dev["Wu_t"], dev["Wd"], g, y, sws)
                e1[1].record()
            # the in-library dense bf16 FFN of the same tokens (streams Wg, Wu, Wd)
            cold()
            e2 = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            e2[0].record()
            tw.dense_ffn_forward(dev["x"], dev["Wg_t"], dev["Wu_t"], Wd_dense, hd, yd)
            e2[1].record()
            torch.cuda.synchronize()
            if it >= 5:
                tg.append(e[0].elapsed_time(e[1]))
                tf.append(e[1].elapsed_time(e[2]))
                if sws is not None:
                    ts.append(e1[0].elapsed_time(e1[1]))
                td.append(e2[0].elapsed_time(e2[1]))
        if sws is not None:  # warm L2: the same launch back to back
            for it in range(25):
                # a 50 us device-side wait queued first, so that the start
                # event and the launch are both queued before the GPU gets
                # to them (no host latency in the interval); it touches no
                # memory, so L2 stays warm
                torch.cuda._sleep(100000)
                e3 = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                e3[0].record()
                tw.twell_ffn_small_batch(dev["x"], dev["Wg_t"], dev["Wu_t"], dev["Wd"], g, y, sws)
                e3[1].record()
                torch.cuda.synchronize()
                if it >= 5:
                    tw_warm.append(e3[0].elapsed_time(e3[1]))
        nnz = int(g.cnt.to(torch.int64).sum().item())
        mg, mf = float(np.median(tg)), float(np.median(tf))
        wg_bytes = F * d * 2
        gate_gbs = wg_bytes / (mg * 1e-3) / 1e9
        rows = nnz * 2 * d * 2  # Wu and Wd rows gathered (an upper bound on unique bytes)
        r = {"l2": "cold (512 MB read, then a one-element kernel, between iterations)", "nnz": nnz,
             "two_calls": {"gate_us": mg * 1e3, "fused_us": mf * 1e3,
                           "tokens_per_s": T / ((mg + mf) * 1e-3),
                           "gate_hbm_GBps": gate_gbs, "gate_hbm_frac": gate_gbs / hbm,
                           "gate_frac_of_stream_floor": floor_us / (mg * 1e3),
                           "fused_gathered_GBps": rows / (mf * 1e-3) / 1e9,
                           "library_launches": 2 if T <= 8 else 5}}
        if ts:
            ms = float(np.median(ts))
            step_gbs = (wg_bytes + rows) / (ms * 1e-3) / 1e9
            r["single_launch"] = {"step_us": ms * 1e3, "tokens_per_s": T / (ms * 1e-3),
                                  "bytes": wg_bytes + rows, "hbm_GBps": step_gbs,
                                  "hbm_frac": step_gbs / hbm,
                                  "frac_of_stream_floor": floor_us / (ms * 1e3),
                                  "library_launches": 1,
                                  "speedup_vs_two_calls": (mg + mf) / ms,
                                  "warm_l2_step_us": float(np.median(tw_warm)) * 1e3}
        md = float(np.median(td))
        dense_bytes = 3 * F * d * 2
        r["dense_comparator"] = {
            "what": "dense_ffn_forward (tcgen05 GEMMs, bf16 h and y), cold L2",
            "step_us": md * 1e3, "streamed_bytes": dense_bytes,
            "hbm_GBps": dense_bytes / (md * 1e-3) / 1e9,
            "sparse_speedup": md / (float(np.median(ts)) if ts else (mg + mf))}
        out[f"T{T}"] = r
        del hd, yd
    del flush, Wd_dense
    return out


def training_leg(torch, tw, dist=None, world=1):
    """One training step of the hybrid path at the train_2b shape per GPU: gate
    GEMM -> TwELL -> hybrid, hybrid forward, hybrid backward (with the L1
    term); on N GPUs each rank takes its own train_2b batch (weak scaling)
    and the weight gradients are summed with one all-reduce (NCCL)."""
    from activation_sparse_transformer_tma_b200 import dp

    w = synth.make_workload("train_2b")
    T, d, F, C, C_h = w["T"], w["d"], w["F"], w["C"], w["C_h"]
    dev = {k: torch.from_numpy(w[k].view(np.int16)).cuda().view(torch.bfloat16)
           for k in ("x", "Wg_t", "Wu_t", "Wd", "dy")}
    cap = T // 4
    g = tw.Twell(T, F, C, dtype=torch.bfloat16, spill_cap=(F // 128) * T // 8)
    hy = tw.Hybrid(T, F, C_h, dtype=torch.bfloat16, backup_cap=cap)
    y = torch.empty((T, d), dtype=torch.float32, device="cuda")
    dx = torch.empty((T, d), dtype=torch.float32, device="cuda")
    grads = dp.GradBuffer(F, d, "cuda")
    ws = torch.empty(tw.hybrid_ffn_backward_workspace_size(T, d, F, C_h, cap), dtype=torch.uint8,
                     device="cuda")
    fws = torch.empty(tw.hybrid_ffn_forward_workspace_size(T, d), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    names = ["gate_twell_gemm", "twell_to_hybrid", "hybrid_ffn_forward", "hybrid_ffn_backward"]
    if world > 1:
        names.append("grad_allreduce")
    times = {n: [] for n in names}
    for it in range(8):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
        e[0].record()
        tw.twell_gate_gemm(dev["x"], dev["Wg_t"], g, None, st)
        e[1].record()
        tw.twell_to_hybrid(g, hy, st)
        e[2].record()
        tw.hybrid_ffn_forward(dev["x"], hy, dev["Wu_t"], dev["Wd"], y, fws, st)
        e[3].record()
        tw.hybrid_ffn_backward(dev["x"], dev["dy"], hy, dev["Wg_t"], dev["Wu_t"], dev["Wd"],
                               w["lam"], dx, grads.dWg_t, grads.dWu_t, grads.dWd, ws, st)
        e[4].record()
        if world > 1:
            grads.allreduce()
            e[5].record()
        torch.cuda.synchronize()
        if it >= 3:
            for i, n in enumerate(names):
                times[n].append(e[i].elapsed_time(e[i + 1]))
    ms = {n: float(np.median(v)) for n, v in times.items()}
    phases_sum = sum(ms.values())

    # The step itself: whole steps back to back between two events, as the
    # inference step is timed (the phase times above carry an event and, for
    # the first phase, the host's launch latency at each boundary).
    def sparse_step():
        tw.twell_gate_gemm(dev["x"], dev["Wg_t"], g, None, st)
        tw.twell_to_hybrid(g, hy, st)
        tw.hybrid_ffn_forward(dev["x"], hy, dev["Wu_t"], dev["Wd"], y, fws, st)
        tw.hybrid_ffn_backward(dev["x"], dev["dy"], hy, dev["Wg_t"], dev["Wu_t"], dev["Wd"],
                               w["lam"], dx, grads.dWg_t, grads.dWu_t, grads.dWd, ws, st)
        if world > 1:
            grads.allreduce()

    step = back_to_back_ms(torch, sparse_step)
    n_backup = int(hy.n_backup.item())
    st_sparse = int(st.item())
    # bytes of the hybrid step: activations kept from the forward for the
    # backward (the hybrid g and u with indices and row metadata), and the
    # calls' transient workspaces; exact from the tensors and size queries
    esz = 2
    ell = T * C_h * (esz + esz + 2) + 2 * 4 * T
    saved_alloc = ell + cap * (4 + 2 * F * esz) + 4
    saved_fit = ell + n_backup * (4 + 2 * F * esz) + 4
    twell_bytes = sum(t.numel() * t.element_size() for t in (g.val, g.idx, g.cnt, g.spill_ref,
                                                              g.spill_tk, g.spill_val, g.spill_n))
    sparse_ws = fws.numel() + ws.numel()
    # the backward workspace bounds every backup row by F records; a caller
    # that sizes its backup capacity to the rows it uses needs this much
    sparse_ws_fit = fws.numel() + tw.hybrid_ffn_backward_workspace_size(T, d, F, C_h, n_backup)
    del g, hy, fws, ws
    torch.cuda.empty_cache()

    # the in-library dense bf16 training FFN of the same shape: forward
    # (saves g, u, h) and backward (dx, dWg, dWu, dWd), tcgen05 GEMMs
    dws = tw.dense_train_workspace(T, F)
    dst = torch.zeros(1, dtype=torch.int32, device="cuda")
    dn = {"dense_forward": [], "dense_backward": []}
    for it in range(8):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record()
        tw.dense_ffn_train_forward(dev["x"], dev["Wg_t"], dev["Wu_t"], dev["Wd"], dws, y, dst)
        e[1].record()
        tw.dense_ffn_train_backward(dev["x"], dev["dy"], dev["Wg_t"], dev["Wu_t"], dev["Wd"],
                                    w["lam"], dws, dx, grads.dWg_t, grads.dWu_t, grads.dWd, dst)
        e[2].record()
        torch.cuda.synchronize()
        if it >= 3:
            dn["dense_forward"].append(e[0].elapsed_time(e[1]))
            dn["dense_backward"].append(e[1].elapsed_time(e[2]))
    dms = {n: float(np.median(v)) for n, v in dn.items()}

    def dense_step_fn():
        tw.dense_ffn_train_forward(dev["x"], dev["Wg_t"], dev["Wu_t"], dev["Wd"], dws, y, dst)
        tw.dense_ffn_train_backward(dev["x"], dev["dy"], dev["Wg_t"], dev["Wu_t"], dev["Wd"],
                                    w["lam"], dws, dx, grads.dWg_t, grads.dWu_t, grads.dWd, dst)

    dense_step = back_to_back_ms(torch, dense_step_fn)
    dense_saved = tw.dense_ffn_train_saved_bytes(T, F)
    dense_ws = tw.dense_ffn_train_workspace_size(T, F)
    del dws
    if world > 1:  # the slowest rank sets the step time
        tt = torch.tensor([step], device="cuda")
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        step = float(tt.item())
    out = {"workload": "train_2b", "T": T, "d": d, "F": F, "C": C, "C_h": C_h,
           "ms": ms, "ms_per_step": step, "tokens_per_s": world * T / (step * 1e-3),
           "timing": "ms_per_step: 10 whole steps back to back between two CUDA events, median "
                     "of 3 such runs; ms: each phase between events, median of 5 steps",
           "phases_sum_ms": phases_sum,
           "n_backup": n_backup, "backup_cap": cap, "device_status": st_sparse,
           "dense": {"ms": dms, "ms_per_step": dense_step, "phases_sum_ms": sum(dms.values()),
                     "tokens_per_s": T / (dense_step * 1e-3),
                     "flops_per_step": 9 * 2.0 * T * d * F,
                     "tflops": 9 * 2.0 * T * d * F / (dense_step * 1e-3) / 1e12,
                     "device_status": int(dst.item())},
           "sparse_speedup_vs_dense": dense_step / step,
           "sparse_speedup_vs_dense_phases": sum(dms.values()) / phases_sum,
           "memory_bytes": {
               "what": "FFN-layer activation bytes per GPU, excluding x, dy, the weights and "
                       "their gradients (the same for both paths)",
               "sparse_saved_fwd_to_bwd": saved_alloc,
               "sparse_saved_fwd_to_bwd_exact_fit": saved_fit,
               "sparse_twell_transient": twell_bytes,
               "sparse_workspaces": sparse_ws,
               "sparse_peak": saved_alloc + max(twell_bytes, sparse_ws),
               "sparse_workspaces_exact_fit": sparse_ws_fit,
               "sparse_peak_exact_fit": saved_fit + max(twell_bytes, sparse_ws_fit),
               "dense_saved_fwd_to_bwd": dense_saved,
               "dense_workspace": dense_ws,
               "dense_peak": dense_ws,
               "peak_ratio_sparse_over_dense": (saved_alloc + max(twell_bytes, sparse_ws))
                                               / dense_ws,
               "peak_ratio_exact_fit": (saved_fit + max(twell_bytes, sparse_ws_fit))
                                       / dense_ws}}
    if world > 1:
        out["parallelism"] = f"dp{world}: one fp32 all-reduce of dWg, dWu, dWd ({3 * F * d * 4} B)"
    return out


def back_to_back_ms(torch, fn, steps=10, runs=3):
    """Milliseconds per call of fn, from `steps` calls back to back between two
    CUDA events on the current stream (a device-side wait queued first, so the
    host's launch latency is not in the interval); median of `runs`."""
    for _ in range(2):
        fn()
    torch.cuda.synchronize()
    res = []
    for _ in range(runs):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        torch.cuda._sleep(200000)
        e[0].record()
        for _ in range(steps):
            fn()
        e[1].record()
        torch.cuda.synchronize()
        res.append(e[0].elapsed_time(e[1]) / steps)
    return float(np.median(res))


def row_gather_rate(torch, tw, mat):
    """Bytes per second of scattered whole-row gathers from `mat` (bf16,
    L2-resident after the first pass), or None for other dtypes."""
    if mat is None:
        return None
    chk = torch.zeros(1, dtype=torch.int32, device="cuda")
    rows, d = mat.shape
    n = 1 << 20  # 1 Mi rows
    ts = []
    for it in range(6):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        tw.measure_row_gather(mat, n, it + 1, chk)
        b.record()
        torch.cuda.synchronize()
        if it >= 1:
            ts.append(a.elapsed_time(b))
    return n * d * 2 / (float(np.median(ts)) * 1e-3)


def dense_leg(torch, tw, x, Wg, Wu, Wd, T, d, F, ms_sparse, args):
    """The in-library dense bf16 FFN of the same shape (tcgen05, no cuBLAS)."""
    Wd_dense = Wd.t().contiguous()
    h = torch.empty((T, F), dtype=torch.bfloat16, device="cuda")
    yd = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        tw.dense_ffn_forward(x, Wg, Wu, Wd_dense, h, yd)
    torch.cuda.synchronize()
    n = max(5, min(args.steps, 100))
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(n):
        tw.dense_ffn_forward(x, Wg, Wu, Wd_dense, h, yd)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / n
    flops = 2.0 * T * d * F * 3
    return {"ms_per_step": ms, "tokens_per_s": T / (ms * 1e-3), "tflops": flops / (ms * 1e-3) / 1e12,
            "sparse_speedup": ms / ms_sparse}


def cpu_baseline_leg(w, y_gpu):
    """Oracle timed on a bounded sample (rank 0); also checks the timed y rows."""
    import oracle
    import torch
    rows = synth.subsample_rows(w["T"], 128, seed=5)
    dt = w["dtype"]
    x = synth.widen(w["x"], dt)
    Wg, Wu, Wd = (synth.widen(w[k], dt) for k in ("Wg_t", "Wu_t", "Wd"))
    t0 = time.perf_counter()
    g = oracle.gate_rows(x, Wg, rows, g_round=dt)
    enc = oracle.twell_encode(g, w["W"], w["C"])
    y_ref = oracle.twell_ffn(x[rows], enc, Wu, Wd)
    el = time.perf_counter() - t0
    yg = y_gpu[torch.as_tensor(rows, device=y_gpu.device).long()].float().cpu().numpy()
    err = float(np.max(np.abs(yg - y_ref)) / np.sqrt(np.mean(y_ref ** 2)))
    return {"value": len(rows) / el, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{len(rows)} seeded tokens of {w['name']}: gate + TwELL encode + sparse "
                      f"FFN in fp64, 1 thread of {os.cpu_count()} host cores",
            "parity_max_err_over_rms": err, "parity_tol": 1e-2}


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
