#!/usr/bin/env python
"""Benchmark of the HSA hot path at the Wan-1.3B block shape on B200.

One step = one HSA denoising iteration of a Wan-1.3B-shaped DiT block (bf16,
N = 32760 tokens from a 21x30x52 latent-patch grid, D = 1536, 12 heads, FFN
8960, 512-token text context) with every token active, so every part of the
hot path runs: gather + LayerNorm/modulation, QKV GEMM + q/k RMSNorm + 3D
RoPE + KV-cache scatter, |A| x N attention, O-projection, cross-attention,
FFN, velocity scatter + cached Euler with the fused L1 score, and the
regrouping of the tokens (25/25/50 %).  A sweep times the layer step at
|A|/N = 0.5 and 0.25 (active set: top-M tokens by L1 score of two velocity
draws).  Inputs are seeded synthetic stand-ins (random-init weights).

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Multi-GPU: independent replicas, one per rank (the path has no exchange).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from token_sparse_denoising_b200 import synthetic as S  # noqa: E402

METRIC = "HSA layer-step ms (Wan-1.3B block, |A|/N=1, full iteration)"
GRID = S.WAN13_GRID
SHAPE = S.WAN13_BLOCK
GROUP_FRACS = (0.25, 0.25, 0.5)
DSIGMA = -1.0 / 40.0
SEED = 2
ATTN_SRC = os.path.join(ROOT, "token_sparse_denoising_b200", "csrc", "attn_tc.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_traffic.json")


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=30)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["hsa", "reference"], default="hsa")
    p.add_argument("--no-sweep", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-configs", action="store_true",
                   help="skip the other workloads measured beside the headline (tiny loop, 30-block loop, "
                        "Wan-14B block, attention and Euler sweeps)")
    p.add_argument("--mode", choices=["step", "loop", "sweep", "wan14", "tiny", "headpar", "cross", "gemm"],
                   default="step",
                   help="step: the headline line; loop: 30-block Wan-1.3B loop, HSA vs uniform 40 steps; "
                        "sweep: attention + Euler kernel sweep; wan14: Wan-14B block active-fraction sweep; "
                        "tiny: the fp32 parity workload as a whole run; headpar: one Wan-14B block split by "
                        "heads over the ranks (NCCL between the phases), |A|/N = 1; cross: the "
                        "cross-attention shape alone (32760 queries x 512 context rows); gemm: the block's "
                        "GEMMs alone against cuBLAS")
    return p.parse_args()


def workload_config(frac=1.0):
    return {"workload": f"wan1.3b-block N={GRID.N} ({GRID.frames}x{GRID.height}x{GRID.width}) D={SHAPE.D} "
                        f"H={SHAPE.H} F={SHAPE.F} ctx={SHAPE.ctx_len} |A|/N={frac:g}",
            "tokens": GRID.N, "active_fraction": frac, "groups": list(GROUP_FRACS),
            "l2": "no flush: the step's working set (~1.3 GB) is larger than the 126 MB L2",
            "parallelism": "replicas"}


def synthetic_inputs():
    N, D = GRID.N, SHAPE.D
    return {
        "bw": S.block_weights(SEED, SHAPE, bf16=True),
        "pos": S.token_positions(GRID),
        "x0": S.normal(SEED * 10 + 1, (N, D)),
        "vh0": S.normal(SEED * 10 + 2, (N, D)),
        "ctx": S.normal(SEED * 10 + 3, (SHAPE.ctx_len, D), 1.0, True),
        "kc0": S.normal(SEED * 10 + 4, (N, D), 1.0, True),
        "vc0": S.normal(SEED * 10 + 5, (N, D), 1.0, True),
        "va": S.normal(SEED * 10 + 6, (N, D)),
        "vb": S.normal(SEED * 10 + 7, (N, D)),
    }


# ---------------------------------------------------------------- clocks during the timed region

class ClockSampler:
    """SM clock, instantaneous power and clock-event reasons, sampled from before the warm-up:
    NVML read every 10 ms on a host thread (read-only queries), and nvidia-smi every 50 ms beside
    it as a cross-check (alone where NVML cannot be used).  stop() keeps the samples whose
    timestamps fall inside the timed region (host clock window set by mark_start / mark_end)."""

    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, index: int):
        self.t0 = self.t1 = None
        self.rows = []                          # (time, sm MHz, max MHz, power W, [reasons])
        self.proc = self.thread = None
        self.stop_flag = False
        try:
            import threading
            import pynvml as N
            import torch
            N.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(index).uuid)
            self.h = N.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
            bits = {"hw_slowdown": N.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": N.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": N.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": N.nvmlClocksEventReasonSwPowerCap}
            max_mhz = float(N.nvmlDeviceGetMaxClockInfo(self.h, N.NVML_CLOCK_SM))

            def poll():
                while not self.stop_flag:
                    r = N.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    pw = N.nvmlDeviceGetFieldValues(self.h, [N.NVML_FI_DEV_POWER_INSTANT])[0]
                    self.rows.append((time.time(), float(N.nvmlDeviceGetClockInfo(self.h, N.NVML_CLOCK_SM)),
                                      max_mhz, pw.value.uiVal / 1000.0 if pw.nvmlReturn == 0 else float("nan"),
                                      [n for n in self.NAMES if r & bits[n]]))
                    time.sleep(0.01)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
        except Exception:
            self.thread = None
        self._start_smi(index)
        self.source = "NVML every 10 ms" if self.thread is not None else "nvidia-smi every 50 ms"
        time.sleep(0.2)                        # sampling runs before the work starts

    def _start_smi(self, index):
        self.path = tempfile.mktemp(suffix=".csv")
        q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw.instant,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def _smi_rows(self):
        import datetime
        if self.proc is None:
            return []
        self.proc.terminate()
        self.proc.wait(timeout=10)
        rows = []
        for line in open(self.path):
            f = [v.strip() for v in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(f[2]), float(f[3]), float(f[4]),
                             [n for n, v in zip(self.NAMES, f[6:10]) if v.lower() == "active"]))
            except ValueError:
                continue
        os.unlink(self.path)
        return rows

    def _select(self, rows):
        window = "timed region"
        sel = [r for r in rows if self.t0 is not None and self.t0 <= r[0] <= self.t1]
        if len(sel) < 2:                        # a very short timed region: add the warm-up just before it
            window = "warm-up and timed region"
            sel = [r for r in rows if self.t0 is not None and self.t0 - 1.0 <= r[0] <= self.t1]
        if not sel:
            window, sel = "whole run", rows
        return window, sel

    def stop(self):
        smi = self._smi_rows()
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=5)
            rows = list(self.rows)
        elif smi:
            rows = smi
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        window, sel = self._select(rows)
        reasons = sorted({n for r in sel for n in r[4]})
        out = {"sm_mhz": statistics.median(r[1] for r in sel) if sel else None,
               "sm_max_mhz": sel[-1][2] if sel else None, "reasons": reasons,
               "power_w_median": round(statistics.median(r[3] for r in sel), 1) if sel else None,
               "samples": len(sel), "window": window, "source": self.source}
        if self.thread is not None and smi:
            w2, s2 = self._select(smi)
            out["nvidia_smi"] = {"sm_mhz": statistics.median(r[1] for r in s2),
                                 "power_w_median": statistics.median(r[3] for r in s2),
                                 "reasons": sorted({n for r in s2 for n in r[4]}), "samples": len(s2),
                                 "window": w2}
        return out


# ---------------------------------------------------------------- the CUDA path

class Step:
    """Device state of the workload and one HSA iteration through the C ABI."""

    def __init__(self, inp, device):
        import torch
        from token_sparse_denoising_b200 import hsa, pipeline
        self.torch, self.hsa = torch, hsa
        N, D = GRID.N, SHAPE.D
        self.N = N
        self.sizes = S.group_sizes(N, GROUP_FRACS)
        self.model = pipeline.SingleBlockModel(inp["bw"], inp["pos"], N, bf16=True, ctx=inp["ctx"],
                                               cache_init=(inp["kc0"], inp["vc0"]), device=device)
        self.x = torch.from_numpy(inp["x0"]).to(device)
        self.vhat = torch.from_numpy(inp["vh0"]).to(device)
        self.score = torch.zeros(N, device=device)
        self.group = torch.zeros(N, dtype=torch.int8, device=device)
        self.order = torch.arange(N, dtype=torch.int32, device=device)
        self.sel_ws = torch.empty(max(hsa.select_tokens_workspace_size(N, len(self.sizes)), 1), dtype=torch.uint8,
                                  device=device)
        # active sets of the sweep: top-M tokens by the L1 score of two velocity draws
        va, vb = torch.from_numpy(inp["va"]).to(device), torch.from_numpy(inp["vb"]).to(device)
        s = torch.empty(N, device=device)
        hsa.l1_score(va, vb, s)
        self.active = {}
        for f in (0.5, 0.25):
            M = S.active_fraction_rows(N, f)
            g = torch.empty(N, dtype=torch.int8, device=device)
            o = torch.empty(N, dtype=torch.int32, device=device)
            hsa.select_tokens(s, [M, N - M], g, o)
            self.active[f] = o[:M].clone()
        del va, vb
        torch.cuda.synchronize()

    def full(self):
        """One iteration with every token active (all rows of the hot path)."""
        hsa = self.hsa
        idx = self.order
        vA = self.model.velocity(self.x, idx)
        hsa.euler_update(self.x, self.vhat, vA, idx, DSIGMA, score=self.score)
        hsa.select_tokens(self.score, self.sizes, self.group, self.order, ws=self.sel_ws)

    def partial(self, f):
        """One iteration of the cached window: the layer step on the top-M set, then cached Euler."""
        hsa = self.hsa
        idx = self.active[f]
        vA = self.model.velocity(self.x, idx)
        hsa.euler_update(self.x, self.vhat, vA, idx, DSIGMA)


def time_device(fn, steps, barrier):
    import torch
    st = torch.cuda.current_stream()
    barrier()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    for _ in range(steps):
        fn()
    b.record(st)
    b.synchronize()
    torch.cuda.synchronize()
    barrier()
    return a.elapsed_time(b)


def time_e2e(step, x_host_np, n, barrier):
    """ms for n iterations through the C ABI's host-buffer entry point (hsa_iteration_host): every
    iteration uploads its latent from pinned host memory, runs the full iteration (layer step on
    every token, cached Euler with the fused score, regrouping) and downloads the updated latent.
    Two device slots alternate, so the library overlaps iteration k+1's upload (H2D stream) and
    iteration k's download (D2H stream) with compute; every copy is inside the timed region."""
    import torch
    hsa = step.hsa
    N, D = step.N, SHAPE.D
    hx = torch.from_numpy(x_host_np).pin_memory()
    hout = [torch.empty_like(hx).pin_memory() for _ in range(2)]
    slots = [hsa.HostSlot(N, D), hsa.HostSlot(N, D)]
    comp = torch.cuda.current_stream()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    m = step.model

    def run(count):
        for k in range(count):
            hsa.iteration_host(m.w, m.kc, m.vc, step.order, m.pos, m.xA, step.vhat, DSIGMA, hx, hout[k % 2],
                               slots[k % 2], m.ws, ctx_k=m.ctx_k, ctx_v=m.ctx_v, score=step.score,
                               group_sizes=step.sizes, group=step.group, order=step.order, sel_ws=step.sel_ws,
                               stream=comp, stream_h2d=h2d, stream_d2h=d2h)

    run(2)                                                  # warm-up
    torch.cuda.synchronize()
    barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(h2d)
    run(n)
    d2h.wait_stream(comp)
    d2h.wait_stream(h2d)
    end.record(d2h)
    end.synchronize()
    torch.cuda.synchronize()
    barrier()
    return start.elapsed_time(end)


def attn_flops_per_full_step():
    M = L = GRID.N
    return 4.0 * M * L * 128 * SHAPE.H + 4.0 * M * SHAPE.ctx_len * 128 * SHAPE.H


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("bf16_tflops_sustained") or d["bf16_tflops"], d["bf16_tflops"], d["hbm_gbs"], "measured"
    return 1400.0, 1590.0, 6650.0, "fallback"


def traffic_per_launch():
    """DRAM bytes of one attention launch from the committed ncu summary, if it is of this source."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    d = json.load(open(TRAFFIC_FILE))
    sha = hashlib.sha256(open(ATTN_SRC, "rb").read()).hexdigest()
    if d.get("source_sha256") != sha:
        return None
    return d.get("dram_bytes_per_launch")


def run_gpu(args, rank, world, barrier, allmax):
    import torch
    from token_sparse_denoising_b200 import hsa
    hsa.load()
    device = torch.device("cuda", torch.cuda.current_device())
    inp = synthetic_inputs()
    step = Step(inp, device)
    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    for _ in range(args.warmup):
        step.full()
    torch.cuda.synchronize()
    assert hsa.device_status() == 0, "device status after warm-up"

    # ---- timed region: K full iterations, per-kernel-class events on
    hsa.timing_reset()
    hsa.timing_enable(True)
    l0 = hsa.launch_count()
    if clocks:
        clocks.mark_start()
    ms = time_device(step.full, args.steps, barrier)
    if clocks:
        clocks.mark_end()
    launches = hsa.launch_count() - l0
    hsa.timing_enable(False)
    attn_ms, attn_n = hsa.timing_read(hsa.KCLASS_ATTENTION)
    gemm_ms, gemm_n = hsa.timing_read(hsa.KCLASS_GEMM)
    other_ms, other_n = hsa.timing_read(hsa.KCLASS_OTHER)
    hsa.timing_reset()
    clk = clocks.stop() if clocks else None
    ms_step = allmax(ms) / args.steps
    status = hsa.device_status()
    assert status == 0, f"device status {status}"

    sweep = {}
    if not args.no_sweep:
        for f in (0.5, 0.25):
            for _ in range(2):
                step.partial(f)
            sweep[str(f)] = allmax(time_device(lambda: step.partial(f), max(3, args.steps // 2), barrier)) / \
                max(3, args.steps // 2)
        sweep["1.0"] = ms_step

    e2e = None
    if not args.no_e2e:
        n_e2e = max(3, args.steps // 2)
        e_ms = allmax(time_e2e(step, inp["x0"], n_e2e, barrier)) / n_e2e
        nbytes = GRID.N * SHAPE.D * 4
        e2e = {"value": round(e_ms, 4), "unit": "ms", "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
               "api": "hsa_iteration_host (C ABI, host buffers)",
               "overlap": "two device slots: step k+1's upload and step k's download run on two copy streams "
                          "during compute"}

    peak_sus, peak_burst, hbm, src = load_peaks()
    attn_per_step = attn_ms / args.steps
    achieved = attn_flops_per_full_step() / (attn_per_step * 1e-3) / 1e12
    traffic = traffic_per_launch()
    timed_s = ms_step * args.steps / 1e3
    out = {
        "metric": METRIC, "value": round(ms_step, 4), "unit": "ms", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded random-init weights and inputs)",
        "config": workload_config(1.0),
        "roofline": {"bound": "tensor", "kernel": "k_attn_tc (self + cross attention launches)",
                     "achieved": round(achieved, 1), "peak": peak_burst, "unit": "TFLOP/s",
                     "frac": round(achieved / peak_burst, 4),
                     "peak_note": f"{src} burst bf16 (the timed region lasts {timed_s:.2f} s, too short for the "
                                  f"sustained figure); of {src} sustained {peak_sus}: frac "
                                  f"{achieved / peak_sus:.3f}; of datasheet dense bf16 2250: frac "
                                  f"{achieved / 2250.0:.3f}",
                     "traffic": traffic, "launches_per_step": attn_n // max(args.steps, 1),
                     "flops_per_step": attn_flops_per_full_step()},
        "breakdown_ms_per_step": {"attention": round(attn_per_step, 4), "gemm": round(gemm_ms / args.steps, 4),
                                  "other": round(other_ms / args.steps, 4)},
        "sweep_ms": {k: round(v, 4) for k, v in sweep.items()},
        "whole_job": {"replicas": world, "layer_steps_per_s": round(world * 1000.0 / ms_step, 2),
                      "note": "independent replicas, one per rank; value is the max over ranks of ms per step"},
        "gpu_launches": int(launches),
        "clocks": clk,
        "e2e": e2e,
    }
    return out


# ---------------------------------------------------------------- the other workloads

def _events():
    import torch
    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


def measure_loop(graph: bool = True, n_blocks: int | None = None):
    """Full Wan-1.3B-shaped loop: latent 16x21x60x104 patchified 1x2x2 (N=32760, C=64), 30 blocks,
    T=40; HSA with budgets {40,20,10} sized 25/25/50 % and m=4 against the uniform 40-step run.
    Each run is timed eagerly (host launches) and, with `graph`, as one recorded CUDA graph of all
    T steps.  Weights are drawn on the device (same recipe, N(0, 0.02^2))."""
    import torch
    from token_sparse_denoising_b200 import hsa, pipeline
    hsa.load()
    wl = S.WAN13_LOOP
    N = wl.grid.N
    nb = wl.n_blocks if n_blocks is None else n_blocks
    dev = torch.device("cuda", torch.cuda.current_device())
    pm = S.patch_model_weights_on_device(wl.seed, wl.shape, wl.C, nb, True, dev)
    pos = S.token_positions(wl.grid)
    gen = torch.Generator(device=dev)
    gen.manual_seed(wl.seed)
    ctx = S.device_normal(gen, (wl.shape.ctx_len, wl.shape.D), 1.0, True, dev)
    x0 = S.device_normal(gen, (N, wl.C), 1.0, False, dev)
    vh0 = S.device_normal(gen, (N, wl.C), 1.0, False, dev)
    model = pipeline.PatchModel(pm, pos, N, bf16=True, ctx=ctx, device=dev)
    del pm
    out = {"workload": f"{wl.name}: {nb} blocks D=1536 H=12 F=8960 ctx=512, latent 16x21x60x104 patchified 1x2x2 "
                       f"(N={N}, C=64), T=40, budgets {{40,20,10}} at 25/25/50 %, m=4, shifted sigma (shift 5)",
           "weights": "device-drawn N(0, 0.02^2), seeded"}
    for name, budgets, fracs in (("hsa", wl.budgets, wl.fracs), ("uniform", (wl.T,), (1.0,))):
        sizes = S.group_sizes(N, fracs)
        run = pipeline.HSARun(model, x0, vh0, wl.T, budgets, sizes, wl.m, wl.sigma_kind, wl.shift, device=dev)
        run.step()                                     # warm-up iteration (not timed)
        run = pipeline.HSARun(model, x0, vh0, wl.T, budgets, sizes, wl.m, wl.sigma_kind, wl.shift, device=dev)
        torch.cuda.synchronize()
        a, b = _events()
        a.record()
        run.run()
        b.record()
        b.synchronize()
        assert hsa.device_status() == 0
        out[name] = {"ms": round(a.elapsed_time(b), 1), "token_steps": int(run.n_active.sum()),
                     "active_fraction": round(float(run.n_active.sum()) / (wl.T * N), 4)}
        if graph:
            x_eager = run.x.clone()
            run = pipeline.HSARun(model, x0, vh0, wl.T, budgets, sizes, wl.m, wl.sigma_kind, wl.shift, device=dev)
            n0 = hsa.launch_count()
            t0 = time.perf_counter()
            g = run.capture()
            torch.cuda.synchronize()
            cap_s = time.perf_counter() - t0
            recorded = hsa.launch_count() - n0
            a, b = _events()
            a.record()
            run.replay(g)
            b.record()
            b.synchronize()
            assert hsa.device_status() == 0
            out[name]["graph"] = {"ms": round(a.elapsed_time(b), 1), "capture_s": round(cap_s, 2),
                                  "launches_recorded": int(recorded),
                                  "bitwise_equal_to_eager": bool(torch.equal(run.x, x_eager))}
            del g
    out["speedup"] = round(out["uniform"]["ms"] / out["hsa"]["ms"], 3)
    out["ideal_speedup"] = round(out["uniform"]["token_steps"] / out["hsa"]["token_steps"], 3)
    if graph:
        out["speedup_graph"] = round(out["uniform"]["graph"]["ms"] / out["hsa"]["graph"]["ms"], 3)
    del model
    torch.cuda.empty_cache()
    return out


def measure_tiny(with_oracle: bool = True, reps: int = 5):
    """The tiny fp32 workload as a whole run: 4x16x16 tokens, D = 256, one block, T = 8, budgets
    {8, 4} at 50/50 %, m = 1 (fp32 on the CUDA cores).  Timed eagerly and as one recorded CUDA
    graph, against the uniform 8-step run; with `with_oracle`, the oracle's whole loop on the host
    cores beside it (the loop timed in full, no sampling)."""
    import torch
    from token_sparse_denoising_b200 import hsa, pipeline
    hsa.load()
    wl = S.TINY_FP32
    N, D = wl.grid.N, wl.shape.D
    bw = S.block_weights(wl.seed, wl.shape, False)
    pos = S.token_positions(wl.grid)
    x0, vh0 = S.normal(wl.seed * 10 + 1, (N, D)), S.normal(wl.seed * 10 + 2, (N, D))
    model = pipeline.SingleBlockModel(bw, pos, N, bf16=False)
    out = {"workload": f"{wl.name}: N={N} (4x16x16) D={D} H=2 F=1024 fp32, T={wl.T}, budgets {{8,4}} at 50/50 %, "
                       f"m={wl.m}, linear sigma"}
    for name, budgets, fracs in (("hsa", wl.budgets, wl.fracs), ("uniform", (wl.T,), (1.0,))):
        sizes = S.group_sizes(N, fracs)
        run = pipeline.HSARun(model, x0, vh0, wl.T, budgets, sizes, wl.m, wl.sigma_kind, wl.shift)
        run.run()                                      # warm-up run
        times = []
        for _ in range(reps):
            run.reset(x0, vh0)
            torch.cuda.synchronize()
            a, b = _events()
            a.record()
            run.run()
            b.record()
            b.synchronize()
            times.append(a.elapsed_time(b))
        run.reset(x0, vh0)
        g = run.capture()
        gtimes = []
        for _ in range(reps):
            run.reset(x0, vh0)
            torch.cuda.synchronize()
            a, b = _events()
            a.record()
            run.replay(g)
            b.record()
            b.synchronize()
            gtimes.append(a.elapsed_time(b))
        del g
        assert hsa.device_status() == 0
        out[name] = {"ms": round(statistics.median(times), 3), "graph_ms": round(statistics.median(gtimes), 3),
                     "token_steps": int(run.n_active.sum())}
        if with_oracle:
            from oracle import hsa_oracle as O

            def vel(xA, idx, caches):
                o, Kc, Vc = O.dit_block_active(bw, xA, idx, pos, caches[0], caches[1])
                return o, (Kc, Vc)

            plan = O.make_plan(wl.T, budgets, sizes, wl.m, wl.sigma_kind, wl.shift, N)
            z = np.zeros((N, D))
            t0 = time.perf_counter()
            O.hsa_denoise(x0, vh0, plan, vel, (z, z))
            out[name]["oracle_ms"] = round((time.perf_counter() - t0) * 1e3, 1)
    out["speedup"] = round(out["uniform"]["ms"] / out["hsa"]["ms"], 3)
    out["speedup_graph"] = round(out["uniform"]["graph_ms"] / out["hsa"]["graph_ms"], 3)
    if with_oracle:
        out["oracle"] = {"kind": "oracle", "cores": blas_threads(), "sample": "the whole T = 8 loop, unsampled"}
    return out


def measure_cross(reps: int = 100, gen=None):
    """The cross-attention shape alone: every active query of the Wan-1.3B block (32760) against
    the 512-row text context, 12 heads, bf16; 30 warm-up launches (the clock settles from idle over
    a few milliseconds), then `reps` timed back to back."""
    import torch
    from token_sparse_denoising_b200 import hsa
    hsa.load()
    _, peak_burst, _, _ = load_peaks()
    if gen is None:
        gen = torch.Generator(device="cuda")
        gen.manual_seed(5)
    M, L = S.WAN13_GRID.N, S.WAN13_BLOCK.ctx_len
    k = S.device_normal(gen, (L, 1536), 1.0, True, "cuda")
    v = S.device_normal(gen, (L, 1536), 1.0, True, "cuda")
    q = S.device_normal(gen, (M, 1536), 1.0, True, "cuda")
    o = torch.empty_like(q)
    for _ in range(30):
        hsa.attention(q, k, v, 12, o)
    ms = time_device(lambda: hsa.attention(q, k, v, 12, o), reps, lambda: None) / reps
    tf = 4.0 * M * L * 128 * 12 / (ms * 1e-3) / 1e12
    assert hsa.device_status() == 0
    return {"M": M, "L": L, "H": 12, "ms": round(ms, 4), "tflops": round(tf, 1), "frac_of_burst": round(tf / peak_burst, 3)}


def measure_gemm(gen=None, reps: int = 20):
    """The Wan-1.3B block's GEMMs at |A|/N = 1 (M = 32760), each alone: the library's tcgen05 kernel
    with its fused epilogue against cuBLAS (torch.nn.functional.linear, bf16 out, no epilogue) on
    the same inputs, back to back; the working sets exceed L2."""
    import torch
    from token_sparse_denoising_b200 import hsa
    hsa.load()
    _, peak_burst, _, _ = load_peaks()
    if gen is None:
        gen = torch.Generator(device="cuda")
        gen.manual_seed(5)
    M, D, F = S.WAN13_GRID.N, S.WAN13_BLOCK.D, S.WAN13_BLOCK.F
    out = []
    # the residual GEMMs also with the plain bf16 store, the epilogue cuBLAS is timed with
    for name, kin, nout, epi in (("qkv", D, 3 * D, hsa.EPI_STORE), ("o_proj", D, D, hsa.EPI_RESID),
                                 ("o_proj_store", D, D, hsa.EPI_STORE), ("ffn1_gelu", D, F, hsa.EPI_GELU),
                                 ("ffn2", F, D, hsa.EPI_RESID), ("ffn2_store", F, D, hsa.EPI_STORE)):
        x = S.device_normal(gen, (M, kin), 1.0, True, "cuda")
        w = S.device_normal(gen, (nout, kin), 0.02, True, "cuda")
        b = torch.zeros(nout, device="cuda")
        gate = torch.full((nout,), 0.5, device="cuda")
        resid = epi == hsa.EPI_RESID
        y = torch.zeros((M, nout), device="cuda") if resid else torch.empty((M, nout), dtype=torch.bfloat16,
                                                                              device="cuda")
        run = lambda: hsa.linear(x, w, b, epi, y, gate=gate if resid else None)
        ref = lambda: torch.nn.functional.linear(x, w)
        for _ in range(10):
            run()
            ref()
        ms = time_device(run, reps, lambda: None) / reps
        ms_ref = time_device(ref, reps, lambda: None) / reps
        flop = 2.0 * M * kin * nout
        out.append({"gemm": name, "M": M, "K": kin, "N": nout, "ms": round(ms, 4),
                    "tflops": round(flop / (ms * 1e-3) / 1e12, 1),
                    "frac_of_burst": round(flop / (ms * 1e-3) / 1e12 / peak_burst, 3),
                    "cublas_ms": round(ms_ref, 4), "vs_cublas": round(ms_ref / ms, 3),
                    "epilogue": {0: "bias, bf16 out", 1: "bias + GELU, bf16 out",
                                 2: "fp32 residual += gate * (acc + bias), TMA reduce-add"}[epi]})
        del x, w, y
    assert hsa.device_status() == 0
    torch.cuda.empty_cache()
    return out


def measure_sweep(reps: int = 5):
    """The cross-attention shape and the block's GEMMs (against cuBLAS), attention at N in {8190,
    32760, 75600} x |A|/N in {1, .5, .25, .125} (12 heads, bf16 Q/K/V N(0,1)), and the Euler update
    on N x 64 fp32 latents: one launch after an L2 flush, and back to back in one CUDA graph."""
    import torch
    from token_sparse_denoising_b200 import hsa
    hsa.load()
    _, peak_burst, hbm, src = load_peaks()
    res = {"attention": [], "euler": [], "peaks": f"{src}: burst bf16 {peak_burst} TFLOP/s, HBM {hbm} GB/s",
           "order": "cross-attention and GEMMs first, then the attention sweep, then the Euler update (the "
                    "long attention launches hold the GPU at its power cap, which lowers the clock of "
                    "whatever follows)"}
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5)
    res["cross_attention"] = measure_cross(gen=gen)
    res["gemm"] = measure_gemm(gen)
    for N in (8190, 32760, 75600):
        k = S.device_normal(gen, (N, 1536), 1.0, True, "cuda")
        v = S.device_normal(gen, (N, 1536), 1.0, True, "cuda")
        for f in (1.0, 0.5, 0.25, 0.125):
            M = S.active_fraction_rows(N, f)
            q = S.device_normal(gen, (M, 1536), 1.0, True, "cuda")
            o = torch.empty_like(q)
            need = hsa.attention_workspace_size(M, N, 12, hsa.HSA_BF16)
            ws = torch.empty(need, dtype=torch.uint8, device="cuda") if need else None
            for _ in range(2):
                hsa.attention(q, k, v, 12, o, ws=ws)
            ms = time_device(lambda: hsa.attention(q, k, v, 12, o, ws=ws), reps, lambda: None) / reps
            tf = 4.0 * M * N * 128 * 12 / (ms * 1e-3) / 1e12
            res["attention"].append({"N": N, "frac": f, "M": M, "ms": round(ms, 4), "tflops": round(tf, 1),
                                     "frac_of_burst": round(tf / peak_burst, 3)})
        if N == 32760:
            # the oracle's attention of 8 query rows over the same keys (copied to the host)
            from oracle import hsa_oracle as O
            kh, vh_ = k.float().cpu().numpy().astype(np.float64), v.float().cpu().numpy().astype(np.float64)
            qh = S.device_normal(gen, (8, 1536), 1.0, True, "cuda").float().cpu().numpy().astype(np.float64)
            t0 = time.perf_counter()
            O.attention(qh, kh, vh_)
            row_ms = (time.perf_counter() - t0) * 1e3 / 8
            res["oracle"] = {"kind": "oracle", "cores": blas_threads(), "N": N,
                             "measured_per_unit_ms": {"query_row_ms": round(row_ms, 3)},
                             "value_ms_full": round(row_ms * N, 1),
                             "sample": f"fp64 numpy oracle attention of 8 query rows over {N} keys, 12 heads; "
                                       f"value = query_row_ms x {N} (the |A|/N = 1 launch)"}
            del kh, vh_
        del k, v
    flush = torch.empty(256 * 1024 * 1024 // 4, device="cuda")      # 256 MB > L2: evicts between launches
    flush_r = torch.zeros(256 * 1024 * 1024 // 4, device="cuda")
    for N in (8190, 32760, 75600):
        x = torch.randn((N, 64), device="cuda", generator=gen)
        vh = torch.randn((N, 64), device="cuda", generator=gen)
        times = []
        for _ in range(max(reps, 5)):
            # the flush keeps the GPU busy while the host enqueues the timed launch, so the
            # event interval holds the kernel alone
            a, b = _events()
            flush.zero_()
            flush_r.sum()              # read over the dirty lines: they are written back here, not in the launch
            a.record()
            hsa.euler_update(x, vh, None, None, -0.025)
            b.record()
            b.synchronize()
            times.append(a.elapsed_time(b))
        ms = statistics.median(times)
        gbs = 12 * N * 64 / (ms * 1e-3) / 1e9
        entry = {"N": N, "C": 64, "us": round(ms * 1e3, 2), "bytes": 12 * N * 64, "gbs": round(gbs, 1),
                 "frac_of_hbm": round(gbs / hbm, 3),
                 "l2": "written (256 MB) then read (256 MB) before each launch, so no dirty line of the flush is "
                       "written back inside the timed launch"}
        del x, vh
        # back to back, as in a recorded run: the launches over distinct (x, v_hat) sets, whose total
        # is >= 2x L2, recorded as one CUDA graph (the host's per-call cost is then outside the
        # interval), and the same launches issued one by one from Python for comparison
        sets = max(2, (512 << 20) // (8 * N * 64))
        xs = [torch.randn((N, 64), device="cuda", generator=gen) for _ in range(sets)]
        vs = [torch.randn((N, 64), device="cuda", generator=gen) for _ in range(sets)]

        def issue():
            for k in range(sets):
                hsa.euler_update(xs[k], vs[k], None, None, -0.025)

        for _ in range(2):
            issue()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=side):
                issue()
        torch.cuda.current_stream().wait_stream(side)
        for _ in range(2):
            graph.replay()

        def per_launch(fn):
            out = []
            for _ in range(5):
                a, b = _events()
                a.record()
                fn()
                b.record()
                b.synchronize()
                out.append(a.elapsed_time(b) / sets)
            return statistics.median(out)

        ms_b = per_launch(graph.replay)
        ms_e = per_launch(issue)
        del graph
        gbs_b = 12 * N * 64 / (ms_b * 1e-3) / 1e9
        entry["back_to_back"] = {"us_per_launch": round(ms_b * 1e3, 2), "gbs": round(gbs_b, 1),
                                 "frac_of_hbm": round(gbs_b / hbm, 3), "sets": sets,
                                 "working_set_mb": round(sets * 8 * N * 64 / 1e6, 1),
                                 "launch": "one CUDA graph of the launches",
                                 "issued_from_python_us_per_launch": round(ms_e * 1e3, 2)}
        res["euler"].append(entry)
        del xs, vs
    del flush, flush_r
    torch.cuda.empty_cache()
    return res


def measure_wan14(patterns=("contiguous", "scattered"), reps: int = 3, with_oracle: bool = False):
    """Wan-14B block (D=5120, 40 heads, FFN 13824, no context) at |A|/N in {1, .5, .25, .125}:
    layer-step ms for contiguous and/or scattered active sets.  Weights drawn on the device.  With
    `with_oracle`, the oracle on the same weights and inputs (copied to the host) on a sample: the
    q/k/v projections of 128 tokens and attention over all N cache rows + O-projection + FFN of 4
    query rows, extrapolated to the |A|/N = 1 step."""
    import torch
    from token_sparse_denoising_b200 import hsa
    hsa.load()
    grid, shape = S.WAN13_GRID, S.WAN14_BLOCK
    N, D = grid.N, shape.D
    dev = torch.device("cuda", torch.cuda.current_device())
    w = hsa.LayerWeights(S.block_weights_on_device(4, shape, True, dev), dev, True)
    gen = torch.Generator(device=dev)
    gen.manual_seed(14)
    kc = S.device_normal(gen, (N, D), 1.0, True, dev)
    vc = S.device_normal(gen, (N, D), 1.0, True, dev)
    x = S.device_normal(gen, (N, D), 1.0, False, dev)
    pos = torch.from_numpy(S.token_positions(grid)).to(dev)
    ws = torch.empty(hsa.layer_step_workspace_size(N, D, shape.F, hsa.HSA_BF16), dtype=torch.uint8, device=dev)
    xA = torch.empty((N, D), device=dev)
    peak_burst = load_peaks()[1]
    res = {"workload": "wan14b-block N=32760 (21x30x52) D=5120 H=40 F=13824, no context", "points": []}
    for f in (1.0, 0.5, 0.25, 0.125):
        M = S.active_fraction_rows(N, f)
        for pattern in patterns:
            idx = torch.from_numpy((S.contiguous_mask if pattern == "contiguous" else S.scattered_mask)(46, N, M)).to(dev)
            fn = lambda: hsa.layer_step(w, kc, vc, xA[:M], idx, pos, ws, x_src=x)
            fn()
            ms = time_device(fn, reps, lambda: None) / reps
            flops = 4.0 * M * N * 128 * 40 + 2.0 * M * (3 * D * D + D * D + 2 * D * shape.F)
            tf = flops / (ms * 1e-3) / 1e12
            res["points"].append({"frac": f, "pattern": pattern, "M": M, "ms": round(ms, 3), "tflops": round(tf, 1),
                                  "frac_of_burst": round(tf / peak_burst, 3)})
    assert hsa.device_status() == 0
    if with_oracle:
        res["oracle"] = _oracle_block_sample(w, x, kc, vc, S.token_positions(grid), n_tok=128, n_rows=4)
    del w, kc, vc, x, ws, xA
    torch.cuda.empty_cache()
    return res


def _oracle_block_sample(w, x, kc, vc, pos, n_tok: int, n_rows: int):
    """The fp64 oracle on a sample of one |A|/N = 1 step of a block whose inputs live on the device
    (pulled to the host first, not timed): per-token and per-query-row times and the extrapolation."""
    from oracle import hsa_oracle as O
    N, D = x.shape
    host = lambda t: t.float().cpu().numpy()
    bw = S.BlockWeights(**{k: host(w.t[k]) for k in ("w_qkv", "b_qkv", "g_q", "g_k", "w_o", "b_o", "w_1", "b_1",
                                                       "w_2", "b_2", "mod")})
    X = host(x[:: N // n_tok][:n_tok]).astype(np.float64)
    tok = np.arange(0, N, N // n_tok)[:n_tok]
    Kc, Vc = host(kc).astype(np.float64), host(vc).astype(np.float64)
    t0 = time.perf_counter()
    q, k, v = O.qkv_projection(bw, X, pos[tok])
    t1 = time.perf_counter()
    O.block_tail(bw, X[:n_rows], O.attention(q[:n_rows], Kc, Vc), None)
    t2 = time.perf_counter()
    tok_ms, row_ms = (t1 - t0) * 1e3 / n_tok, (t2 - t1) * 1e3 / n_rows
    return {"kind": "oracle", "cores": blas_threads(), "value_ms_full_step": round((tok_ms + row_ms) * N, 1),
            "measured_per_unit_ms": {"token_ms": round(tok_ms, 4), "query_row_ms": round(row_ms, 3)},
            "sample": f"fp64 numpy oracle: q/k/v projections of {n_tok} tokens, attention over all {N} cache rows "
                      f"+ O-projection + FFN of {n_rows} query rows; value = (token_ms + query_row_ms) x {N}, "
                      f"the |A|/N = 1 step"}


def run_loop(args):
    return {"mode": "loop", **measure_loop(graph=True)}


def run_tiny(args):
    return {"mode": "tiny", **measure_tiny(with_oracle=True)}


def run_sweep(args):
    return {"mode": "sweep", **measure_sweep()}


def run_wan14(args):
    return {"mode": "wan14", **measure_wan14()}


def run_headpar(args, rank, world, barrier, allmax, dist):
    """One Wan-14B-shaped block (N = 32760, D = 5120, 40 heads, FFN 13824, every token active) split
    by heads over the `world` ranks: rank r holds 40/world heads (their q/k/v rows, KV cache columns
    and W_o columns), 13824/world FFN columns and 1/world of the residual rows; all-gather /
    all-reduce / reduce-scatter over NCCL between the phases.  ms per block step, max over ranks."""
    import torch
    from token_sparse_denoising_b200 import hsa, sharded
    hsa.load()
    grid, shape = S.WAN13_GRID, S.WAN14_BLOCK
    N, D = grid.N, shape.D
    dev = torch.device("cuda", torch.cuda.current_device())
    shard = sharded.HeadShard(rank, world, shape.H, shape.F, N)
    bw = S.block_weights_on_device(4, shape, True, dev)        # the same draws on every rank
    gen = torch.Generator(device=dev)
    gen.manual_seed(14)
    kc = S.device_normal(gen, (N, D), 1.0, True, dev)
    vc = S.device_normal(gen, (N, D), 1.0, True, dev)
    x = S.device_normal(gen, (N, D), 1.0, False, dev)
    blk = sharded.HeadParallelBlock(bw, shard, N, dev, cache_init=(kc, vc))
    del bw, kc, vc
    torch.cuda.empty_cache()
    idx = torch.arange(N, dtype=torch.int32, device=dev)
    pos = torch.from_numpy(S.token_positions(grid)).to(dev)
    if dist is None:
        step = lambda: sharded.EmulatedGroup.run([blk.step(x, idx, pos)])
    else:
        step = lambda: sharded.run_collectives(blk.step(x, idx, pos), dist)
    for _ in range(max(args.warmup, 1)):
        step()
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 10))
    ms = allmax(time_device(step, steps, barrier)) / steps
    assert hsa.device_status() == 0
    flops = 4.0 * N * N * 128 * shape.H + 2.0 * N * (3 * D * D + D * D + 2 * D * shape.F)
    return {"mode": "headpar", "metric": "Wan-14B block step ms, heads split over the ranks", "value": round(ms, 3),
            "unit": "ms", "n_gpus": world, "steps": steps, "higher_is_better": False, "scaling": "strong",
            "config": {"workload": "wan14b-block N=32760 D=5120 H=40 F=13824 |A|/N=1",
                       "parallelism": f"heads/{world} per rank, NCCL all-gather + all-reduce + reduce-scatter"},
            "tflops_aggregate": round(flops / (ms * 1e-3) / 1e12, 1)}


def measure_configs():
    """The other workloads, measured beside the headline step on the same GPU in the same run."""
    t0 = time.perf_counter()
    out = {"attention_euler_sweep": measure_sweep(),
           "wan14_block": measure_wan14(with_oracle=True),
           "tiny_fp32_loop": measure_tiny(with_oracle=True), "wan13_loop": measure_loop(graph=False)}
    out["wall_s"] = round(time.perf_counter() - t0, 1)
    return out


# ---------------------------------------------------------------- the oracle on the host cores

# One sample of a full iteration, used by both the CPU baseline beside the GPU numbers and the
# reference arm: the q/k/v projections, Euler update and score of SAMPLE[0] tokens, and attention
# over all N cache rows + O-projection + cross-attention + FFN of SAMPLE[1] query rows.
SAMPLE = (4096, 128)
BASELINE_SECONDS = 10.0          # host work of the CPU baseline: repeats of the sample


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_step_sample(inp, sample=SAMPLE):
    """Time the oracle on a bounded sample of one full iteration.

    Every part of the step is linear in the rows it touches, so each is timed on a spread
    sample and scaled: the q/k/v projections (LN, GEMM, RMSNorm, RoPE) and the cached Euler
    update + L1 score of n_proj tokens (x N/n_proj); attention over all N cache rows +
    O-projection + cross-attention + FFN of n_rows query rows (x N/n_rows); the regrouping
    runs on all N scores.  Returns the extrapolated ms per step, the sample's wall seconds
    and the measured per-unit times.
    """
    from oracle import hsa_oracle as O
    N = GRID.N
    n_proj, n_rows = min(sample[0], N), min(sample[1], sample[0], N)
    bw, pos = inp["bw"], inp["pos"]
    ctx_kv = O.context_kv(bw, inp["ctx"])            # once per run: not part of a step
    proj = np.arange(0, N, N // n_proj)[:n_proj]
    qrows = np.arange(0, n_proj, n_proj // n_rows)[:n_rows]
    X = inp["x0"][proj].astype(np.float64)
    Kc, Vc = inp["kc0"].astype(np.float64), inp["vc0"].astype(np.float64)
    t0 = time.perf_counter()
    q, k, v = O.qkv_projection(bw, X, pos[proj])
    Kc[proj], Vc[proj] = k, v
    t1 = time.perf_counter()
    O.block_tail(bw, X[qrows], O.attention(q[qrows], Kc, Vc), ctx_kv)
    t2 = time.perf_counter()
    vA = inp["va"][proj].astype(np.float64)          # a stand-in velocity of the same shape
    score = O.l1_relative_change(vA, inp["vh0"][proj])
    O.cached_euler(inp["x0"][proj], inp["vh0"][proj], vA, np.arange(len(proj)), DSIGMA)
    t3 = time.perf_counter()
    O.select_groups(np.resize(score.astype(np.float32), N), S.group_sizes(N, GROUP_FRACS))
    t4 = time.perf_counter()
    per_token = (t1 - t0) + (t3 - t2)
    est_ms = (per_token * N / len(proj) + (t2 - t1) * N / len(qrows) + (t4 - t3)) * 1e3
    units = {"token_ms": per_token * 1e3 / len(proj), "query_row_ms": (t2 - t1) * 1e3 / len(qrows),
             "regroup_ms": (t4 - t3) * 1e3}
    return est_ms, (t4 - t0), units


def _sample_text(reps, units):
    N = GRID.N
    return (f"fp64 numpy oracle, {reps} repeat(s) of one sample of a full iteration: q/k/v projections + "
            f"Euler/score of {SAMPLE[0]} of {N} tokens (measured {units['token_ms']:.4f} ms per token, x{N}), "
            f"attention over all {N} cache rows + O/cross/FFN of {SAMPLE[1]} query rows (measured "
            f"{units['query_row_ms']:.3f} ms per row, x{N}), regrouping of {N} scores "
            f"({units['regroup_ms']:.1f} ms); value = the linear extrapolation to one full step")


def cpu_baseline(inp):
    vals, units, wall = [], [], 0.0
    while wall < BASELINE_SECONDS or len(vals) < 2:
        v, w, u = oracle_step_sample(inp)
        vals.append(v)
        units.append(u)
        wall += w
    med = lambda key: statistics.median(u[key] for u in units)
    u = {k: med(k) for k in units[0]}
    return {"value": round(statistics.median(vals), 1), "unit": "ms", "cores": blas_threads(), "kind": "oracle",
            "sample": _sample_text(len(vals), u), "measured_per_unit_ms": {k: round(x, 5) for k, x in u.items()},
            "wall_s": round(wall, 2)}


def run_reference(args):
    """The reference arm: the oracle as it stands on the host cores, one sample of a full
    iteration per step (the same sample as the CPU baseline of the GPU line); the value is the
    median of the steps' extrapolated ms per full step."""
    inp = synthetic_inputs()
    for _ in range(args.warmup):
        oracle_step_sample(inp)
    vals, units, wall = [], [], 0.0
    for _ in range(args.steps):
        v, w, u = oracle_step_sample(inp)
        vals.append(v)
        units.append(u)
        wall += w
    value = float(statistics.median(vals))
    u = {k: statistics.median(x[k] for x in units) for k in units[0]}
    return {"impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": "ms", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(value, 1), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(1.0),
            "cpu_baseline": {"value": round(value, 1), "unit": "ms", "cores": blas_threads(), "kind": "oracle",
                             "sample": _sample_text(args.steps, u),
                             "measured_per_unit_ms": {k: round(x, 5) for k, x in u.items()}},
            "e2e": {"value": round(value, 1), "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "timing_note": "each step times one bounded sample and extrapolates it to a full step, so "
                           "ms_per_step x steps is far longer than the run; sample_wall_s is what was spent",
            "sample_wall_s": round(wall, 1)}


# ---------------------------------------------------------------- main

def collectives(dist, device):
    """Barrier and max-over-ranks of a float; plain pass-throughs on one process.

    `dist` is torch.distributed after init_process_group (NCCL on the GPUs, gloo in the
    CPU tests) or None.  Every rank calls both in the same order.
    """
    import torch

    def barrier():
        if dist is not None:
            dist.barrier()

    def allmax(v: float) -> float:
        if dist is None:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    return barrier, allmax


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0

    import torch
    torch.cuda.set_device(local)
    if args.mode == "headpar":
        dist = None
        if world > 1 or "RANK" in os.environ:          # under torchrun: NCCL even for one rank
            import datetime
            import torch.distributed as dist
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        barrier, allmax = collectives(dist, "cuda")
        try:
            out = run_headpar(args, rank, world, barrier, allmax, dist)
        finally:
            if dist is not None:
                dist.barrier()
                dist.destroy_process_group()
        if rank == 0:
            print(json.dumps(out), flush=True)
        return 0
    if args.mode != "step":
        if rank == 0:
            fn = {"loop": run_loop, "sweep": run_sweep, "wan14": run_wan14, "tiny": run_tiny,
                  "cross": lambda a: {"mode": "cross", **measure_cross()},
                  "gemm": lambda a: {"mode": "gemm", "gemm": measure_gemm()}}[args.mode]
            print(json.dumps(fn(args)), flush=True)
        return 0
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    barrier, allmax = collectives(dist, "cuda")

    try:
        out = run_gpu(args, rank, world, barrier, allmax)
    finally:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_configs:
            out["configs"] = measure_configs()
        if world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_baseline(synthetic_inputs())
            loop = out.get("configs", {}).get("wan13_loop")
            if loop:
                u = out["cpu_baseline"]["measured_per_unit_ms"]
                blocks = S.WAN13_LOOP.n_blocks
                for name in ("hsa", "uniform"):
                    loop[name]["oracle_ms_estimate"] = round(
                        loop[name]["token_steps"] * (u["token_ms"] + u["query_row_ms"]) * blocks, 0)
                loop["oracle_note"] = ("estimate, not a run: the oracle's measured per-token and per-query-row "
                                       f"costs of one Wan-1.3B block x {blocks} blocks x the run's token-steps")
        print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
