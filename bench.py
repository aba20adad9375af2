#!/usr/bin/env python
"""Benchmark of the Mamba-1 selective-SSM layer core on B200.

One step = the whole hot path over one batch, for every layer of the
workload: causal conv1d + SiLU forward, selective scan forward, selective
scan backward, conv1d backward. Default workload: the long-context shape,
4 independent layers of B=2, d_inner=1536, d_state=16, L=32768, bf16
activations with fp32 state (inputs of each layer ~0.8 GB, larger than L2,
layers rotated, so no L2 flush is needed).

Prints one JSON line (rank 0). `value` is layer-tokens/s of the whole step
with inputs resident in HBM; `e2e` is the same metric through the same C-ABI
calls with host buffers (pinned host -> device copies of every input and
device -> host copies of every output inside the timed region).

`--impl reference` times the fp64 CPU oracle on a bounded sample of the same
workload (the reference arm for this project); the oracle is also timed as
`cpu_baseline` on rank 0 at N=1.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "scan fwd+bwd tokens/s (B2×1536ch×32K, N=16); achieved HBM GB/s % of roofline"
UNIT = "layer-tokens/s"
SFU_EX2_PER_CLK_PER_SM = 16  # MUFU ex2 results per SM per clock (ssm_probe_ex2_rate measures it)


# DRAM bytes (read + write) per launch of the current N = 16 scan kernels at
# the 32K bench workload (one layer B2 D1536 N16 L32768 bf16, 11-warp CTAs),
# from one ncu capture of these kernels at that shape (its summary is kept with
# the profiles); a kernel changed since its capture has no entry.
NCU_TRAFFIC = {"scan_bwd": 1832.669e6 + 597.325e6, "scan_fwd": 612.897e6 + 1155.971e6}


def _peaks():
    """HBM copy bandwidth and dense bf16 tensor throughput of this machine's B200s
    (MEASURED_PEAKS.json when present; else the earlier measurement on this
    pool: 6650 GB/s, 1590 TFLOP/s)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": float(pk["hbm_gbs"]), "sm_max_mhz": float(pk.get("sm_max_mhz", 1965.0)),
                "bf16_tflops": float(pk.get("bf16_tflops", 1590.0)), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0, "bf16_tflops": 1590.0, "source": "fallback"}


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------
_REASONS = ["gpu_idle", "applications_clocks_setting", "sw_power_cap", "hw_slowdown", "sync_boost",
            "sw_thermal_slowdown", "hw_thermal_slowdown", "hw_power_brake_slowdown",
            "display_clock_setting"]


class ClockSampler:
    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.th = threading.Thread(target=self._read, daemon=True)
        self.th.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.th.join(timeout=2)
        mhz, mx, reasons = [], [], set()
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 8:
                continue
            try:
                mhz.append(float(f[0]))
                mx.append(float(f[1]))
                act = int(f[3], 16) if f[3].startswith("0x") else int(f[3])
            except ValueError:
                continue
            for bit, name in enumerate(_REASONS):
                if act & (1 << bit) and name != "gpu_idle":
                    reasons.add(name)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(mhz)}


# ----------------------------------------------------------------------------
# one layer on the device
# ----------------------------------------------------------------------------
class Layer:
    """Device buffers of one layer and the four C-ABI calls of a step."""

    def __init__(self, inp, device, n_splits):
        import torch
        import selective_state_space_35_b200 as ssm
        self.ssm = ssm
        self.shape = inp.shape
        B, D, N, L = inp.shape.B, inp.shape.D, inp.shape.N, inp.shape.L
        bf = torch.bfloat16

        def act(t):
            return torch.from_numpy(t.bits.view(np.int16)).view(bf).to(device)

        self.host = {k: getattr(inp, k) for k in ("x", "z", "delta", "Bm", "Cm", "dout")}
        self.x, self.z, self.delta = act(inp.x), act(inp.z), act(inp.delta)
        self.Bm, self.Cm, self.dout = act(inp.Bm), act(inp.Cm), act(inp.dout)
        f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)  # noqa: E731
        self.A, self.Dskip, self.dbias = f32(inp.A), f32(inp.Dskip), f32(inp.delta_bias)
        self.w, self.cb = f32(inp.conv_w), f32(inp.conv_b)
        self.seq = (torch.from_numpy(inp.seq_idx).to(device) if inp.seq_idx is not None else None)
        e = lambda: torch.empty((B, D, L), dtype=bf, device=device)  # noqa: E731
        self.u, self.out, self.dx = e(), e(), e()
        self.final_state = torch.empty((B, D, N), dtype=torch.float32, device=device)
        self.g = {"du": e(), "ddelta": e(), "dz": e(),
                  "dA": torch.empty((D, N), dtype=torch.float32, device=device),
                  "dB": torch.empty((B, N, L), dtype=torch.float32, device=device),
                  "dC": torch.empty((B, N, L), dtype=torch.float32, device=device),
                  "dD": torch.empty((D,), dtype=torch.float32, device=device),
                  "ddelta_bias": torch.empty((D,), dtype=torch.float32, device=device)}
        self.dw = torch.empty((D, 4), dtype=torch.float32, device=device)
        self.dcb = torch.empty((D,), dtype=torch.float32, device=device)
        p = ssm.scan_params(self.u, self.delta, self.A, self.Bm, self.Cm, z=self.z, Dskip=self.Dskip,
                            delta_bias=self.dbias, seq_idx=self.seq, n_splits=n_splits,
                            out=self.out, final_state=self.final_state)
        self.ws = torch.empty(ssm.scan_workspace_size(p), dtype=torch.uint8, device=device)
        self.cws = torch.empty(ssm.ssm_conv1d_bwd_workspace_size(B, D, L, 4), dtype=torch.uint8,
                               device=device)
        self.n_splits = n_splits
        self.kw = dict(z=self.z, Dskip=self.Dskip, delta_bias=self.dbias, seq_idx=self.seq,
                       n_splits=n_splits)

    def launches(self, deterministic=False) -> int:
        """Kernels of this library one step of this layer launches."""
        nch = (self.shape.L + 255) // 256
        P = self.n_splits
        if P == 0:  # mirror the library's automatic choice
            rows = self.shape.B * self.shape.D
            P = 1 if rows >= 148 * 8 else -(-148 * 8 // rows)
        P = max(1, min(P, nch))
        cps = -(-nch // P)
        P = -(-nch // cps)
        extra = 2 if P > 1 else 0
        # N = 16 on one range per row: B / C packing + scan forward
        fwd = 2 if (P == 1 and self.shape.N == 16 and self.shape.L % 8 == 0) else 1 + extra
        return 1 + fwd + (2 + extra + (1 if deterministic else 0)) + 2

    def bytes_held(self) -> dict:
        """Device bytes of this layer: the scan and conv workspaces, and all
        buffers (inputs, outputs, gradients, workspaces)."""
        import torch
        tens = [v for v in vars(self).values() if isinstance(v, torch.Tensor)]
        tens += [v for v in self.g.values() if isinstance(v, torch.Tensor)]
        return {"scan_workspace": self.ws.numel(), "conv_bwd_workspace": self.cws.numel(),
                "all_buffers": sum(t.numel() * t.element_size() for t in tens)}

    def step(self, ev=None):
        ssm = self.ssm
        if ev is not None:
            ev[0].record()
        ssm.conv1d_fwd(self.x, self.w, self.cb, self.seq, out=self.u)
        if ev is not None:
            ev[1].record()
        ssm.scan_fwd(self.u, self.delta, self.A, self.Bm, self.Cm, out=self.out,
                     workspace=self.ws,
                     final_state=self.final_state if self.shape.final_state else None, **self.kw)
        if ev is not None:
            ev[2].record()
        ssm.scan_bwd(self.u, self.delta, self.A, self.Bm, self.Cm, self.dout, self.ws,
                     grads=self.g, **self.kw)
        if ev is not None:
            ev[3].record()
        ssm.conv1d_bwd(self.x, self.w, self.cb, self.seq, self.g["du"], dx=self.dx, dw=self.dw,
                       dbias=self.dcb, workspace=self.cws)
        if ev is not None:
            ev[4].record()


# ----------------------------------------------------------------------------
# CPU oracle timing (bounded sample of the same workload)
# ----------------------------------------------------------------------------
def oracle_sample(inp, seconds: float, threads: int):
    """Run the fp64 oracle on channel rows of batch row 0 until `seconds` pass.

    Returns (layer-tokens/s equivalent, rows done, seconds, threads)."""
    import oracle
    sh = inp.shape
    D, L = sh.D, sh.L
    rows_per = max(1, threads)
    done, t_total, d0 = 0, 0.0, 0
    bf16 = sh.dtype == "bf16"

    def f64(t, sl):
        v = synth.bf16_bits_to_f32(t.bits[sl]) if t.bits is not None else t.f32[sl]
        return v.astype(np.float64)

    stored = oracle.round_bf16 if bf16 else (lambda a: a)  # the activation dtype's rounding
    while t_total < seconds and d0 < D:
        d1 = min(D, d0 + rows_per)
        sl = np.s_[0:1, d0:d1, :]
        x, z, dl, go = f64(inp.x, sl), f64(inp.z, sl), f64(inp.delta, sl), f64(inp.dout, sl)
        Bm, Cm = f64(inp.Bm, np.s_[0:1]), f64(inp.Cm, np.s_[0:1])
        seq = None if inp.seq_idx is None else np.ascontiguousarray(inp.seq_idx[0:1])
        A, Dk, db = inp.A[d0:d1], inp.Dskip[d0:d1], inp.delta_bias[d0:d1]
        w, cb = inp.conv_w[d0:d1], inp.conv_b[d0:d1]
        t0 = time.perf_counter()
        _, u = oracle.conv1d_fwd(x, w, cb, seq)
        u = stored(u)
        kw = dict(z=z, Dskip=Dk, delta_bias=db, seq_idx=seq, nthreads=threads)
        oracle.scan_fwd(u, dl, A, Bm, Cm, **kw)
        g = oracle.scan_bwd(u, dl, A, Bm, Cm, go, **kw)
        oracle.conv1d_bwd(x, w, cb, seq, stored(g["du"]))
        t_total += time.perf_counter() - t0
        done += d1 - d0
        d0 = d1
    # a full layer is B*D such rows and carries B*L tokens
    tok_s = (done * L) / (D * t_total) if t_total > 0 else 0.0
    return tok_s, done, t_total


def cpu_count() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, cfg, rank):
    if rank != 0:
        return 0
    sh = synth.CONFIGS[cfg]
    sh1 = synth.Shape(sh.name, sh.B, sh.D, sh.N, sh.L, sh.dtype, packed=sh.packed)
    inp = synth.make_inputs(sh1, synth.seed_for(cfg, 0), want_f64=False)
    threads = cpu_count()
    budget = max(1.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(inp, budget * 0.25, threads)
    vals, secs, rows = [], 0.0, 0
    for _ in range(args.steps):
        v, r, s = oracle_sample(inp, budget, threads)
        vals.append(v)
        secs += s
        rows += r
    val = float(np.mean(vals)) if vals else 0.0
    sample = (f"{rows} channel rows x {sh.L} tokens of layer 0 ({sh.name}), conv+scan fwd+bwd in "
              f"fp64, over {args.steps} steps of ~{budget:.1f} s")
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * secs / max(1, args.steps), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(sh, cfg),
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(sh, cfg):
    return {"workload": f"{sh.name} bf16, conv1d+SiLU -> selective scan fwd+bwd -> conv1d bwd",
            "layers": sh.layers, "B": sh.B, "D": sh.D, "N": sh.N, "L": sh.L,
            "conv_width": 4, "storage": sh.dtype, "state": "f32", "packed": sh.packed,
            "l2": "inputs larger than L2 (each layer's inputs > 126 MB, layers rotated); no flush"}


# ----------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=3, choices=(2, 3, 4, 5),
                    help="bench workload (the bf16 configs; 1 is a parity case only)")
    ap.add_argument("--n-splits", type=int, default=0)
    ap.add_argument("--layers", type=int, default=0, help="limit the layer count (profiling)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-decode", action="store_true", help="skip the recurrent-step measurement")
    ap.add_argument("--no-complex", action="store_true", help="skip the complex-A scan measurement")
    ap.add_argument("--no-cp", action="store_true",
                    help="skip the per-rank measurement of the context-parallel kernels")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the scan measurement on the other full-size workloads")
    ap.add_argument("--no-deterministic", action="store_true",
                    help="skip the measurement of the deterministic backward")
    ap.add_argument("--no-ssd", action="store_true", help="skip the Mamba-2 SSD forward measurement")
    ap.add_argument("--no-fused", action="store_true",
                    help="skip the fused conv + scan forward measurement")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = args.config
    if args.impl == "reference":
        return run_reference(args, cfg, rank)

    import torch
    import torch.distributed as dist
    from selective_state_space_35_b200 import build
    build.build()
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)

    sh = synth.CONFIGS[cfg]
    nlayers = args.layers if args.layers > 0 else sh.layers
    inps = [synth.make_inputs(sh, synth.seed_for(cfg, l), want_f64=False) for l in range(nlayers)]
    layers = [Layer(inp, device, args.n_splits) for inp in inps]
    stream = torch.cuda.current_stream(device)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        for ly in layers:
            ly.step()
    torch.cuda.synchronize()

    nlay = len(layers)
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(nlay)]
           for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                          else int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank]))
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for s in range(args.steps):
        for i, ly in enumerate(layers):
            ly.step(evs[s][i])
    stop.record(stream)
    torch.cuda.synchronize()
    barrier()
    ck = clocks.stop()
    ms = start.elapsed_time(stop)
    if world > 1:
        t = torch.tensor([ms], device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    ms_step = ms / args.steps
    tokens_step = nlay * sh.B * sh.L
    value = world * tokens_step / (ms_step * 1e-3)

    # per-call durations (events bracket each C-ABI call on the launching stream)
    names = ["conv1d_fwd", "scan_fwd", "scan_bwd", "conv1d_bwd"]
    per = {n: [] for n in names}
    for s in range(args.steps):
        for i in range(nlay):
            e = evs[s][i]
            for k, n in enumerate(names):
                per[n].append(e[k].elapsed_time(e[k + 1]))
    avg = {n: float(np.mean(v)) for n, v in per.items()}
    scan_ms = avg["scan_fwd"] + avg["scan_bwd"]
    B, D, N, L = sh.B, sh.D, sh.N, sh.L
    pk = _peaks()
    e_sz = 2
    bytes_tok = {"scan_fwd": 4 * D * e_sz + 2 * N * e_sz,
                 "scan_bwd": 7 * D * e_sz + 2 * N * e_sz + 2 * N * 4,
                 "conv1d_fwd": 2 * D * e_sz, "conv1d_bwd": 3 * D * e_sz}
    hbm = {n: bytes_tok[n] * B * L / (avg[n] * 1e-3) / 1e9 for n in names}
    dom = max(names, key=lambda n: avg[n])
    exps = B * D * L * N
    ex2_peak = SFU_EX2_PER_CLK_PER_SM * 148 * pk["sm_max_mhz"] * 1e6 / 1e12  # T ex2/s
    if dom.startswith("scan"):
        achieved = exps / (avg[dom] * 1e-3) / 1e12
        roof = {"bound": "alu", "achieved": achieved, "peak": ex2_peak, "unit": "Tex2/s",
                "frac": achieved / ex2_peak, "traffic": NCU_TRAFFIC.get(dom) if cfg == 3 else None,
                "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + "
                                "dram__bytes_write.sum)",
                "kernel": f"ssm_{dom}",
                "peak_source": "derived: 16 ex2/clk/SM x 148 SMs x max SM clock (of measured "
                               "clock)", "work_per_launch": f"{exps} ex2 (B*D*L*N)"}
    else:
        achieved = hbm[dom]
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "traffic": None, "kernel": f"ssm_{dom}"}
    t_sfu = 2 * exps / (ex2_peak * 1e12) * 1e3
    t_hbm = (bytes_tok["scan_fwd"] + bytes_tok["scan_bwd"]) * B * L / (pk["hbm_gbs"] * 1e9) * 1e3
    # secondary bound: the fp32 arithmetic the recurrences need per (token,
    # state), ~4 ops forward and ~13 backward besides the exp, on 128 fp32
    # lanes per SM at the max SM clock (an FMA counted as one op)
    fp32_lane_ops = 148 * 128 * pk["sm_max_mhz"] * 1e6
    t_fp32 = {"scan_fwd": exps * 4 / fp32_lane_ops * 1e3, "scan_bwd": exps * 13 / fp32_lane_ops * 1e3}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": dict(workload_config(sh, cfg), parallelism=f"replicas x{world}"),
        "roofline": roof,
        "scan": {"tokens_per_s": world * B * L / (scan_ms * 1e-3),  # scan fwd+bwd per layer
                 "ms_per_layer": {n: avg[n] for n in names},
                 "hbm_gbs": hbm, "hbm_frac_of_measured": {n: hbm[n] / pk["hbm_gbs"] for n in names},
                 "hbm_frac_of_nominal_8tbs": {n: hbm[n] / 8000.0 for n in names},
                 "roofline_ms_per_layer": {"sfu_2BDLN": t_sfu, "hbm_alg_bytes": t_hbm,
                                           "fp32_pipe": t_fp32},
                 "frac_of_roofline": max(t_sfu, t_hbm) / scan_ms},
        "gpu_launches": args.steps * sum(ly.launches() for ly in layers),
        "clocks": ck,
        "bytes_per_layer": layers[0].bytes_held(),
    }

    # e2e: host buffers in, host buffers out, through the same calls
    if not args.no_e2e:
        line["e2e"] = e2e(layers, device, args, world)

    if not args.no_decode:
        line["decode"] = decode_bench(device, sh, pk)
    if not args.no_complex:
        line["complex_a"] = complex_bench(device, layers[0], pk)
    if not args.no_cp:
        line["cp_shard"] = cp_shard_bench(device, layers[0], ranks=8)
    if not args.no_deterministic:
        line["deterministic_bwd"] = deterministic_bench(layers[0], avg["scan_bwd"])
    if not args.no_ssd:
        line["ssd"] = ssd_bench(device, pk)
    if not args.no_fused:
        line["fused_fwd"] = fused_fwd_bench(layers[0], avg["conv1d_fwd"] + avg["scan_fwd"])
    line["peaks"] = {k: pk[k] for k in ("hbm_gbs", "bf16_tflops", "sm_max_mhz", "source")}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = cpu_count()
        v, rows, secs = oracle_sample(inps[0], args.cpu_seconds, threads)
        v1, rows1, secs1 = oracle_sample(inps[0], max(2.0, args.cpu_seconds / 3), 1)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": f"{rows} channel rows x {L} tokens of layer 0, conv+scan "
                                          f"fwd+bwd in fp64, {secs:.1f} s",
                                "single_thread": {"value": v1, "cores": 1,
                                                  "sample": f"{rows1} channel rows x {L} tokens, "
                                                            f"{secs1:.1f} s"}}
    del inps
    if not args.no_configs:
        del layers
        torch.cuda.empty_cache()
        line["other_configs"] = {str(c): config_bench(c, device, pk) for c in (2, 4, 5)}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def scan_roofline(sh, fwd_ms, bwd_ms, pk):
    """Algorithmic HBM bytes and the SFU / HBM bounds of the scan fwd + bwd of
    one layer of shape `sh` (bf16 activations)."""
    B, D, N, L = sh.B, sh.D, sh.N, sh.L
    e_sz = 2
    by_fwd = (4 * D * e_sz + 2 * N * e_sz) * B * L
    by_bwd = (7 * D * e_sz + 2 * N * e_sz + 2 * N * 4) * B * L
    exps = B * D * L * N
    ex2_peak = SFU_EX2_PER_CLK_PER_SM * 148 * pk["sm_max_mhz"] * 1e6
    t_sfu = 2 * exps / ex2_peak * 1e3
    t_hbm = (by_fwd + by_bwd) / (pk["hbm_gbs"] * 1e9) * 1e3
    return {"hbm_gbs": {"scan_fwd": by_fwd / (fwd_ms * 1e-3) / 1e9,
                        "scan_bwd": by_bwd / (bwd_ms * 1e-3) / 1e9},
            "roofline_ms": {"sfu_2BDLN": t_sfu, "hbm_alg_bytes": t_hbm},
            "frac_of_roofline": max(t_sfu, t_hbm) / (fwd_ms + bwd_ms)}


def config_bench(cfg, device, pk, reps=5):
    """One layer of another full-size workload: the four calls of a step timed
    with CUDA events per call over `reps` steps after 3 warm-up steps (inputs
    larger than L2 for every config; the same buffers each step)."""
    import torch
    sh = synth.CONFIGS[cfg]
    inp = synth.make_inputs(sh, synth.seed_for(cfg, 0), want_f64=False)
    ly = Layer(inp, device, 0)
    del inp
    for _ in range(3):
        ly.step()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(reps)]
    for e in ev:
        ly.step(e)
    torch.cuda.synchronize()
    names = ["conv1d_fwd", "scan_fwd", "scan_bwd", "conv1d_bwd"]
    ms = {n: sum(e[k].elapsed_time(e[k + 1]) for e in ev) / reps for k, n in enumerate(names)}
    scan_ms = ms["scan_fwd"] + ms["scan_bwd"]
    step_ms = sum(ms.values())
    r = {"workload": sh.name + (", packed documents" if sh.packed else "")
                     + (", final state returned" if sh.final_state else ""),
         "ms_per_layer": ms, "scan_tokens_per_s": sh.B * sh.L / (scan_ms * 1e-3),
         "step_tokens_per_s": sh.B * sh.L / (step_ms * 1e-3),
         "bytes_per_layer": ly.bytes_held(), "launches": (reps + 3) * ly.launches()}
    r.update(scan_roofline(sh, ms["scan_fwd"], ms["scan_bwd"], pk))
    del ly
    torch.cuda.empty_cache()
    return r


def ssd_bench(device, pk, B=2, L=8192, H=64, P=64, G=1, N=128, reps=5):
    """Mamba-2 SSD forward and backward on the tensor cores at a d_inner =
    4096 shape (64 heads of 64, one B / C group, state 128), B2 L8192 bf16:
    CUDA events over `reps` calls after two warm-up calls (inputs 0.28 GB,
    larger than L2). The forward is timed alone (inference: no saved states)
    and as the training forward that saves the chunk states; the backward
    from those states and a seeded dy."""
    import torch
    import selective_state_space_35_b200 as ssm
    si = synth.ssd_inputs(B, L, H, P, G, N, synth.seed_for(11))

    def bf(t):
        return torch.from_numpy(t.bits.view(np.int16).copy()).view(torch.bfloat16).to(device)

    def f32(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)

    x, dtr, Bm, Cm = bf(si.x), bf(si.dt_raw), bf(si.Bm), bf(si.Cm)
    A, D, db = f32(si.A), f32(si.D), f32(si.dt_bias)
    rng = np.random.Generator(np.random.PCG64(synth.seed_for(12)))
    dy = torch.from_numpy(synth.f32_to_bf16_bits(rng.standard_normal((B, L, H, P)).astype(np.float32))
                          .view(np.int16)).view(torch.bfloat16).to(device)
    y = torch.empty_like(x)
    cs = torch.empty(ssm.ssd_chunk_states_shape(B, L, H, P, N), dtype=torch.float32, device=device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    ms = timed(lambda: ssm.ssd_fwd(x, dtr, A, Bm, Cm, D=D, dt_bias=db, out=y))
    ms_train = timed(lambda: ssm.ssd_fwd(x, dtr, A, Bm, Cm, D=D, dt_bias=db, out=y, chunk_states=cs))
    ms_bwd = timed(lambda: ssm.ssd_bwd(x, dtr, A, Bm, Cm, dy, cs, D=D, dt_bias=db))
    Q = 128
    chunks = B * H * (-(-L // Q))
    # per chunk: C B^T (2 Q Q N), Y_diag (2 Q P Q), Y_off (2 Q P N), chunk state (2 N P Q)
    flops = chunks * (2 * Q * Q * N + 2 * Q * P * Q + 2 * Q * P * N + 2 * N * P * Q)
    issued = flops + chunks * 2 * Q * P * Q  # the remainder product of the decay-masked C B^T
    # backward per chunk: C B^T, dy x^T, B dH, C Hp, C^T dYs, M^T dy, dS B, dYs Hp^T, dS^T C, x dH^T
    flops_bwd = chunks * 2 * (Q * Q * N + Q * Q * P + Q * P * N + Q * P * N + N * P * Q + Q * P * Q
                              + Q * N * Q + Q * N * P + Q * N * Q + Q * N * P)
    nbytes = 2 * B * L * H * P * 2 + 2 * B * L * G * N * 2 + B * L * H * 2
    cs_bytes = cs.numel() * 4
    # backward: x, dy, dx, B, C, dt, ddt (fp32), dB / dC (fp32 atomics), chunk states read
    nbytes_bwd = (3 * B * L * H * P * 2 + 2 * B * L * G * N * 2 + B * L * H * (2 + 4)
                  + 2 * B * L * G * N * 4 + cs_bytes)
    tf = flops / (ms * 1e-3) / 1e12
    tf_bwd = flops_bwd / (ms_bwd * 1e-3) / 1e12
    return {"workload": f"Mamba-2 SSD forward and backward, B{B} L{L} H{H} P{P} G{G} N{N} bf16, "
                        f"chunks of {Q}, tcgen05 bf16 products with fp32 TMEM accumulators",
            "ms": ms, "tokens_per_s": B * L / (ms * 1e-3), "tflops": tf,
            "tflops_issued": issued / (ms * 1e-3) / 1e12,
            "tensor_frac_of_peak": tf / pk["bf16_tflops"], "hbm_gbs": nbytes / (ms * 1e-3) / 1e9,
            "flops_per_call": flops, "bytes_per_call": nbytes,
            "fwd_saving_states_ms": ms_train, "chunk_states_bytes": cs_bytes,
            "bwd_ms": ms_bwd, "bwd_tflops": tf_bwd, "bwd_tensor_frac_of_peak": tf_bwd / pk["bf16_tflops"],
            "bwd_flops_per_call": flops_bwd, "bwd_hbm_gbs": nbytes_bwd / (ms_bwd * 1e-3) / 1e9,
            "train_tokens_per_s": B * L / ((ms_train + ms_bwd) * 1e-3),
            "launches": 3 * (reps + 2)}


def deterministic_bench(ly, bwd_ms, reps=5):
    """The scan backward with deterministic dB / dC (fixed-order sums of the
    channel groups' partials) on the bench layer, timed with CUDA events over
    `reps` launches after one warm-up, beside the atomic backward's time."""
    import torch
    import selective_state_space_35_b200 as ssm
    g = {k: torch.empty_like(v) for k, v in ly.g.items()}
    p = ssm.scan_params(ly.u, ly.delta, ly.A, ly.Bm, ly.Cm, z=ly.z, Dskip=ly.Dskip,
                        delta_bias=ly.dbias, seq_idx=ly.seq, n_splits=ly.n_splits, out=ly.out,
                        workspace=ly.ws)
    gr = ssm.ssm_scan_grads()
    gr.struct_size = ctypes.sizeof(ssm.ssm_scan_grads)
    gr.deterministic = 1
    nbytes = ssm.ssm_scan_bwd_workspace_size(p, gr)
    bws = torch.empty(nbytes, dtype=torch.uint8, device=ly.u.device)

    def run():
        ssm.scan_bwd(ly.u, ly.delta, ly.A, ly.Bm, ly.Cm, ly.dout, ly.ws, grads=g,
                     deterministic=True, bwd_workspace=bws, **ly.kw)

    run()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        run()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    same = all(torch.equal(g[k], ly.g[k]) for k in ("du", "ddelta", "dA", "dD"))
    del bws, g
    return {"ms_per_layer": ms, "atomic_ms_per_layer": bwd_ms, "cost": ms / bwd_ms - 1.0,
            "workspace_bytes": nbytes, "other_grads_bitwise_equal_to_atomic": same,
            "launches": (reps + 1) * 3}


def fused_fwd_bench(ly, sep_ms, reps=5):
    """The fused conv + SiLU + scan forward (ssm_conv1d_scan_fwd) on the bench
    layer, timed with CUDA events over `reps` launches after one warm-up,
    beside the separate conv1d + scan forward of the timed step, whose u and
    out it must reproduce bitwise."""
    import torch
    import selective_state_space_35_b200 as ssm
    u, out, ws = torch.empty_like(ly.u), torch.empty_like(ly.out), torch.empty_like(ly.ws)

    def run():
        ssm.conv1d_scan_fwd(ly.x, ly.w, ly.cb, ly.delta, ly.A, ly.Bm, ly.Cm, u=u, out=out,
                            workspace=ws, return_final_state=ly.shape.final_state, **ly.kw)

    run()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        run()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    same = bool(torch.equal(u, ly.u) and torch.equal(out, ly.out))
    del u, out, ws
    return {"ms_per_layer": ms, "separate_ms_per_layer": sep_ms, "gain": 1.0 - ms / sep_ms,
            "u_out_bitwise_equal_to_separate": same, "launches": (reps + 1) * 2}


def complex_bench(device, ly, pk, reps=5):
    """The scan with a complex diagonal A (S4D-Lin: A = -1/2 + i pi n) on the
    bench layer's shape and activations: B and C take (re, im) planes from the
    layer's own B and C. Forward and backward timed separately with CUDA
    events over `reps` launches each (inputs > L2)."""
    import torch
    import selective_state_space_35_b200 as ssm
    B, D, N, L = ly.shape.B, ly.shape.D, ly.shape.N, ly.shape.L
    Bc = torch.stack([ly.Bm, ly.Cm], dim=2).contiguous()
    Cc = torch.stack([ly.Cm, ly.Bm], dim=2).contiguous()
    A = torch.zeros((D, N, 2), dtype=torch.float32, device=device)
    A[..., 0] = -0.5
    A[..., 1] = torch.arange(N, dtype=torch.float32, device=device) * math.pi
    kw = dict(z=ly.z, Dskip=ly.Dskip, delta_bias=ly.dbias, seq_idx=ly.seq)
    out, _, ws = ssm.scan_fwd(ly.x, ly.delta, A, Bc, Cc, **kw)
    g = ssm.scan_bwd(ly.x, ly.delta, A, Bc, Cc, ly.dout, ws, **kw)
    torch.cuda.synchronize()

    # fwd and bwd alternate (so a profiler's launch filter sees one of each
    # per round); each is timed with its own events
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps + 1)]
    for e in ev:
        e[0].record()
        ssm.scan_fwd(ly.x, ly.delta, A, Bc, Cc, out=out, workspace=ws, **kw)
        e[1].record()
        ssm.scan_bwd(ly.x, ly.delta, A, Bc, Cc, ly.dout, ws, grads=g, **kw)
        e[2].record()
    torch.cuda.synchronize()
    fwd = sum(e[0].elapsed_time(e[1]) for e in ev[1:]) / reps   # the first pass warms up
    bwd = sum(e[1].elapsed_time(e[2]) for e in ev[1:]) / reps
    del ws, g, out
    return {"workload": f"complex diagonal A (S4D-Lin), B{B} x D{D} x N{N} x L{L}, bf16 "
                        "activations, fp32 complex state, fwd + bwd",
            "fwd_ms": fwd, "bwd_ms": bwd, "tokens_per_s": B * L / ((fwd + bwd) * 1e-3),
            "launches": 3 * (reps + 2)}


def cp_shard_bench(device, ly, ranks=8, reps=5):
    """One rank's compute when the bench layer's sequence is cut into `ranks`
    contiguous shards: the forward and backward summaries of its shard, the
    carry folds over all ranks' summaries, and the shard's scan forward and
    backward. It is timed on one GPU with CUDA events. The exchanges (a
    3-token halo each way, 2 x [B, D, N] fp32 summaries per rank and
    direction) are not part of it."""
    import torch
    import selective_state_space_35_b200 as ssm
    B, D, N, L = ly.shape.B, ly.shape.D, ly.shape.N, ly.shape.L
    Ls = L // ranks
    sl = lambda t: t[..., :Ls].contiguous()  # noqa: E731
    u, dl, z, go, Bm, Cm = (sl(t) for t in (ly.x, ly.delta, ly.z, ly.dout, ly.Bm, ly.Cm))
    kw = dict(z=z, Dskip=ly.Dskip, delta_bias=ly.dbias)
    h0 = torch.zeros((B, D, N), dtype=torch.float32, device=device)
    out, _, ws = ssm.scan_fwd(u, dl, ly.A, Bm, Cm, initial_state=h0, **kw)
    g = ssm.scan_bwd(u, dl, ly.A, Bm, Cm, go, ws, initial_state=h0, dfinal_state=h0, **kw)
    sws = torch.empty_like(ws)
    dec, end = ssm.scan_fwd_summary(u, dl, ly.A, Bm, delta_bias=ly.dbias, workspace=sws)
    stack = torch.stack([dec] * ranks).contiguous()
    vals = torch.stack([end] * ranks).contiguous()
    hin = torch.empty_like(h0)

    steps = {
        "fwd_summary": lambda: ssm.scan_fwd_summary(u, dl, ly.A, Bm, delta_bias=ly.dbias,
                                                    workspace=sws),
        "bwd_summary": lambda: ssm.scan_bwd_summary(dl, ly.A, Cm, go, z=z, delta_bias=ly.dbias,
                                                    workspace=sws),
        "carry_fwd": lambda: ssm.state_carry(stack, vals, ranks - 1, out=hin),
        "carry_bwd": lambda: ssm.state_carry(stack, vals, 0, reverse=True, out=hin),
        "scan_fwd": lambda: ssm.scan_fwd(u, dl, ly.A, Bm, Cm, out=out, workspace=ws,
                                         initial_state=hin, **kw),
        "scan_bwd": lambda: ssm.scan_bwd(u, dl, ly.A, Bm, Cm, go, ws, grads=g,
                                         initial_state=hin, dfinal_state=hin, **kw),
    }
    ms = {}
    for name, fn in steps.items():
        fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        ms[name] = e0.elapsed_time(e1) / reps
    rank_ms = sum(ms.values())
    del ws, sws, g, out
    return {"workload": f"one rank of {ranks}: B{B} x D{D} x N{N} x L{Ls} shard of the L{L} row, "
                        "bf16 activations, no L2 flush between repeats",
            "ms": ms, "rank_scan_ms": rank_ms,
            "overhead_vs_plain_shard": rank_ms / (ms["scan_fwd"] + ms["scan_bwd"]) - 1.0,
            "launches": 9 * (reps + 1) + 5}


def decode_bench(device, sh, pk, rows_b=2048, steps=200, graph_steps=50):
    """The recurrent one-token step at the bench layer's width: `rows_b`
    sequences x D channels x N states (bf16 activations, fp32 state). The
    state (rows_b*D*N*4 bytes, 201 MB at 2048 x 1536 x 16) exceeds the 126 MB
    L2, so every step reads and writes it in HBM. Timed two ways with CUDA
    events: back-to-back launches, and a CUDA graph of `graph_steps` steps
    (kernel time without launch gaps)."""
    import torch
    import selective_state_space_35_b200 as ssm
    D, N = sh.D, sh.N
    di = synth.decode_inputs(rows_b, D, N, 1, "bf16", synth.seed_for(9))

    def bf(t):
        return torch.from_numpy(t.bits.view(np.int16).copy()).view(torch.bfloat16).to(device)

    def f32(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)

    x, dl, z, Bm, Cm = bf(di.x)[0], bf(di.delta)[0], bf(di.z)[0], bf(di.Bm)[0], bf(di.Cm)[0]
    cs, st = bf(di.conv_state), f32(di.h0)
    A, w, cb, Dk, db = (f32(di.A), f32(di.conv_w), f32(di.conv_b), f32(di.Dskip),
                        f32(di.delta_bias))
    out = torch.empty_like(x)

    def step():
        ssm.decode_step(x, cs, w, dl, A, Bm, Cm, st, conv_bias=cb, z=z, Dskip=Dk,
                        delta_bias=db, out=out)

    for _ in range(20):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    us_launch = e0.elapsed_time(e1) / steps * 1e3
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(graph_steps):
            step()
    g.replay()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(4):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    us_graph = e0.elapsed_time(e1) / (4 * graph_steps) * 1e3
    del g
    e_sz, rows = 2, rows_b * D
    # state read + write; x, delta, z, out and the 3-token window read + write
    # per row; B and C per sequence; A, conv weight and bias, D, delta bias
    nbytes = (rows * N * 4 * 2 + rows * e_sz * 10 + rows_b * N * e_sz * 2 + D * N * 4
              + D * 4 * 4 + 3 * D * 4)
    gbs = nbytes / (us_graph * 1e-6) / 1e9
    return {"workload": f"recurrent step, {rows_b} sequences x D{D} x N{N}, bf16 activations, "
                        f"fp32 state ({rows * N * 4 / 1e6:.0f} MB > L2)",
            "us_per_step": us_launch, "us_per_step_graph": us_graph,
            "tokens_per_s": rows_b / (us_graph * 1e-6), "bytes_per_step": nbytes,
            "hbm_gbs": gbs, "hbm_frac_of_measured": gbs / pk["hbm_gbs"],
            "launches": steps + 20 + 5 * graph_steps}


def e2e(layers, device, args, world):
    """Whole step through the public API from pinned host memory: every step
    copies each layer's inputs in and its results out. Copies run on their
    own streams so that layer i's compute overlaps layer i+1's inputs and
    layer i-1's results (events keep each layer's buffers until their copies
    are done); the step is timed with CUDA events on the compute stream, after
    it has waited for the last copy out."""
    import torch
    import torch.distributed as dist
    bf = torch.bfloat16
    pinned_in = []
    for ly in layers:
        d = {}
        for k in ("x", "z", "delta", "Bm", "Cm", "dout"):
            t = torch.from_numpy(ly.host[k].bits.view(np.int16)).view(bf)
            d[k] = t.pin_memory()
        pinned_in.append(d)

    def outputs(ly):
        return {"out": ly.out, "dx": ly.dx, "ddelta": ly.g["ddelta"], "dz": ly.g["dz"],
                "dB": ly.g["dB"], "dC": ly.g["dC"], "dA": ly.g["dA"], "dD": ly.g["dD"],
                "ddelta_bias": ly.g["ddelta_bias"], "dconv_w": ly.dw, "dconv_b": ly.dcb}

    pinned_out = [{k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
                   for k, v in outputs(ly).items()} for ly in layers]
    h2d = sum(t.numel() * t.element_size() for d in pinned_in for t in d.values())
    d2h = sum(t.numel() * t.element_size() for d in pinned_out for t in d.values())

    comp = torch.cuda.current_stream(device)
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    in_free = [torch.cuda.Event() for _ in layers]    # compute of the layer is done
    out_free = [torch.cuda.Event() for _ in layers]   # the layer's results are copied out
    for e in in_free + out_free:
        e.record(comp)

    def step():
        for i, (ly, hin) in enumerate(zip(layers, pinned_in)):
            s_in.wait_event(in_free[i])  # the previous step has finished reading the inputs
            with torch.cuda.stream(s_in):
                for k, t in hin.items():
                    getattr(ly, k).copy_(t, non_blocking=True)
            ready = torch.cuda.Event()
            ready.record(s_in)
            comp.wait_event(ready)
            comp.wait_event(out_free[i])  # the previous step's results are out
            ly.step()
            in_free[i].record(comp)
            s_out.wait_event(in_free[i])
            with torch.cuda.stream(s_out):
                for k, t in outputs(ly).items():
                    pinned_out[i][k].copy_(t, non_blocking=True)
            out_free[i].record(s_out)

    step()
    torch.cuda.synchronize()
    n = max(1, args.e2e_steps)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    a.record(comp)
    s_in.wait_event(a)
    for _ in range(n):
        step()
    comp.wait_event(out_free[-1])
    b.record(comp)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    if world > 1:
        t = torch.tensor([ms], device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    sh = layers[0].shape
    tokens = world * len(layers) * sh.B * sh.L
    return {"value": tokens / (ms / n * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n, "ms_per_step": ms / n,
            "copies": "inputs in and results out every step, overlapped with compute on two "
                      "copy streams"}


if __name__ == "__main__":
    sys.exit(main())
