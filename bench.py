#!/usr/bin/env python
"""Benchmark of the Flash EQ-Linear hot path on B200.

One step = the whole path for every layer of the workload: weight
pre-transform (the DFT of W along the group axis), forward, input gradient
and weight/bias gradient.  The default workload is p4 (T=4) EQ-ViT-B MLP
shapes in bf16: fc1 768->3072 and fc2 3072->768 over 64 images x 197 tokens.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 every rank processes its own batch (weak scaling) and the dW/db
gradients are summed over ranks with NCCL, the data-parallel exchange of the
backward pass.  Launched by torch.distributed.run, each rank reads its
RANK / LOCAL_RANK / WORLD_SIZE from the environment; launched directly with
--gpus N > 1, the script starts the N local ranks itself.  Rank 0 prints one
JSON line.

Regions timed with CUDA events on the launching streams:
  * the headline: exactly K whole steps, nothing else in between;
  * per kernel: each (layer, pass) call launched back to back on its own, for
    the roofline of the dominant kernel and the per-call breakdown;
  * sub-measurements on other workloads of the same path (the p4 FP16 forward
    at EQ-ViT-B shapes, the EQ-Swin-T stage-1 step, the T=8 FP16 layer), each
    with its own roofline fractions;
  * end to end: the same step through the public API with the inputs copied
    from pinned host memory and the results copied back every step.

`--impl reference` times the CPU oracle (plain loops over the layer's
definition, double precision) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import platform
import socket
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from group_circulant_linear_b200 import dp, inputs, workloads  # noqa: E402

METRIC = "EQ-Linear p4 fwd+bwd TFLOP/s (dense-equiv) & fraction of tensor-pipe roofline"
UNIT = "TFLOP/s"
N_SETS = 3        # rotating input sets, together larger than the 126 MB L2
KERNEL_REPS = 50  # back-to-back launches per (layer, pass) in the per-kernel region


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=workloads.DEFAULT_BENCH, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sub", action="store_true", help="skip the sub-measurements")
    ap.add_argument("--path", choices=("fused", "plain"), default="plain",
                    help="fused: forward and dx stash the spectra, dW from the spectra; "
                         "plain: dW transforms x and gy itself")
    ap.add_argument("--order", choices=("layer", "training"), default="layer",
                    help="layer: each layer's forward and backward in turn; training: every forward, "
                         "then the backward passes in reverse layer order")
    ap.add_argument("--tail-split", action="store_true",
                    help="switch the forward / dx tail split on for every layer (eqlin_set_tail_split)")
    return ap.parse_args(argv)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16": float(d["bf16_tflops"]),
                "bf16_sustained": float(d["bf16_tflops_sustained"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


def dense_flop_step(layers):
    """Dense-equivalent FLOP of one step: 2*N*C*D for each pass of each layer."""
    return sum(L.dense_flop() * len(L.passes) for L in layers)


def cpu_info() -> dict:
    model = platform.processor() or ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count()}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of one GPU, read line by line on a background thread.

    Samples are kept only while `active` is set (the timed regions); the
    summary takes the samples drawn under load (power at least half of the
    maximum seen) for the median SM clock and the throttle reasons."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device: int, period_ms: int = 100):
        self.rows, self.active, self.error = [], False, None
        self.proc = self.thread = None
        try:
            gid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            gid = str(device)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits",
                 "-lms", str(period_ms), "-i", gid], stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                text=True, bufsize=1)
        except Exception as e:  # reported in the summary
            self.error = f"nvidia-smi did not start: {e}"
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            if not self.active:
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                self.rows.append((float(parts[0]), float(parts[1]), float(parts[2]), parts[4:]))
            except ValueError:
                continue

    def stop(self) -> dict:
        self.active = False
        if self.proc is None:
            return {"sm_mhz": None, "samples": 0, "note": self.error}
        self.proc.terminate()
        try:
            _, err = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            err = ""
        if self.thread is not None:
            self.thread.join(timeout=5)
        rows = list(self.rows)
        if not rows:
            return {"sm_mhz": None, "samples": 0,
                    "note": "no nvidia-smi samples during the timed regions" + (f": {err.strip()[:200]}" if err else "")}
        pmax = max(r[2] for r in rows)
        loaded = [r for r in rows if r[2] >= 0.5 * pmax] or rows
        reasons = sorted({self.REASONS[i] for r in loaded for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(loaded), "power_w_max": pmax}


# --------------------------------------------------------------- CPU oracle
def oracle_data(layers, seed: int = 0):
    """The workload's seeded inputs, as the float64 arrays the oracle reads."""
    data = []
    for L in layers:
        inp = inputs.make_inputs(L.T, L.Cp, L.Dp, L.N, L.dtype, seed=seed)
        data.append({k: v.double().numpy() for k, v in inp.items()})
    return data


_RATES = {}


def _oracle_rates(layers, data):
    """The oracle's rates (dense-equivalent FLOP/s) for token rows and for
    weight pairs, measured once per process on a probe that gives each of its
    threads a few rows / pairs, as the samples will."""
    import numpy as np

    import oracle
    L0, d0 = layers[0], data[0]
    key = (L0.T, L0.Cp, L0.Dp, L0.N)
    if key not in _RATES:
        per_thread = 4 * oracle.threads()
        probe = min(per_thread, L0.N)
        t = time.perf_counter()
        oracle.forward(d0["x"], d0["W"], d0["b"], rows=np.arange(probe))
        row_rate = probe * 2 * L0.C * L0.D / max(time.perf_counter() - t, 1e-6)
        t = time.perf_counter()
        oracle.backward_dw(d0["x"], d0["gy"], L0.T, L0.Cp, L0.Dp, pairs=[[0, 0]] * per_thread, want_db=False)
        dw_rate = per_thread * L0.T * 2 * L0.N * L0.T / max(time.perf_counter() - t, 1e-6)
        _RATES[key] = (row_rate, dw_rate)
    return _RATES[key]


def oracle_sample(layers, data, budget_s: float, seed: int = 0):
    """Time the oracle on a bounded sample of every layer's fwd, dx and dW work.

    Returns (dense-equivalent FLOP done, seconds, threads, description)."""
    import numpy as np

    import oracle
    oracle.build()
    row_rate, dw_rate = _oracle_rates(layers, data)
    done, desc, t_total = 0, [], 0.0
    for L, d in zip(layers, data):
        share_s = budget_s / (len(layers) * len(L.passes))     # seconds per pass
        rows = max(1, min(L.N, int(share_s * row_rate / (2 * L.C * L.D))))
        sel = np.linspace(0, L.N - 1, rows).astype(np.int64)
        pairs_n = max(1, min(L.Dp * L.Cp, int(share_s * dw_rate / (2 * L.N * L.T * L.T))))
        rng = np.random.default_rng(seed)
        pairs = np.stack([rng.integers(0, L.Dp, pairs_n), rng.integers(0, L.Cp, pairs_n)], 1)
        t = time.perf_counter()
        if "fwd" in L.passes:
            oracle.forward(d["x"], d["W"], d["b"], rows=sel)
            done += rows * 2 * L.C * L.D
        if "dx" in L.passes:
            oracle.backward_dx(d["gy"], d["W"], rows=sel)
            done += rows * 2 * L.C * L.D
        if "dw" in L.passes:
            oracle.backward_dw(d["x"], d["gy"], L.T, L.Cp, L.Dp, pairs=pairs, want_db=False)
            done += pairs_n * L.T * 2 * L.N * L.T
        t_total += time.perf_counter() - t
        desc.append(f"{L.name}: {rows} of {L.N} token rows (fwd, dx), {pairs_n} of {L.Dp * L.Cp} "
                    f"(d,c) weight pairs over all tokens (dW)")
    return done, t_total, oracle.threads(), "; ".join(desc)


def run_reference(args, layers, rank):
    if rank != 0:
        return
    # each step is a bounded sample; the whole run stays within ~2 minutes
    per_step = max(0.05, min(10.0, 120.0 / max(1, args.steps + args.warmup)))
    data = oracle_data(layers)
    for _ in range(args.warmup):
        oracle_sample(layers, data, per_step)
    flop = secs = 0.0
    desc, threads = "", 1
    for _ in range(args.steps):
        f, s, threads, desc = oracle_sample(layers, data, per_step)
        flop += f
        secs += s
    value = flop / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": args.workload,
                   "layers": [dict(name=L.name, T=L.T, Cp=L.Cp, Dp=L.Dp, N=L.N) for L in layers]},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": "per step: " + desc, **cpu_info()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------- roofline
def kernel_src_sha(name: str) -> str:
    path = os.path.join(ROOT, "group_circulant_linear_b200", "csrc", name)
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def profiled_traffic(kernel_key: str):
    """DRAM bytes per launch from a committed ncu summary, if every source it
    was taken on is unchanged; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[kernel_key]
        if [kernel_src_sha(s) for s in e["srcs"]] == list(e["src_sha"]):
            return float(e["bytes_per_launch"])
    except Exception:
        pass
    return None


def pass_work(L, kind, fused=False):
    """(actual FLOP, algorithmic bytes) of one call of a pass.  The stash forms
    (fused path) also write the input's spectrum, as many elements as the input."""
    if kind == "set_weights":
        return 0, L.Dp * L.Cp * L.T * 2 * 2
    if kind == "fwd_gauss":
        # the three-product form: per complex frequency 3 real GEMMs, not 4
        R = workloads.real_gemms(L.T)
        n_complex = (L.T - 1) // 2
        return L.actual_flop() * (R - n_complex) // R, L.bytes_fwd()
    e = workloads.BYTES[L.dtype]
    extra = 0
    if fused and kind == "fwd":
        extra = L.N * L.C * e
    elif fused and kind == "dx":
        extra = L.N * L.D * e
    return L.actual_flop(), (L.bytes_dw() if kind == "dw" else L.bytes_fwd()) + extra


def roofline_of(L, kind, us, pk, fused=False):
    """Roofline of one call of `kind` on layer L that took `us` microseconds.

    The bound is the resource the call's arithmetic intensity points at:
    tensor when its FLOP per algorithmic byte reach half the measured ridge
    (dense bf16 peak / copy bandwidth), else HBM.  Calls timed in sub-second
    regions use the burst tensor peak (FP16 and BF16 have the same nominal
    rate).  `frac_roofline` = max(FLOP / tensor peak, bytes / HBM) / time."""
    flop, byt = pass_work(L, kind, fused)
    t = us * 1e-6
    tens = pk["bf16"] * 1e12
    hbm = pk["hbm_gbs"] * 1e9
    r = {"us": round(us, 2), "tflops": flop / t / 1e12 if flop else 0.0, "gbs": byt / t / 1e9,
         "frac_tensor": flop / t / tens if flop else 0.0, "frac_hbm": byt / t / hbm,
         "frac_roofline": max(flop / tens, byt / hbm) / t}
    if L.dtype == "f32" and (L.T in (1, 2, 4) or (L.T == 8 and kind in ("fwd", "dx"))) and kind != "set_weights":
        # 3xTF32: three kind::tf32 MMAs per real product, against the TF32
        # peak (the measured bf16 peak x the nominal TF32/BF16 ratio of 1/2)
        mma_flop, peak = 3 * flop, pk["bf16"] / 2
        r.update(bound="tensor", achieved=mma_flop / t / 1e12, peak=peak, unit="TFLOP/s (tf32 MMA)",
                 frac=mma_flop / t / (peak * 1e12), fp32_equiv_tflops=r["tflops"],
                 frac_hbm=byt / t / hbm)
        r["frac_roofline"] = max(mma_flop / (peak * 1e12), byt / hbm) / t
    elif L.dtype == "f32":
        # FP32 on the CUDA cores: FFMA peak 148 SMs x 128 lanes x 2 x 1965 MHz (nominal)
        ffma = 148 * 128 * 2 * 1.965e9
        r.update(bound="alu", achieved=r["tflops"], peak=ffma / 1e12, unit="TFLOP/s (FFMA)",
                 frac=flop / t / ffma)
        r["frac_roofline"] = max(flop / ffma, byt / hbm) / t
    else:
        ridge = tens / hbm
        if flop and flop / byt >= ridge / 2:
            r.update(bound="tensor", achieved=r["tflops"], peak=pk["bf16"], unit="TFLOP/s", frac=r["frac_tensor"])
        else:
            r.update(bound="hbm", achieved=r["gbs"], peak=pk["hbm_gbs"], unit="GB/s", frac=r["frac_hbm"])
    r["intensity_flop_per_byte"] = flop / byt
    return r


# ----------------------------------------------------------------- our arm
class Layers:
    """Device state of a workload's layers: handles, weights, rotating input sets, outputs.

    fused: forward and dx are the stash forms (they also write the spectra
    X = DFT(x) and G = DFT(gy)) and dW/db come from the spectra; otherwise
    dW/db transform x and gy themselves."""

    def __init__(self, layers, dev, rank, seed_base=0, fused=True, tail_split=False):
        from group_circulant_linear_b200 import eqlin
        self.eqlin = eqlin
        self.layers = layers
        self.fused = fused
        self.st = []
        for li, L in enumerate(layers):
            dt = inputs.DTYPES[L.dtype]
            w = inputs.make_inputs(L.T, L.Cp, L.Dp, 1, L.dtype, seed=seed_base + 1000 + li, with_gy=False,
                                   device=dev)
            sets = [inputs.make_inputs(L.T, L.Cp, L.Dp, L.N, L.dtype, seed=seed_base + 17 * rank + 100 * li + s,
                                       with_gy=("dx" in L.passes or "dw" in L.passes), device=dev)
                    for s in range(N_SETS)]
            h = eqlin.create(L.T, L.Cp, L.Dp, dt)
            if tail_split:
                eqlin.set_tail_split(h, True)
            entry = dict(L=L, h=h, W=w["W"], b=w["b"], sets=sets,
                         y=torch.empty((L.N, L.D), dtype=dt, device=dev),
                         dx=torch.empty((L.N, L.C), dtype=dt, device=dev),
                         dW=torch.empty((L.Dp, L.Cp, L.T), dtype=torch.float32, device=dev),
                         db=torch.empty((L.Dp,), dtype=torch.float32, device=dev))
            if fused:
                # one spectra pair per input set: dW of set i reads what the
                # stash forms wrote for set i
                entry["xs"] = [eqlin.empty_spectra(h, "x", L.N, device=dev) for _ in range(N_SETS)]
                entry["gs"] = [eqlin.empty_spectra(h, "gy", L.N, device=dev) for _ in range(N_SETS)]
            # weights loaded once here; a step also reloads them (set_weights is part of the step)
            eqlin.set_weights(h, entry["W"], entry["b"])
            self.st.append(entry)

    def set_bytes(self):
        return sum(sum(t.numel() * t.element_size() for t in s["sets"][0].values()) for s in self.st)

    def call(self, s, kind, i, stream=None):
        e, j = self.eqlin, i % N_SETS
        inp = s["sets"][j]
        if kind == "set_weights":
            e.set_weights(s["h"], s["W"], s["b"], stream)
        elif kind == "fwd_gauss":
            e.forward_gauss(s["h"], inp["x"], s["y"], stream)
        elif kind == "fwd":
            if self.fused:
                e.forward_stash(s["h"], inp["x"], s["y"], s["xs"][j], stream)
            else:
                e.forward(s["h"], inp["x"], s["y"], stream)
        elif kind == "dx":
            if self.fused:
                e.backward_dx_stash(s["h"], inp["gy"], s["dx"], s["gs"][j], stream)
            else:
                e.backward_dx(s["h"], inp["gy"], s["dx"], stream)
        elif self.fused:
            e.backward_dw_spectra(s["h"], s["xs"][j], s["gs"][j], s["L"].N, s["dW"], s["db"], stream)
        else:
            e.backward_dw(s["h"], inp["x"], inp["gy"], s["dW"], s["db"], stream)

    def errors(self):
        return [self.eqlin.get_error(s["h"]) for s in self.st]

    def close(self):
        for s in self.st:
            s["h"].close()


def time_calls(state, li, kind, reps, stream):
    """Average microseconds of one (layer, pass) call, `reps` launches back to
    back between two events on the launching stream (inputs rotate)."""
    s = state.st[li]
    for i in range(3):
        state.call(s, kind, i, stream)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(reps):
        state.call(s, kind, i, stream)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps * 1e3


def sub_measurements(dev, pk, reps, fused):
    """The same path on other workload shapes, each call timed on its own."""
    out = {}
    vit_b_f16 = [workloads.Layer(L.name + " f16", L.T, L.Cp, L.Dp, L.N, "f16", ("fwd",))
                 for L in workloads.WORKLOADS["eq-vit-b-mlp-bf16-fwdbwd"]]
    t8 = [L for L in workloads.WORKLOADS["cyclic-sweep-fwdbwd"] if L.T == 8 and L.dtype == "f16"]
    f32 = [L for L in workloads.WORKLOADS["cyclic-sweep-fwdbwd"] if L.dtype == "f32"]
    # the orders with sqrt(3)/2 twiddles, at the sweep's N and about its width (C = C'T near 1024)
    t36 = [workloads.Layer(f"cyclic T={T} f16", T, C, C, 16384, "f16", ("fwd", "dx", "dw"))
           for T, C in ((3, 336), (6, 168))]
    gauss = [workloads.Layer(L.name + " f16", L.T, L.Cp, L.Dp, L.N, "f16", ("fwd", "fwd_gauss"))
             for L in workloads.WORKLOADS["eq-vit-b-mlp-bf16-fwdbwd"]]
    subs = {
        "p4 FP16 forward, EQ-ViT-B MLP shapes": vit_b_f16,
        # the complex products as four real GEMMs (fwd) or three (fwd_gauss, tiles of <= 96 channels)
        "p4 FP16 forward, four- against three-product complex products": gauss,
        "EQ-Swin-T stage-1 step (f16)": workloads.WORKLOADS["eq-swin-t-s1-f16-fwdbwd"],
        "cyclic T=8 f16 layer": t8,
        "cyclic T=3 and T=6 f16 layers": t36,
        # FP32: every pass on 3xTF32 tensor cores for T = 2, 4; T = 8's
        # forward and dx on them, its dW on the CUDA cores
        "cyclic FP32 layers (3xTF32)": f32,
    }
    stream = torch.cuda.current_stream()
    for name, layers in subs.items():
        f = fused and "dw" in layers[0].passes
        state = Layers(layers, dev, 0, seed_base=5000, fused=f)
        rows, tot_us, dense = [], 0.0, 0
        for li, L in enumerate(layers):
            for kind in L.passes:
                us = time_calls(state, li, kind, reps, stream)
                rows.append({"layer": L.name, "pass": kind, **roofline_of(L, kind, us, pk, f)})
                tot_us += us
                dense += L.dense_flop()
        assert all(e == 0 for e in state.errors()), f"device-side timeout in {name}"
        state.close()
        del state
        torch.cuda.empty_cache()
        out[name] = {"calls": rows, "dense_tflops": dense / (tot_us * 1e-6) / 1e12,
                     "us_sum": round(tot_us, 2), "path": "fused" if f else "plain"}
    return out


def main(argv=None):
    args = parse(argv)
    layers = workloads.WORKLOADS[args.workload]
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ and args.impl == "ours":
        launch_local(args.gpus, argv if argv is not None else sys.argv[1:])
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = world > 1
    if args.impl == "reference":
        run_reference(args, layers, rank)     # rank 0 only; no GPU, no process group
        return
    if dist:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    fused = args.path == "fused"
    state = Layers(layers, dev, rank, fused=fused, tail_split=args.tail_split)
    eqlin = state.eqlin
    st = state.st

    # A step runs every layer's weight transform, forward, dx and dW/db:
    # layer by layer (--order layer), or every forward first and then the
    # backward passes in reverse layer order (--order training).  dW/db of a
    # layer runs on a second stream.  Plain path: it reads the same inputs as
    # dx and writes nothing dx reads, so it starts beside that dx.  Fused path:
    # it reads the spectrum its dx writes, so it starts after that dx and runs
    # beside what follows on the main stream.  The main stream waits for it
    # before each step ends (and before an all-reduce of dW/db).
    side = torch.cuda.Stream(device=dev)

    def backward(s, i):
        if not fused:
            side.wait_stream(stream)
        state.call(s, "dx", i)
        if fused:
            side.wait_stream(stream)
        state.call(s, "dw", i, stream=side)
        if dist:
            stream.wait_stream(side)
            dp.allreduce_grads((s["dW"], s["db"]))

    def step(i):
        if args.order == "layer":
            for s in st:
                state.call(s, "set_weights", i)
                state.call(s, "fwd", i)
                backward(s, i)
        else:
            for s in st:
                state.call(s, "set_weights", i)
                state.call(s, "fwd", i)
            for s in reversed(st):
                backward(s, i)
        stream.wait_stream(side)

    def barrier():
        if dist:
            torch.distributed.barrier()

    clocks = ClockSampler(local)
    clocks.active = True
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    n0 = eqlin.launch_count()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(i)
    t1.record(stream)
    torch.cuda.synchronize()
    launches = eqlin.launch_count() - n0
    barrier()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    if dist:
        tt = torch.tensor([ms], device=dev)
        torch.distributed.all_reduce(tt, op=torch.distributed.ReduceOp.MAX)
        ms = float(tt.item())
    assert all(e == 0 for e in state.errors()), "device-side timeout in the timed region"
    ms_per_step = ms / args.steps
    flop_step = dense_flop_step(layers)
    value = flop_step * world / (ms_per_step * 1e-3) / 1e12

    # ---------------------------------------------- per-kernel roofline
    pk = peaks()
    per = {}
    for li, L in enumerate(layers):
        for kind in ("set_weights",) + tuple(L.passes):
            per[(li, kind)] = time_calls(state, li, kind, KERNEL_REPS, stream)
    # the same forward / dx calls with the opt-in tail split (eqlin_set_tail_split):
    # shorter lone calls where the last wave of tiles would leave SMs idle
    split_us = {}
    if not args.no_sub and not args.tail_split:
        for li, L in enumerate(layers):
            h = state.st[li]["h"]
            state.eqlin.set_tail_split(h, True)
            for kind in (k for k in L.passes if k in ("fwd", "dx")):
                split_us[f"{L.name}/{kind}"] = round(time_calls(state, li, kind, KERNEL_REPS, stream), 2)
            state.eqlin.set_tail_split(h, False)
    clk = clocks.stop()
    assert all(e == 0 for e in state.errors()), "device-side timeout in the per-kernel region"
    dom = max(per, key=per.get)
    Ld = layers[dom[0]]
    roof = roofline_of(Ld, dom[1], per[dom], pk, fused)
    apply_k = "tc_apply_stash" if fused else "tc_apply"
    kernel_of = {"fwd": apply_k, "dx": apply_k, "dw": "dws" if fused else "dw", "set_weights": "pretransform"}
    key = f"{kernel_of[dom[1]]}:{Ld.name}:{dom[1]}"
    roof["kernel"] = key
    roof["peak_kind"] = (f"{pk['source']} " + ("bf16 dense, burst (call timed in a sub-second region)"
                                               if roof["bound"] == "tensor" else "HBM copy"))
    roof["traffic"] = profiled_traffic(key)
    breakdown = {f"{layers[li].name}/{kind}": round(us, 2) for (li, kind), us in per.items()}
    per_call = {f"{layers[li].name}/{kind}": roofline_of(layers[li], kind, us, pk, fused)
                for (li, kind), us in per.items() if kind != "set_weights"}

    # ---------------------------------------------------------- e2e
    e2e = None
    if not args.no_e2e:
        host = []
        for s in st:
            inp = s["sets"][0]
            host.append({k: v.cpu().pin_memory() for k, v in
                         (("x", inp["x"]), ("gy", inp["gy"]), ("W", s["W"]), ("b", s["b"]))})
            host[-1].update({k: torch.empty(s[k].shape, dtype=s[k].dtype, pin_memory=True)
                             for k in ("y", "dx", "dW", "db")})
        dbuf = [{k: torch.empty_like(s["sets"][0][k]) for k in ("x", "gy")} for s in st]
        h2d = sum(host[i][k].numel() * host[i][k].element_size() for i in range(len(st)) for k in ("x", "gy", "W", "b"))
        d2h = sum(host[i][k].numel() * host[i][k].element_size() for i in range(len(st)) for k in ("y", "dx", "dW", "db"))
        # Host->device copies of every layer's inputs on an upload stream,
        # kernels on the main streams, device->host copies of each layer's
        # results on a download stream, so that both copy directions and the
        # kernels overlap.  A layer's input buffers are overwritten (next step)
        # only after its kernels have read them, and its outputs only after
        # their copies have run.
        h2d_stream = torch.cuda.Stream(device=dev)
        d2h_stream = torch.cuda.Stream(device=dev)
        copied = [None] * len(st)
        consumed = [None] * len(st)

        def e2e_step():
            uploaded = []
            for i, s in enumerate(st):
                hb, db_ = host[i], dbuf[i]
                with torch.cuda.stream(h2d_stream):
                    if consumed[i] is not None:
                        h2d_stream.wait_event(consumed[i])
                    db_["x"].copy_(hb["x"], non_blocking=True)
                    db_["gy"].copy_(hb["gy"], non_blocking=True)
                    s["W"].copy_(hb["W"], non_blocking=True)
                    s["b"].copy_(hb["b"], non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(h2d_stream)
                    uploaded.append(ev)
            for i, s in enumerate(st):
                hb, db_ = host[i], dbuf[i]
                stream.wait_event(uploaded[i])
                if copied[i] is not None:
                    stream.wait_event(copied[i])
                eqlin.set_weights(s["h"], s["W"], s["b"])
                if fused:
                    eqlin.forward_stash(s["h"], db_["x"], s["y"], s["xs"][0])
                    eqlin.backward(s["h"], db_["gy"], s["xs"][0], s["dx"], s["gs"][0], s["dW"], s["db"])
                else:
                    eqlin.forward(s["h"], db_["x"], s["y"])
                    side.wait_stream(stream)
                    eqlin.backward_dx(s["h"], db_["gy"], s["dx"])
                    eqlin.backward_dw(s["h"], db_["x"], db_["gy"], s["dW"], s["db"], stream=side)
                    stream.wait_stream(side)
                if dist:
                    dp.allreduce_grads((s["dW"], s["db"]))
                consumed[i] = torch.cuda.Event()
                consumed[i].record(stream)
                d2h_stream.wait_stream(stream)
                with torch.cuda.stream(d2h_stream):
                    for k in ("y", "dx", "dW", "db"):
                        hb[k].copy_(s[k], non_blocking=True)
                    copied[i] = torch.cuda.Event()
                    copied[i].record(d2h_stream)

        ke = max(3, min(args.steps, 30))
        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(ke):
            e2e_step()
        stream.wait_stream(d2h_stream)      # the last results are on the host
        stream.wait_stream(h2d_stream)
        b.record(stream)
        torch.cuda.synchronize()
        ems = a.elapsed_time(b) / ke
        if dist:
            tt = torch.tensor([ems], device=dev)
            torch.distributed.all_reduce(tt, op=torch.distributed.ReduceOp.MAX)
            ems = float(tt.item())
        e2e = {"value": flop_step * world / (ems * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ems}

    set_bytes = state.set_bytes()
    config = {
        "workload": args.workload,
        "layers": [dict(name=L.name, T=L.T, Cp=L.Cp, Dp=L.Dp, N=L.N, passes=list(L.passes)) for L in layers],
        "path": args.path,
        "order": args.order,
        "tail_split": args.tail_split,
        "step": ("per layer: set_weights (weight DFT), forward"
                 + (" writing X = DFT(x)" if fused else "")
                 + ", dx" + (" writing G = DFT(gy)" if fused else "")
                 + ", dW/db" + (" from the spectra, after dx" if fused else " transforming x and gy, beside dx")
                 + " on a second stream; "
                 + ("layer by layer" if args.order == "layer"
                    else "every forward first, then the backward passes in reverse layer order")
                 + (" + NCCL all-reduce of dW/db" if dist else "")),
        "tokens_per_gpu": layers[0].N,
        "l2": f"inputs rotate over {N_SETS} sets of {set_bytes / 1e6:.0f} MB each "
              f"({N_SETS * set_bytes / 1e6:.0f} MB > 126 MB L2)",
        "actual_tflops": sum(L.actual_flop() * len(L.passes) for L in layers) * world
                         / (ms_per_step * 1e-3) / 1e12,
        "kernel_us": breakdown,
        "per_call_roofline": per_call,
        "kernel_us_sampling": f"CUDA events around {KERNEL_REPS} back-to-back launches of each call, "
                              "after the headline region",
        "kernel_us_tail_split": split_us or None,
    }
    state.close()
    del state, st
    torch.cuda.empty_cache()

    sub = None
    if rank == 0 and not args.no_sub:
        sub = sub_measurements(dev, pk, KERNEL_REPS, fused)

    # ---------------------------------------------------- CPU baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f, secs, threads, desc = oracle_sample(layers, oracle_data(layers), budget_s=12.0)
        cpu = {"value": f / secs / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": desc, "seconds": secs, **cpu_info()}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": layers[0].dtype, "data": "synthetic",
            "config": config,
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk,
            "sub": sub,
        }
        print(json.dumps(line), flush=True)
    if dist:
        torch.distributed.destroy_process_group()


# ----------------------------------------------------- local multi-rank launch
def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_env(rank: int, world: int, port: int) -> dict:
    """Environment of local rank `rank` of `world` on this node (torchrun's variables)."""
    return {"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
            "LOCAL_WORLD_SIZE": str(world), "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)}


def _rank_entry(rank, world, port, target, argv):
    os.environ.update(rank_env(rank, world, port))
    target(argv)


def launch_local(world: int, argv, target=None):
    """Start `world` local ranks (one process per GPU) and wait for them; a
    rank that fails makes this raise."""
    import torch.multiprocessing as mp
    port = free_port()
    mp.start_processes(_rank_entry, args=(world, port, target or main, list(argv)), nprocs=world,
                       join=True, start_method="spawn")


if __name__ == "__main__":
    main()
