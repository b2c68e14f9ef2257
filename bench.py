#!/usr/bin/env python
"""Benchmark of the Flash EQ-Linear hot path on B200.

One step = the whole path for every layer of the workload: weight
pre-transform (the DFT of W along the group axis), forward, input gradient
and weight/bias gradient.  The default workload is p4 (T=4) EQ-ViT-B MLP
shapes in bf16: fc1 768->3072 and fc2 3072->768 over 64 images x 197 tokens.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torch.distributed.run) every rank processes its own
batch (weak scaling) and the dW/db gradients are summed over ranks with NCCL,
the data-parallel exchange of the backward pass.  Rank 0 prints one JSON line.

`--impl reference` times the CPU oracle (plain loops over the layer's
definition, double precision) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from group_circulant_linear_b200 import dp, inputs, workloads  # noqa: E402

METRIC = "EQ-Linear p4 fwd+bwd TFLOP/s (dense-equiv) & fraction of tensor-pipe roofline"
UNIT = "TFLOP/s"
N_SETS = 3   # rotating input sets, together larger than the 126 MB L2
REC_EVERY = 8   # timed steps per step with per-call events (kernel_ms, roofline)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=workloads.DEFAULT_BENCH, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


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


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device: int):
        self.proc = None
        try:
            props = torch.cuda.get_device_properties(device)
            gid = "GPU-" + str(props.uuid)
        except Exception:
            gid = str(device)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", gid], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            return None
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), float(parts[2]), parts[3:]))
            except ValueError:
                continue
        if not rows:
            return None
        pmax = max(r[2] for r in rows)
        loaded = [r for r in rows if r[2] >= 0.5 * pmax] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3][1:]) if v.lower() == "active"})
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
                         "sample": "per step: " + desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- our arm
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


def main():
    args = parse()
    layers = workloads.WORKLOADS[args.workload]
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

    from group_circulant_linear_b200 import eqlin
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    # ------------------------------------------------------------ state
    st = []
    for li, L in enumerate(layers):
        dt = inputs.DTYPES[L.dtype]
        w = inputs.make_inputs(L.T, L.Cp, L.Dp, 1, L.dtype, seed=1000 + li, with_gy=False, device=dev)
        sets = [inputs.make_inputs(L.T, L.Cp, L.Dp, L.N, L.dtype, seed=17 * rank + 100 * li + s,
                                   device=dev) for s in range(N_SETS)]
        h = eqlin.create(L.T, L.Cp, L.Dp, dt)
        st.append(dict(L=L, h=h, W=w["W"], b=w["b"], sets=sets,
                       y=torch.empty((L.N, L.D), dtype=dt, device=dev),
                       dx=torch.empty((L.N, L.C), dtype=dt, device=dev),
                       dW=torch.empty((L.Dp, L.Cp, L.T), dtype=torch.float32, device=dev),
                       db=torch.empty((L.Dp,), dtype=torch.float32, device=dev)))

    kinds = ("set_weights", "fwd", "dx", "dw")
    ev_log = []   # (layer index, kind, start event, end event) during the timed region

    # A layer's dW/db and its dx read the same inputs and write nothing the
    # other reads, so dW/db runs on a second stream: its CTAs take the SMs
    # that dx's last, partial wave leaves idle.  The main stream waits for it
    # before each step ends (and before an all-reduce of dW/db).
    side = torch.cuda.Stream(device=dev)

    def step(i, record=False):
        for li, s in enumerate(st):
            inp = s["sets"][i % N_SETS]
            calls = (
                ("set_weights", lambda: eqlin.set_weights(s["h"], s["W"], s["b"])),
                ("fwd", lambda: eqlin.forward(s["h"], inp["x"], s["y"])),
                ("dx", lambda: eqlin.backward_dx(s["h"], inp["gy"], s["dx"])),
                ("dw", lambda: eqlin.backward_dw(s["h"], inp["x"], inp["gy"], s["dW"], s["db"])),
            )
            if record:
                # every call on the main stream, one after another, each
                # between two events: the per-call times
                for kind, fn in calls:
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    fn()
                    e1.record(stream)
                    ev_log.append((li, kind, e0, e1))
            else:
                calls[0][1]()
                calls[1][1]()
                side.wait_stream(stream)
                calls[2][1]()
                eqlin.backward_dw(s["h"], inp["x"], inp["gy"], s["dW"], s["db"], stream=side)
            if dist:
                stream.wait_stream(side)
                dp.allreduce_grads((s["dW"], s["db"]))
        stream.wait_stream(side)

    def barrier():
        if dist:
            torch.distributed.barrier()

    clocks = ClockSampler(local)
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    n0 = eqlin.launch_count()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    # per-call events on every REC_EVERY-th step only: an event between two
    # kernels keeps the second from starting its prologue under the first's tail
    for i in range(args.steps):
        step(i, record=(i % REC_EVERY == 0))
    t1.record(stream)
    torch.cuda.synchronize()
    launches = eqlin.launch_count() - n0
    barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = t0.elapsed_time(t1)
    if dist:
        tt = torch.tensor([ms], device=dev)
        torch.distributed.all_reduce(tt, op=torch.distributed.ReduceOp.MAX)
        ms = float(tt.item())
    for s in st:
        assert eqlin.get_error(s["h"]) == 0, "device-side timeout in the timed region"
    ms_per_step = ms / args.steps
    flop_step = dense_flop_step(layers)
    value = flop_step * world / (ms_per_step * 1e-3) / 1e12

    # ---------------------------------------------- per-kernel roofline
    per = {}
    for li, kind, e0, e1 in ev_log:
        per.setdefault((li, kind), []).append(e0.elapsed_time(e1))
    tot = {k: sum(v) for k, v in per.items()}
    pk = peaks()
    dom = max(tot, key=tot.get)
    Ld = layers[dom[0]]
    avg_ms = statistics.mean(per[dom])
    kernel_of = {"fwd": "tc_apply", "dx": "tc_apply", "dw": "dw", "set_weights": "pretransform"}
    if dom[1] in ("fwd", "dx", "dw"):
        # the bound is the resource the call's arithmetic intensity points at:
        # tensor when its FLOP per algorithmic byte exceed the measured ridge
        flop = Ld.actual_flop()
        byt = Ld.bytes_dw() if dom[1] == "dw" else Ld.bytes_fwd()
        ridge = pk["bf16_sustained"] * 1e12 / (pk["hbm_gbs"] * 1e9)
        if flop / byt >= ridge / 2:
            achieved = flop / (avg_ms * 1e-3) / 1e12
            roof = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_sustained"], "unit": "TFLOP/s",
                    "frac": achieved / pk["bf16_sustained"],
                    "peak_kind": f"{pk['source']} bf16 dense, sustained (kernel timed inside a long step)"}
        else:
            achieved = byt / (avg_ms * 1e-3) / 1e9
            roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": achieved / pk["hbm_gbs"], "peak_kind": f"{pk['source']} HBM copy"}
        roof["intensity_flop_per_byte"] = flop / byt
    else:
        byt = Ld.Dp * Ld.Cp * Ld.T * 2 * 2
        achieved = byt / (avg_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "peak_kind": f"{pk['source']} HBM copy"}
    key = f"{kernel_of[dom[1]]}:{Ld.name}:{dom[1]}"
    roof["kernel"] = key
    roof["traffic"] = profiled_traffic(key)
    breakdown = {f"{layers[li].name}/{kind}": round(statistics.mean(v) * 1e3, 2) for (li, kind), v in per.items()}

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

        def e2e_step():
            for i, s in enumerate(st):
                hb, db_ = host[i], dbuf[i]
                db_["x"].copy_(hb["x"], non_blocking=True)
                db_["gy"].copy_(hb["gy"], non_blocking=True)
                s["W"].copy_(hb["W"], non_blocking=True)
                s["b"].copy_(hb["b"], non_blocking=True)
                eqlin.set_weights(s["h"], s["W"], s["b"])
                eqlin.forward(s["h"], db_["x"], s["y"])
                side.wait_stream(stream)
                eqlin.backward_dx(s["h"], db_["gy"], s["dx"])
                eqlin.backward_dw(s["h"], db_["x"], db_["gy"], s["dW"], s["db"], stream=side)
                stream.wait_stream(side)
                if dist:
                    dp.allreduce_grads((s["dW"], s["db"]))
                for k in ("y", "dx", "dW", "db"):
                    hb[k].copy_(s[k], non_blocking=True)

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
        b.record(stream)
        torch.cuda.synchronize()
        ems = a.elapsed_time(b) / ke
        if dist:
            tt = torch.tensor([ems], device=dev)
            torch.distributed.all_reduce(tt, op=torch.distributed.ReduceOp.MAX)
            ems = float(tt.item())
        e2e = {"value": flop_step * world / (ems * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ems}

    # ---------------------------------------------------- CPU baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f, secs, threads, desc = oracle_sample(layers, oracle_data(layers), budget_s=12.0)
        cpu = {"value": f / secs / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": desc, "seconds": secs}

    if rank == 0:
        set_bytes = sum(sum(t.numel() * t.element_size() for t in s["sets"][0].values()) for s in st)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": layers[0].dtype, "data": "synthetic",
            "config": {
                "workload": args.workload,
                "layers": [dict(name=L.name, T=L.T, Cp=L.Cp, Dp=L.Dp, N=L.N, passes=list(L.passes))
                           for L in layers],
                "step": "per layer: set_weights (weight DFT) + forward + dx + dW/db, dW/db on a second "
                        "stream beside dx"
                        + (" + NCCL all-reduce of dW/db" if dist else ""),
                "tokens_per_gpu": layers[0].N,
                "l2": f"inputs rotate over {N_SETS} sets of {set_bytes / 1e6:.0f} MB each "
                      f"({N_SETS * set_bytes / 1e6:.0f} MB > 126 MB L2)",
                "actual_tflops": sum(L.actual_flop() * len(L.passes) for L in layers) * world
                                 / (ms_per_step * 1e-3) / 1e12,
                "kernel_ms": breakdown,
                "kernel_ms_sampling": f"CUDA events around each call on every {REC_EVERY}th timed step",
            },
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    for s in st:
        s["h"].close()
    if dist:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
