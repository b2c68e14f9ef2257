"""bench.py's host logic on CPU: the local multi-rank launcher and the
roofline arithmetic (no GPU)."""
import json
import os

import pytest

import bench
from group_circulant_linear_b200 import workloads


def test_rank_env():
    env = bench.rank_env(1, 4, 23456)
    assert env == {"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "4", "LOCAL_WORLD_SIZE": "4",
                   "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": "23456"}


def _probe(argv):
    """A rank body: joins a gloo group from the launcher's environment and
    takes the max over ranks of a per-rank value, as bench.py does with its
    timings."""
    import torch
    import torch.distributed as dist
    out = argv[0]
    dist.init_process_group("gloo")
    try:
        r, w = dist.get_rank(), dist.get_world_size()
        t = torch.tensor([float(10 * (r + 1))])
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        with open(os.path.join(out, f"{r}.json"), "w") as f:
            json.dump({"rank": r, "world": w, "env_rank": os.environ["RANK"],
                       "local": os.environ["LOCAL_RANK"], "max": float(t.item())}, f)
    finally:
        dist.destroy_process_group()


def test_launch_local_starts_ranks_that_reduce(tmp_path):
    bench.launch_local(2, [str(tmp_path)], target=_probe)
    got = [json.load(open(tmp_path / f"{r}.json")) for r in range(2)]
    for r, g in enumerate(got):
        assert g["rank"] == r and g["world"] == 2
        assert g["env_rank"] == str(r) and g["local"] == str(r)
        assert g["max"] == 20.0


def test_gpus_flag_launches_local_ranks(monkeypatch):
    calls = []
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(bench, "launch_local", lambda n, argv, target=None: calls.append((n, list(argv))))
    bench.main(["--gpus", "4", "--steps", "3"])
    assert calls == [(4, ["--gpus", "4", "--steps", "3"])]


def test_roofline_arithmetic():
    pk = {"hbm_gbs": 6000.0, "bf16": 1500.0, "bf16_sustained": 1400.0, "source": "test"}
    L = workloads.WORKLOADS["eq-vit-b-mlp-bf16-fwdbwd"][0]
    us = 50.0
    r = bench.roofline_of(L, "fwd", us, pk)
    flop, byt = L.actual_flop(), L.bytes_fwd()
    assert r["tflops"] == pytest.approx(flop / 50e-6 / 1e12)
    assert r["frac_tensor"] == pytest.approx(flop / 50e-6 / 1.5e15)
    assert r["frac_hbm"] == pytest.approx(byt / 50e-6 / 6e12)
    assert r["frac_roofline"] == pytest.approx(max(flop / 1.5e15, byt / 6e12) / 50e-6)
    assert r["bound"] == "tensor" and r["frac"] == r["frac_tensor"]
    S = workloads.WORKLOADS["eq-swin-t-s1-f16-fwdbwd"][0]          # 29 FLOP per byte: HBM-bound
    r = bench.roofline_of(S, "dw", 100.0, pk)
    assert r["bound"] == "hbm" and r["frac"] == pytest.approx(S.bytes_dw() / 100e-6 / 6e12)


@pytest.mark.parametrize("T,kind,bound", [(2, "fwd", "tensor"), (4, "dw", "tensor"), (8, "dx", "tensor"),
                                          (8, "dw", "alu"), (3, "fwd", "alu"), (6, "dw", "alu")])
def test_roofline_fp32_denominators(T, kind, bound):
    """FP32 passes on 3xTF32 are measured as three TF32 MMAs per product against
    half the bf16 peak; FP32 passes on the CUDA cores against the nominal FFMA
    rate; neither against the bf16 ridge that decides f16/bf16 passes."""
    pk = {"hbm_gbs": 6000.0, "bf16": 1500.0, "bf16_sustained": 1400.0, "source": "test"}
    L = workloads.Layer("t", T, 96, 96, 4096, "f32", ("fwd", "dx", "dw"))
    us = 40.0
    flop = L.actual_flop()
    r = bench.roofline_of(L, kind, us, pk)
    assert r["bound"] == bound
    if bound == "tensor":
        assert r["peak"] == 750.0 and r["unit"].startswith("TFLOP/s (tf32")
        assert r["achieved"] == pytest.approx(3 * flop / 40e-6 / 1e12)
        assert r["frac"] == pytest.approx(3 * flop / 40e-6 / 750e12)
        assert r["fp32_equiv_tflops"] == pytest.approx(flop / 40e-6 / 1e12)
    else:
        ffma = 148 * 128 * 2 * 1.965e9
        assert r["unit"] == "TFLOP/s (FFMA)" and r["peak"] == pytest.approx(ffma / 1e12)
        assert r["frac"] == pytest.approx(flop / 40e-6 / ffma)
    assert r["frac_roofline"] >= r["frac"]


def test_tail_split_flag():
    # off unless asked for: the bench's step keeps the library's default
    assert bench.parse([]).tail_split is False
    assert bench.parse(["--tail-split"]).tail_split is True


def test_cpu_info():
    info = bench.cpu_info()
    assert info["nproc"] == os.cpu_count() and isinstance(info["cpu_model"], str)
