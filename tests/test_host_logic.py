"""Host-side accounting and the seeded input recipe (no GPU, no oracle)."""
import json
import math
import os

import pytest
import torch

from group_circulant_linear_b200 import inputs, workloads
from group_circulant_linear_b200.workloads import Layer, real_gemms

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_counts.json")


def _page():
    with open(GOLDEN) as f:
        return {k: v["value"] for k, v in json.load(f).items() if not k.startswith("_")}


def test_real_gemm_counts_match_pages():
    pg = _page()
    assert real_gemms(4) == pg["p4_real_gemms"]
    assert 4 * 4 == pg["p4_dense_gemms"]
    assert round(pg["p4_dense_gemms"] / real_gemms(4), 2) == pg["p4_theoretical_speedup"]
    assert [real_gemms(T) for T in (1, 2, 3, 4, 6, 8)] == [1, 2, 5, 6, 10, 14]


def test_macs_about_2ndc_over_t():
    # R(T) * N*C'*D' = R(T)/T^2 * NCD, which approaches (2/T) * NCD from below.
    for T in (2, 4, 8, 16):
        ratio = real_gemms(T) / T ** 2
        assert ratio <= _page()["mac_reduction_factor_per_T"] / T
        assert ratio >= _page()["mac_reduction_factor_per_T"] / T - 2 / T ** 2 - 1e-12


def test_operator_flops_consistent_with_pages():
    pg = _page()
    # 0.134 G = 2*N*C*D = 2^27 exactly for N=1024, C=D=256 (one shape that fits;
    # the pages do not state theirs).
    L = Layer("pages", 4, 64, 64, 1024, "f32")
    assert round(L.dense_flop() / 1e9, 3) == pg["operator_flops_naive_G"]
    flash = L.actual_flop() / 1e9
    assert flash == pytest.approx(L.dense_flop() / 1e9 * 6 / 16)
    # The pages' 0.052 G sits between the six GEMMs alone and the GEMMs plus
    # O(N*(C+D)) transform adds.
    transforms = 4 * L.N * (L.C + L.D) / 1e9
    assert flash <= pg["operator_flops_flash_G"] <= flash + transforms


def test_parameter_ratio():
    L = Layer("x", 4, 192, 768, 1, "bf16")
    assert (L.C * L.D) / (L.Dp * L.Cp * L.T) == _page()["params_ratio_T4"]


def test_workload_table():
    w = workloads.WORKLOADS
    assert set(w) == {"p4-tiny-f32-fwd", "eq-vit-s-f16-fwd", "eq-vit-b-mlp-bf16-fwdbwd",
                      "eq-swin-t-s1-f16-fwdbwd", "cyclic-sweep-fwdbwd"}
    fc1, fc2 = w["eq-vit-b-mlp-bf16-fwdbwd"]
    assert (fc1.N, fc1.C, fc1.D) == (64 * 197, 768, 3072)
    assert (fc2.N, fc2.C, fc2.D) == (64 * 197, 3072, 768)
    assert fc1.actual_flop() == 2 * 6 * 12608 * 192 * 768
    assert w["eq-swin-t-s1-f16-fwdbwd"][0].N == 401408
    assert {L.T for L in w["cyclic-sweep-fwdbwd"]} == {2, 4, 8}
    assert workloads.DEFAULT_BENCH in w


def test_inputs_recipe_is_seeded_and_distributed():
    a = inputs.make_inputs(4, 16, 8, 4096, "f32", seed=0)
    b = inputs.make_inputs(4, 16, 8, 4096, "f32", seed=0)
    for k in a:
        assert torch.equal(a[k], b[k])
    c = inputs.make_inputs(4, 16, 8, 4096, "f32", seed=1)
    assert not torch.equal(a["x"], c["x"])
    bound = 1 / math.sqrt(64)
    assert a["W"].abs().max() <= bound and a["W"].abs().max() > 0.9 * bound
    assert a["b"].abs().max() <= 0.1
    assert abs(float(a["x"].mean())) < 0.02 and abs(float(a["x"].std()) - 1) < 0.02
    h = inputs.make_inputs(4, 16, 8, 64, "bf16", seed=0)
    assert h["x"].dtype == torch.bfloat16
    assert torch.equal(h["x"], a["x"][:64].to(torch.bfloat16))  # same draws, then cast


def test_integer_inputs():
    z = inputs.make_integer_inputs(4, 8, 8, 100, "f16", amp=4)
    for k in ("x", "W", "gy"):
        v = z[k].float()
        assert torch.equal(v, v.round()) and v.abs().max() <= 4
    assert set(z["b"].float().unique().tolist()) <= {-1.0, 0.0, 1.0}
