"""The autograd layer and the synthetic EQ-ViT block.

CPU: the dense expansion (the naive layer the block is timed against) equals
the oracle's definition, and the block's non-EQ-Linear parts (group
LayerNorm, attention with heads split along C') commute with a cyclic shift
of the group axis.

GPU: ``EQLinear`` forward and all three gradients against the oracle; the
weight transform re-runs after an in-place weight update; the whole block
against an FP32 evaluation of the same block with the dense matrices, and its
equivariance.  The block composes four EQ-Linear layers with attention and
norms in BF16, so its comparison with the FP32 block allows 3e-2 (relative
Frobenius); each layer alone is held to the 2e-2 of the layer tests.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from group_circulant_linear_b200 import inputs

TOL_BF16 = 2e-2
TOL_BLOCK = 3e-2


def rel_err(out, ref) -> float:
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(out - ref) / (den if den > 0 else 1.0))


def _roll_group(a: torch.Tensor, T: int, r: int) -> torch.Tensor:
    """Cyclic shift by r along the group axis of features [..., C'*T]."""
    sh = a.shape
    return torch.roll(a.reshape(*sh[:-1], sh[-1] // T, T), r, dims=-1).reshape(sh)


# ------------------------------------------------------------------ CPU

@pytest.mark.parametrize("T,Cp,Dp", [(4, 3, 5), (1, 4, 3), (2, 3, 2), (8, 2, 3)])
def test_expand_dense_is_the_definition(T, Cp, Dp):
    from group_circulant_linear_b200.block import expand_dense
    inp = inputs.make_inputs(T, Cp, Dp, 7, "f32", seed=9)
    Wd = expand_dense(inp["W"].double())
    y = inp["x"].double() @ Wd.T + inp["b"].double().repeat_interleave(T)
    assert np.allclose(y.numpy(), oracle.forward(inp["x"], inp["W"], inp["b"]), rtol=0, atol=1e-12)


def test_norm_and_attention_commute_with_group_shift():
    from group_circulant_linear_b200.block import GroupLayerNorm, _attention
    torch.manual_seed(0)
    T, Cp, heads = 4, 8, 2
    n = GroupLayerNorm(Cp, T, dtype=torch.float64, device="cpu")
    with torch.no_grad():
        n.weight.uniform_(0.5, 1.5)
        n.bias.uniform_(-0.2, 0.2)
    x = torch.randn(2, 5, Cp * T, dtype=torch.float64)
    h = torch.randn(2, 5, 3 * Cp * T, dtype=torch.float64)
    for r in range(T):
        assert torch.allclose(n(_roll_group(x, T, r)), _roll_group(n(x), T, r), atol=1e-12)
        assert torch.allclose(_attention(_roll_group(h, T, r), heads, Cp, T),
                              _roll_group(_attention(h, heads, Cp, T), T, r), atol=1e-12)


# ------------------------------------------------------------------ GPU

@pytest.mark.gpu
def test_eqlinear_autograd_against_oracle():
    from group_circulant_linear_b200.block import EQLinear
    T, Cp, Dp, N = 4, 64, 96, 300
    layer = EQLinear(Cp, Dp, T, dtype=torch.bfloat16, generator=torch.Generator().manual_seed(3))
    inp = inputs.make_inputs(T, Cp, Dp, N, "bf16", seed=11)
    x = inp["x"].cuda().requires_grad_(True)
    gy = inp["gy"].cuda()
    y = layer(x.view(3, 100, Cp * T))
    y.backward(gy.view(3, 100, Dp * T))
    torch.cuda.synchronize()
    W, b = layer.weight.detach().cpu(), layer.bias.detach().cpu()
    assert rel_err(y.detach().float().cpu().reshape(N, -1), oracle.forward(inp["x"], W, b)) <= TOL_BF16
    assert rel_err(x.grad.float().cpu(), oracle.backward_dx(inp["gy"], W)) <= TOL_BF16
    dW, db = oracle.backward_dw(inp["x"], inp["gy"], T, Cp, Dp)
    assert rel_err(layer.weight.grad.float().cpu(), dW) <= TOL_BF16
    assert rel_err(layer.bias.grad.float().cpu(), db) <= TOL_BF16


@pytest.mark.gpu
def test_eqlinear_rereads_weights_after_update():
    from group_circulant_linear_b200.block import EQLinear
    T, Cp, Dp, N = 4, 32, 32, 64
    layer = EQLinear(Cp, Dp, T, dtype=torch.bfloat16, generator=torch.Generator().manual_seed(4))
    x = inputs.make_inputs(T, Cp, Dp, N, "bf16", seed=12)["x"].cuda()
    layer(x)
    with torch.no_grad():
        layer.weight.mul_(-2.0)        # an optimizer step would update in place like this
        layer.bias.add_(0.5)
    y = layer(x)
    torch.cuda.synchronize()
    want = oracle.forward(x.cpu(), layer.weight.detach().cpu(), layer.bias.detach().cpu())
    assert rel_err(y.detach().float().cpu(), want) <= TOL_BF16


@pytest.mark.gpu
def test_eqlinear_deepcopy_gets_its_own_handle():
    import copy

    from group_circulant_linear_b200.block import EQLinear
    T, Cp, Dp, N = 4, 32, 32, 64
    layer = EQLinear(Cp, Dp, T, dtype=torch.bfloat16, generator=torch.Generator().manual_seed(6))
    x = inputs.make_inputs(T, Cp, Dp, N, "bf16", seed=16)["x"].cuda()
    y = layer(x)
    twin = copy.deepcopy(layer)
    assert twin.h.ptr.value != layer.h.ptr.value
    del layer                     # destroys only the original's handle
    y2 = twin(x)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)


@pytest.mark.gpu
def test_block_against_fp32_dense_block_and_equivariance():
    from group_circulant_linear_b200.block import DenseEQViTBlock, EQViTBlock
    T, Cp, heads, B, L = 4, 32, 4, 2, 50
    blk = EQViTBlock(Cp, heads, T, dtype=torch.bfloat16, seed=5)
    ref = DenseEQViTBlock(blk, dtype=torch.float32)
    g = torch.Generator().manual_seed(13)
    x0 = torch.randn(B, L, Cp * T, generator=g)
    gy = torch.randn(B, L, Cp * T, generator=g).cuda()

    x = x0.cuda().bfloat16().requires_grad_(True)
    y = blk(x)
    y.backward(gy.bfloat16())
    got_dx = x.grad.float().cpu().numpy()
    got_dw = blk.fc1.weight.grad.float().cpu().numpy()
    for p in blk.parameters():
        p.grad = None

    xr = x0.cuda().bfloat16().float().requires_grad_(True)
    yr = ref(xr)
    yr.backward(gy)
    torch.cuda.synchronize()
    assert rel_err(y.detach().float().cpu(), yr.detach().cpu()) <= TOL_BLOCK
    assert rel_err(got_dx, xr.grad.cpu()) <= TOL_BLOCK
    assert rel_err(got_dw, blk.fc1.weight.grad.float().cpu()) <= TOL_BLOCK

    with torch.no_grad():
        xb = x0.cuda().bfloat16()
        y0 = blk(xb)
        for r in range(1, T):
            assert rel_err(blk(_roll_group(xb, T, r)).float().cpu(),
                           _roll_group(y0, T, r).float().cpu()) <= TOL_BF16
    for layer in (blk.qkv, blk.proj, blk.fc1, blk.fc2):
        from group_circulant_linear_b200 import eqlin
        assert eqlin.get_error(layer.h) == 0
