"""The combine fused into the down GEMM (MOE_FUSED_COMBINE=1 when the context is created).

The fused form adds the same rows in the same order as the separate combine kernel, so the
layer output must be bit-identical to the unfused forward, under both weight-major tilings
(1-SM and 2-SM) and at the Hy4 decode and prefill sizes; the row-tiled tilings have no fused
form and fall back to the separate kernel.  The launch count drops by one where it applies.
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_47_b200 as moe
import oracle
from gpu_helpers import Y_REL_TOL, rel_err, route_parity
from workloads import WORKLOADS, make_inputs, make_small, to_device

pytestmark = pytest.mark.gpu


def _forward(inp, fused, monkeypatch, tiles=None):
    if fused:
        monkeypatch.setenv("MOE_FUSED_COMBINE", "1")
    else:
        monkeypatch.delenv("MOE_FUSED_COMBINE", raising=False)
    if tiles:
        monkeypatch.setenv("MOE_GEMM_TILES", tiles)
    else:
        monkeypatch.delenv("MOE_GEMM_TILES", raising=False)
    wl = inp.wl
    h = moe.moe_create(wl.d, wl.E, wl.k, wl.F, wl.S)
    ws = torch.empty(moe.moe_workspace_size(h, wl.T), dtype=torch.uint8, device="cuda")
    y = torch.full((wl.T, wl.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(h, inp.x, inp.W_router, inp.bias, inp.W_gate, inp.W_up, inp.W_down,
                    inp.Ws_gate, inp.Ws_up, inp.Ws_down, y, ws)
    st, detail = moe.moe_device_status(h, wl.T, ws)
    assert st == moe.MOE_OK, hex(detail)
    return y.cpu(), moe.moe_forward_kernel_count(h, wl.T), h, ws


SHAPES = [(64, 256, 16, 2, 128, 1), (600, 256, 4, 2, 128, 1), (130, 320, 5, 3, 384, 2),
          (1, 64, 1, 1, 64, 0), (513, 512, 64, 8, 256, 1)]


@pytest.mark.parametrize("tiles", [None, "swap", "swap_pair", "single", "pair"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "T{}_d{}_E{}_k{}_F{}_S{}".format(*s))
def test_fused_combine_is_bit_identical(shape, tiles, monkeypatch):
    T, d, E, k, F, S = shape
    inp = to_device(make_small(T, d, E, k, F, S, seed=1300 + T, bias_scale=0.2), "cuda")
    y0, n0, _, _ = _forward(inp, False, monkeypatch, tiles)
    y1, n1, _, _ = _forward(inp, True, monkeypatch, tiles)
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
    weight_major = tiles in (None, "swap", "swap_pair")
    assert n1 == (n0 - 1 if weight_major else n0)
    ref = oracle.forward(make_small(T, d, E, k, F, S, seed=1300 + T, bias_scale=0.2))
    assert rel_err(y1.float().numpy(), ref["y"]) < Y_REL_TOL


@pytest.mark.parametrize("name", ["decode", "prefill"])
def test_fused_combine_full_size(name, monkeypatch):
    wl = WORKLOADS[name]
    inp = make_inputs(wl, device="cuda")
    y0, _, _, _ = _forward(inp, False, monkeypatch)
    y1, _, h, ws = _forward(inp, True, monkeypatch)
    same = torch.equal(y0.view(torch.int16), y1.view(torch.int16))
    print(f"{name}: fused combine bit-identical {same}")
    assert same
