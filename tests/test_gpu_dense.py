"""The dense FFN layer (the model's first layer) on the GPU through moe_dense_ffn.

The dense layer is the MoE layer with one routed expert chosen with weight 1 and no shared
expert, which the oracle computes as such (pinned against a float64 dense SwiGLU in
tests/test_oracle.py).  moe_dense_ffn runs the same expert GEMM kernels without router,
dispatch, gather and combine, so where it does not split the down projection over K its
output equals moe_forward's on that one-expert layer bit for bit (the combine of one
weight-1 row reproduces the row's bf16 value); with the split (up to 128 tokens, 1-SM
tiling) the fp32 parts are added before the one rounding -- by the down GEMM's last K range
to finish each output tile, or by a separate kernel for wide layers -- so the two agree
within the bar.
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_47_b200 as moe
import oracle
from gpu_helpers import Y_REL_TOL, rel_err
from workloads import WORKLOADS, make_inputs, make_small, to_device

pytestmark = pytest.mark.gpu

# (16, 8448, 128): 33 output tiles of 256 features, more than the down GEMM's in-kernel sum
# of the K ranges keeps counters for, so the ranges' parts go through the separate sum
SHAPES = [(1, 64, 64), (64, 256, 640), (40, 128, 576), (300, 192, 384), (1000, 128, 192),
          (517, 256, 2304), (16, 8448, 128)]


def _dense(inp, T):
    wl = inp.wl
    h = moe.moe_create(wl.d, 1, 1, wl.F, 0)
    ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
    y = torch.full((T, wl.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    moe.moe_dense_ffn(h, inp.x, inp.W_gate, inp.W_up, inp.W_down, y, ws)
    st, detail = moe.moe_device_status(h, T, ws)
    assert st == moe.MOE_OK, hex(detail)
    return h, ws, y


@pytest.mark.parametrize("tiles", ["auto", "single", "pair", "swap", "swap_pair"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "T{}_d{}_F{}".format(*s))
def test_dense_ffn_matches_oracle_and_the_one_expert_layer(shape, tiles, monkeypatch):
    if tiles != "auto":
        monkeypatch.setenv("MOE_GEMM_TILES", tiles)
    T, d, F = shape
    inp = make_small(T, d, 1, 1, F, 0, seed=1000 + T)
    dev = to_device(inp, "cuda")
    h, ws, y = _dense(dev, T)
    ref = oracle.forward(inp)["y"]
    assert rel_err(y.float().cpu().numpy(), ref) < Y_REL_TOL
    y2 = torch.empty_like(y)
    moe.moe_forward(h, dev.x, dev.W_router, None, dev.W_gate, dev.W_up, dev.W_down, None, None,
                    None, y2, ws)
    torch.cuda.synchronize()
    # the K split needs the 1-SM weight-major tiling and at most 128 tokens
    if T > 128 or tiles in ("single", "pair", "swap_pair"):
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    else:
        assert rel_err(y.float().cpu().numpy(), y2.float().cpu().numpy()) < Y_REL_TOL


def test_dense_ffn_rejects_a_moe_context():
    h = moe.moe_create(64, 4, 2, 64, 1)
    x = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(moe.moe_workspace_size(h, 4), dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):     # the binding checks the dense shape against h.F / h.d
        moe.moe_dense_ffn(h, x, W[:32], W[:32], W[:, :32], x, ws)
    with pytest.raises(moe.MoEError) as e:
        moe.moe_dense_ffn(h, x, W, W, W, x, ws)
    assert e.value.status == moe.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("name", ["dense_decode", "dense_prefill"])
def test_dense_first_layer_full_size(name):
    """The dense first layer at the Hy4 width (d_ff 18432) on decode and prefill batches:
    every token at decode, 48 evenly spaced tokens plus the last one at prefill."""
    wl = WORKLOADS[name]
    inp = make_inputs(wl, device="cuda")
    _, _, y = _dense(inp, wl.T)
    tokens = np.unique(np.concatenate([np.linspace(0, wl.T - 1, min(48, wl.T)).round(),
                                       [wl.T - 1]]).astype(np.int32))
    idx = np.zeros((wl.T, 1), np.int32)
    w = np.ones((wl.T, 1))
    ref = oracle.moe_ffn_tokens(inp.x.cpu(), idx, w, inp.W_gate.cpu(), inp.W_up.cpu(),
                                inp.W_down.cpu(), inp.Ws_gate.cpu(), inp.Ws_up.cpu(),
                                inp.Ws_down.cpu(), tokens, E=1, F=wl.F, S=0)
    err = rel_err(y.float().cpu().numpy()[tokens], ref)
    print(f"{name}: {len(tokens)} tokens, rel err {err:.3e}")
    assert err < Y_REL_TOL, err


@pytest.mark.parametrize("shape", [(64, 256, 640), (517, 256, 2304)],
                         ids=lambda s: "T{}_d{}_F{}".format(*s))
def test_dense_ffn_host_matches_the_device_call(shape):
    """moe_dense_ffn_host on pinned host activations gives moe_dense_ffn's bits.  Calls are
    enqueued back to back without synchronising, each on its own input, so the staging slots
    alternate while earlier layers still run; every output is its own input's."""
    T, d, F = shape
    inputs = [make_small(T, d, 1, 1, F, 0, seed=1200 + T + i) for i in range(3)]
    dev = to_device(inputs[0], "cuda")
    h = moe.moe_create(d, 1, 1, F, 0)
    ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
    want = []
    for inp in inputs:
        y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
        moe.moe_dense_ffn(h, inp.x.cuda(), dev.W_gate, dev.W_up, dev.W_down, y, ws)
        want.append(y.cpu())
    xs = [inp.x.pin_memory() for inp in inputs]
    ys = [torch.full((T, d), float("nan"), dtype=torch.bfloat16).pin_memory() for _ in inputs]
    for _ in range(2):
        for x, y in zip(xs, ys):
            moe.moe_dense_ffn_host(h, x, dev.W_gate, dev.W_up, dev.W_down, y, ws)
    torch.cuda.synchronize()
    st, detail = moe.moe_device_status(h, T, ws)
    assert st == moe.MOE_OK, hex(detail)
    for y, w in zip(ys, want):
        assert torch.equal(y.view(torch.int16), w.view(torch.int16))
