"""Where the layer's output error comes from, measured against the fp64 oracle.

The CUDA path rounds three times: the SwiGLU activations H to bf16 before the down
projection, the per-(slot, expert) rows Y to bf16 inside moe_forward, and the output y to
bf16.  The same routing and inputs go through four routes that add the roundings one at a
time:
  H          moe_expert_ffn's fp32 Y rows, added on the host in fp64;
  H + y      moe_expert_ffn (fp32 Y) then moe_combine (y rounded);
  H + Y      moe_forward_partial over all experts with the shared expert (bf16 Y, y in fp32);
  H + Y + y  moe_forward.
Each error is max|gpu - ref| / max|ref| over the tokens checked; all must stay within the
layer's 1e-2 bar, and the split is printed for the record.
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_47_b200 as moe
import oracle
from gpu_helpers import Y_REL_TOL, rel_err, route_parity
from workloads import WORKLOADS, make_inputs, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_error_budget_of_the_roundings(name):
    wl = WORKLOADS[name]
    if name == "tiny":
        cpu = make_inputs(wl, device="cpu")
        dev = to_device(cpu, "cuda")
    else:
        dev = make_inputs(wl, device="cuda")
        cpu = None
    T, d, E, k, S = wl.T, wl.d, wl.E, wl.k, wl.S
    h = moe.moe_create(d, E, k, wl.F, S)
    ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    pos = torch.empty(T * k, dtype=torch.int32, device="cuda")
    Y = torch.empty(T * k + S * T, d, dtype=torch.float32, device="cuda")
    y_hy = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    y_hY = torch.empty(T, d, dtype=torch.float32, device="cuda")
    y_all = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    W = (dev.W_gate, dev.W_up, dev.W_down, dev.Ws_gate, dev.Ws_up, dev.Ws_down)
    moe.moe_route(h, dev.x, dev.W_router, dev.bias, idx, w, ws)
    moe.moe_dispatch(h, idx, counts, offsets, perm, pos, ws)
    moe.moe_expert_ffn(h, dev.x, perm, offsets, *W, Y, ws)
    moe.moe_combine(h, Y, w, pos, y_hy)
    moe.moe_forward_partial(h, dev.x, dev.W_router, dev.bias, 0, *W, y_hY, ws)
    moe.moe_forward(h, dev.x, dev.W_router, dev.bias, *W, y_all, ws)
    st, detail = moe.moe_device_status(h, T, ws)
    assert st == moe.MOE_OK, hex(detail)

    x_cpu = dev.x.cpu()
    logits = oracle.router_logits(x_cpu, dev.W_router.cpu(), None)
    idx_g = idx.cpu().numpy()
    exempt, idx_o, _ = route_parity(logits, idx_g, w.cpu().numpy(), k)
    idx_use = np.where(exempt[:, None], idx_g, idx_o)
    w_use = oracle.renormalised_gates(logits, idx_use)
    used = sorted(set(idx_use.reshape(-1).tolist()))
    src = cpu if cpu is not None else dev
    ref = oracle.moe_ffn_tokens(
        x_cpu, idx_use, w_use, {e: src.W_gate[e].cpu() for e in used},
        {e: src.W_up[e].cpu() for e in used}, {e: src.W_down[e].cpu() for e in used},
        src.Ws_gate.cpu(), src.Ws_up.cpu(), src.Ws_down.cpu(), None, E=E, F=wl.F, S=S)
    y_h = oracle.combine(Y.cpu().double().numpy(), w.cpu().double().numpy(),
                         pos.cpu().numpy(), T, k, S)
    errs = {"H": rel_err(y_h, ref), "H+y": rel_err(y_hy.float().cpu().numpy(), ref),
            "H+Y": rel_err(y_hY.cpu().numpy(), ref),
            "H+Y+y": rel_err(y_all.float().cpu().numpy(), ref)}
    print(f"{name}: error budget " + ", ".join(f"{k_} {v:.3e}" for k_, v in errs.items()))
    for v in errs.values():
        assert v < Y_REL_TOL
    # the layer output's own rounding (bf16, half an ulp = 2^-9 of an element) bounds the
    # difference it adds
    assert errs["H+y"] <= errs["H"] + 2.0 ** -8
