"""The iHC wrapper on the GPU (moe_ihc_mix, moe_forward_ihc) against the oracle.

x = sum_j alpha_j H_j is checked against the oracle's fp64 mix within its one bf16 rounding.
The layer is then checked on the GPU's x (the routing of near-tie tokens depends on every bit
of x, so both sides start from the same bf16 input), and the updated streams
H'_i = H_i + sum_j B_ij H_j + gamma_i y against the oracle's update of the oracle's y.
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_47_b200 as moe
import oracle
from gpu_helpers import Y_REL_TOL, rel_err, route_parity
from workloads import WORKLOADS, Inputs, make_inputs, make_small, to_device

pytestmark = pytest.mark.gpu


def _coeffs(n, seed):
    g = torch.Generator().manual_seed(seed)
    alpha = (0.1 + 0.4 * torch.rand(n, generator=g)).float()
    B = (0.1 * torch.randn(n, n, generator=g)).float()
    gamma = (0.5 + torch.rand(n, generator=g)).float()
    return alpha, B, gamma


def _check(inp_cpu, dev, H, alpha, B, gamma, tokens=None):
    wl = inp_cpu.wl
    T, n = H.shape[0], H.shape[1]
    h = moe.moe_create(wl.d, wl.E, wl.k, wl.F, wl.S)
    ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
    Hd = H.cuda()
    a, Bd, gd = alpha.cuda(), B.cuda(), gamma.cuda()
    x = torch.empty(T, wl.d, dtype=torch.bfloat16, device="cuda")
    moe.moe_ihc_mix(h, Hd, a, x)
    H_out = torch.full_like(Hd, float("nan"))
    moe.moe_forward_ihc(h, Hd, a, Bd, gd, dev.W_router, dev.bias, dev.W_gate, dev.W_up,
                        dev.W_down, dev.Ws_gate, dev.Ws_up, dev.Ws_down, H_out, ws)
    st, detail = moe.moe_device_status(h, T, ws)
    assert st == moe.MOE_OK, hex(detail)
    # the mix: one bf16 rounding (half an ulp, 2^-9 relative) of an fp32 sum of n products,
    # whose own error is a few fp32 ulps of the terms' magnitudes (it shows where they cancel)
    x_ref = oracle.ihc_mix_in(H, alpha.double().numpy())
    scale = oracle.ihc_mix_in(np.abs(oracle._as_f64(H)), np.abs(alpha.double().numpy()))
    xg = x.float().cpu().numpy()
    assert np.all(np.abs(xg - x_ref) <= np.abs(x_ref) * 2.0 ** -8 + scale * 2.0 ** -20)
    # the layer on the GPU's x, then the stream update
    v = moe.workspace_views(h, T, ws)
    x_cpu = x.cpu()
    logits = oracle.router_logits(x_cpu, inp_cpu.W_router,
                                  None if inp_cpu.bias is None else inp_cpu.bias)
    exempt, idx_o, _ = route_parity(logits, v["topk_idx"].cpu().numpy(),
                                    v["topk_w"].cpu().numpy(), wl.k)
    idx_use = np.where(exempt[:, None], v["topk_idx"].cpu().numpy(), idx_o)
    layer_inp = Inputs(wl.with_(T=T), x_cpu, inp_cpu.W_router, inp_cpu.bias, inp_cpu.W_gate,
                       inp_cpu.W_up, inp_cpu.W_down, inp_cpu.Ws_gate, inp_cpu.Ws_up,
                       inp_cpu.Ws_down)
    y_ref = oracle.forward(layer_inp, tokens=tokens, idx_override=idx_use)["y"]
    sel = slice(None) if tokens is None else tokens
    H_ref = oracle.ihc_update(H[sel], B.double().numpy(), gamma.double().numpy(), y_ref)
    got = H_out.float().cpu().numpy()[sel]
    err = rel_err(got, H_ref)
    # the layer's own part: gamma_i y against the oracle's, with the stream terms taken out
    part_ref = H_ref - oracle.ihc_update(H[sel], B.double().numpy(), np.zeros(n), 0 * y_ref)
    part_got = got - oracle.ihc_update(H[sel], B.double().numpy(), np.zeros(n), 0 * y_ref)
    return err, rel_err(part_got, part_ref), Hd, H_out, h, ws, (a, Bd, gd), dev


SHAPES = [  # T, d, E, k, F, S, n
    (64, 256, 16, 2, 128, 1, 4),
    (130, 320, 5, 3, 384, 2, 3),
    (7, 128, 3, 2, 64, 1, 1),
    (600, 256, 4, 2, 128, 1, 4),     # the 2-SM GEMMs
    (40, 256, 8, 8, 128, 0, 8),      # no shared expert, eight streams
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "T{}_d{}_E{}_k{}_F{}_S{}_n{}".format(*s))
def test_ihc_layer_matches_oracle(shape):
    T, d, E, k, F, S, n = shape
    inp = make_small(T, d, E, k, F, S, seed=1500 + T, bias_scale=0.2)
    g = torch.Generator().manual_seed(T + n)
    H = torch.randn(T, n, d, generator=g).to(torch.bfloat16)
    alpha, B, gamma = _coeffs(n, 7 + n)
    err, part_err, Hd, H_out, h, ws, (a, Bd, gd), dev = _check(inp, to_device(inp, "cuda"), H,
                                                                 alpha, B, gamma)
    print(f"iHC T={T} n={n}: rel err {err:.3e}, layer part {part_err:.3e}")
    assert err < Y_REL_TOL
    assert part_err < 0.05      # limited by the bf16 rounding of H' (|H'| >> |gamma y| here)
    # in place (H_out = H) gives the same bits
    Hc = Hd.clone()
    moe.moe_forward_ihc(h, Hc, a, Bd, gd, dev.W_router, dev.bias, dev.W_gate, dev.W_up,
                        dev.W_down, dev.Ws_gate, dev.Ws_up, dev.Ws_down, Hc, ws)
    torch.cuda.synchronize()
    assert torch.equal(Hc.view(torch.int16), H_out.view(torch.int16))


def test_ihc_one_stream_is_the_residual_block():
    """n = 1, alpha = 1, B = 0, gamma = 1: x is H bit for bit, and H' = bf16(H + y) where y
    is the layer's fp32 sum, so H' - H matches moe_forward's y within y's own rounding."""
    T, d, E, k, F, S = 64, 256, 16, 2, 128, 1
    inp = make_small(T, d, E, k, F, S, seed=1601)
    dev = to_device(inp, "cuda")
    H = dev.x.view(T, 1, d).contiguous()
    one = torch.ones(1, device="cuda")
    zero = torch.zeros(1, 1, device="cuda")
    h = moe.moe_create(d, E, k, F, S)
    ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
    x = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_ihc_mix(h, H, one, x)
    H_out = torch.empty_like(H)
    moe.moe_forward_ihc(h, H, one, zero, one, dev.W_router, dev.bias, dev.W_gate, dev.W_up,
                        dev.W_down, dev.Ws_gate, dev.Ws_up, dev.Ws_down, H_out, ws)
    y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(h, dev.x, dev.W_router, dev.bias, dev.W_gate, dev.W_up, dev.W_down,
                    dev.Ws_gate, dev.Ws_up, dev.Ws_down, y, ws)
    torch.cuda.synchronize()
    assert torch.equal(x.view(torch.int16), dev.x.view(torch.int16))
    ref = (dev.x.float() + y.float()).cpu().numpy()
    got = H_out.view(T, d).float().cpu().numpy()
    assert np.all(np.abs(got - ref) <= (np.abs(ref) + np.abs(y.float().cpu().numpy())) * 2.0 ** -7
                  + 1e-6)


def test_ihc_hy4_decode_four_streams():
    """The Hy4 decode workload inside four residual streams (the pages' iHC width)."""
    wl = WORKLOADS["decode"]
    dev = make_inputs(wl, device="cuda")
    cpu = Inputs(wl, dev.x.cpu(), dev.W_router.cpu(), None, dev.W_gate, dev.W_up, dev.W_down,
                 dev.Ws_gate.cpu(), dev.Ws_up.cpu(), dev.Ws_down.cpu())
    g = torch.Generator().manual_seed(44)
    H = torch.randn(wl.T, 4, wl.d, generator=g).to(torch.bfloat16)
    alpha, B, gamma = _coeffs(4, 45)
    h = moe.moe_create(wl.d, wl.E, wl.k, wl.F, wl.S)
    ws = torch.empty(moe.moe_workspace_size(h, wl.T), dtype=torch.uint8, device="cuda")
    H_out = torch.empty(wl.T, 4, wl.d, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward_ihc(h, H.cuda(), alpha.cuda(), B.cuda(), gamma.cuda(), dev.W_router, None,
                        dev.W_gate, dev.W_up, dev.W_down, dev.Ws_gate, dev.Ws_up, dev.Ws_down,
                        H_out, ws)
    assert moe.moe_device_status(h, wl.T, ws)[0] == moe.MOE_OK
    x = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device="cuda")
    moe.moe_ihc_mix(h, H.cuda(), alpha.cuda(), x)
    v = moe.workspace_views(h, wl.T, ws)
    logits = oracle.router_logits(x.cpu(), cpu.W_router, None)
    exempt, idx_o, _ = route_parity(logits, v["topk_idx"].cpu().numpy(),
                                    v["topk_w"].cpu().numpy(), wl.k)
    idx_use = np.where(exempt[:, None], v["topk_idx"].cpu().numpy(), idx_o)
    w_use = oracle.renormalised_gates(logits, idx_use)
    used = sorted(set(idx_use.reshape(-1).tolist()))
    y_ref = oracle.moe_ffn_tokens(x.cpu(), idx_use, w_use, {e: dev.W_gate[e].cpu() for e in used},
                                  {e: dev.W_up[e].cpu() for e in used},
                                  {e: dev.W_down[e].cpu() for e in used}, cpu.Ws_gate,
                                  cpu.Ws_up, cpu.Ws_down, None, E=wl.E, F=wl.F, S=wl.S)
    H_ref = oracle.ihc_update(H, B.double().numpy(), gamma.double().numpy(), y_ref)
    err = rel_err(H_out.float().cpu().numpy(), H_ref)
    print(f"decode iHC n=4: rel err {err:.3e}")
    assert err < Y_REL_TOL
