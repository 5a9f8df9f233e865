"""Sharded layer on the GPU: tensor parallelism over d_ff and expert parallelism, through
moe_forward_partial and moe_reduce_partials.

The deployments the pages name (vLLM TP8 on eight GPUs in the gpuvram.cloud model card;
vLLM expert parallelism in the pgsm.cn hands-on) run one shard per GPU and add the
shards' parts.  This run has one GPU, so every shard runs here one after another, on its
own copy of its weights, and the parts are added by moe_reduce_partials exactly as they
would be from the other GPUs' buffers.  Each part is compared with the oracle's part of that
shard and the sum with the oracle's whole layer.
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_47_b200 as moe
import oracle
from gpu_helpers import Y_REL_TOL, rel_err, route_parity
from workloads import WORKLOADS, make_inputs, make_small, to_device

pytestmark = pytest.mark.gpu


def _f_slice(dev, f0, f1):
    rows = lambda W: W[:, f0:f1, :].contiguous()   # noqa: E731
    cols = lambda W: W[:, :, f0:f1].contiguous()   # noqa: E731
    return (rows(dev.W_gate), rows(dev.W_up), cols(dev.W_down),
            rows(dev.Ws_gate), rows(dev.Ws_up), cols(dev.Ws_down))


def _run_shard(wl, dev, F_local, e0, weights, shared, ws_cache):
    h = moe.moe_create(wl.d, wl.E, wl.k, F_local, wl.S)
    ws = torch.empty(moe.moe_workspace_size(h, wl.T), dtype=torch.uint8, device="cuda")
    part = torch.full((wl.T, wl.d), float("nan"), dtype=torch.float32, device="cuda")
    Wg, Wu, Wd = weights
    Sg, Su, Sd = shared if shared is not None else (None, None, None)
    moe.moe_forward_partial(h, dev.x, dev.W_router, dev.bias, e0, Wg, Wu, Wd, Sg, Su, Sd, part,
                            ws)
    st, detail = moe.moe_device_status(h, wl.T, ws)
    assert st == moe.MOE_OK, (st, hex(detail))
    ws_cache.append((h, ws))
    return part


def _routing(inp, h_ws):
    """The GPU's routing (from the last shard's workspace) and the oracle's, with near-tie
    tokens taking the GPU's choice."""
    h, ws = h_ws
    v = moe.workspace_views(h, inp.wl.T, ws)
    logits = oracle.router_logits(inp.x.cpu(), inp.W_router.cpu(),
                                  None if inp.bias is None else inp.bias.cpu())
    idx_g = v["topk_idx"].cpu().numpy()
    exempt, idx_o, _ = route_parity(logits, idx_g, v["topk_w"].cpu().numpy(), inp.wl.k)
    idx_use = np.where(exempt[:, None], idx_g, idx_o)
    return idx_use, oracle.renormalised_gates(logits, idx_use)


def _reduce(h, parts):
    y = torch.empty(parts[0].shape, dtype=torch.bfloat16, device="cuda")
    moe.moe_reduce_partials(h, parts, y)
    torch.cuda.synchronize()
    return y.float().cpu().numpy()


SHAPES = [  # T, d, E, k, F, S, n_shards
    (64, 256, 16, 2, 256, 1, 4),
    (300, 192, 64, 8, 384, 1, 3),      # 128-wide slices: ragged against the 256-row tiles
    (600, 256, 4, 2, 128, 1, 2),       # the 2-SM weight-major GEMMs (>= 96 rows per expert)
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "T{}_d{}_E{}_k{}_F{}_S{}_n{}".format(*s))
def test_d_ff_slices_reduce_to_the_layer(shape):
    T, d, E, k, F, S, n = shape
    inp = make_small(T, d, E, k, F, S, seed=700 + T, bias_scale=0.2)
    dev = to_device(inp, "cuda")
    width = F // n
    parts, keep = [], []
    for r in range(n):
        Wg, Wu, Wd, Sg, Su, Sd = _f_slice(dev, r * width, (r + 1) * width)
        parts.append(_run_shard(inp.wl, dev, width, 0, (Wg, Wu, Wd), (Sg, Su, Sd), keep))
    idx, w = _routing(inp, keep[-1])
    for r in range(n):
        Wg, Wu, Wd, Sg, Su, Sd = (t.cpu() for t in _f_slice(inp, r * width, (r + 1) * width))
        ref = oracle.shard_output(inp.x, idx, w, Wg, Wu, Wd, Sg, Su, Sd)
        assert rel_err(parts[r].cpu().numpy(), ref) < Y_REL_TOL, r
    y = _reduce(keep[0][0], parts)
    ref = oracle.forward(inp, idx_override=idx)["y"]
    assert rel_err(y, ref) < Y_REL_TOL


EP_CASES = [  # T, d, E, k, F, S, expert ranges
    (64, 256, 16, 2, 128, 1, [(0, 5), (5, 6), (11, 5)]),
    (700, 128, 8, 2, 64, 1, [(0, 4), (4, 4)]),                  # 2-SM GEMMs, 175 rows/expert
    (40, 256, 8, 8, 128, 2, [(0, 1), (1, 7)]),                  # k == E, two shared experts
]


@pytest.mark.parametrize("case", EP_CASES, ids=lambda c: "T{}_d{}_E{}_k{}_F{}_S{}".format(*c[:6]))
def test_expert_ranges_reduce_to_the_layer(case):
    T, d, E, k, F, S, ranges = case
    inp = make_small(T, d, E, k, F, S, seed=800 + T, bias_scale=0.3)
    dev = to_device(inp, "cuda")
    parts, keep = [], []
    for r, (e0, n) in enumerate(ranges):
        sl = slice(e0, e0 + n)
        shared = (dev.Ws_gate, dev.Ws_up, dev.Ws_down) if r == 0 else None
        parts.append(_run_shard(inp.wl, dev, F, e0,
                                (dev.W_gate[sl], dev.W_up[sl], dev.W_down[sl]), shared, keep))
    idx, w = _routing(inp, keep[-1])
    for r, (e0, n) in enumerate(ranges):
        sl = slice(e0, e0 + n)
        shared = (inp.Ws_gate, inp.Ws_up, inp.Ws_down) if r == 0 else (None, None, None)
        ref = oracle.shard_output(inp.x, idx, w, inp.W_gate[sl], inp.W_up[sl], inp.W_down[sl],
                                  *shared, expert_begin=e0)
        got = parts[r].cpu().numpy()
        if np.abs(ref).max() == 0:
            assert np.all(got == 0)
        else:
            assert rel_err(got, ref) < Y_REL_TOL, r
    y = _reduce(keep[0][0], parts)
    assert rel_err(y, oracle.forward(inp, idx_override=idx)["y"]) < Y_REL_TOL


def test_partial_rejects_bad_ranges_and_reduce_is_ordered():
    inp = make_small(16, 64, 4, 2, 64, 1, seed=3)
    dev = to_device(inp, "cuda")
    h = moe.moe_create(64, 4, 2, 64, 1)
    ws = torch.empty(moe.moe_workspace_size(h, 16), dtype=torch.uint8, device="cuda")
    part = torch.empty(16, 64, dtype=torch.float32, device="cuda")
    for e0, n in ((-1, 2), (3, 2), (0, 0)):
        with pytest.raises(moe.MoEError) as e:
            moe.moe_forward_partial(h, dev.x, dev.W_router, None, e0, dev.W_gate[:n],
                                    dev.W_up[:n], dev.W_down[:n], None, None, None, part, ws)
        assert e.value.status == moe.MOE_ERR_INVALID_ARG
    # fp32 adds in rank order: 1 + 2^-24 + 2^-24 rounds to 1 one step at a time
    a = torch.ones(16, 64, device="cuda")
    b = torch.full((16, 64), 2.0 ** -24, device="cuda")
    y = torch.empty(16, 64, dtype=torch.bfloat16, device="cuda")
    moe.moe_reduce_partials(h, [a, b, b, -a], y)
    torch.cuda.synchronize()
    assert torch.all(y.float() == 0.0)
    moe.moe_reduce_partials(h, [b, b, a, -a], y)
    torch.cuda.synchronize()
    assert torch.all(y.float() == torch.tensor(2.0 ** -23).bfloat16().float())


@pytest.mark.parametrize("mode", ["tp8", "ep8"])
def test_hy4_decode_on_eight_shards(mode):
    """The Hy4-shaped decode workload split as the pages' eight-GPU deployments would split it:
    TP8 (d_ff slices of 256) or EP8 (32 routed experts per shard, the shared expert on the
    first), every shard run here; the sum against the oracle on every token."""
    wl = WORKLOADS["decode"]
    inp = make_inputs(wl, device="cuda")
    parts, keep = [], []
    for r in range(8):
        if mode == "tp8":
            f0, f1 = r * 256, (r + 1) * 256
            Wg, Wu, Wd, Sg, Su, Sd = _f_slice(inp, f0, f1)
            parts.append(_run_shard(wl, inp, 256, 0, (Wg, Wu, Wd), (Sg, Su, Sd), keep))
            del Wg, Wu, Wd
        else:
            sl = slice(32 * r, 32 * (r + 1))
            shared = (inp.Ws_gate, inp.Ws_up, inp.Ws_down) if r == 0 else None
            parts.append(_run_shard(wl, inp, wl.F, 32 * r,
                                    (inp.W_gate[sl], inp.W_up[sl], inp.W_down[sl]), shared,
                                    keep))
    idx, w = _routing(inp, keep[-1])
    y = _reduce(keep[0][0], parts)
    used = sorted(set(idx.reshape(-1).tolist()))
    weights = {"W_gate": {e: inp.W_gate[e].cpu() for e in used},
               "W_up": {e: inp.W_up[e].cpu() for e in used},
               "W_down": {e: inp.W_down[e].cpu() for e in used}}
    ref = oracle.moe_ffn_tokens(inp.x.cpu(), idx, w, weights["W_gate"], weights["W_up"],
                                weights["W_down"], inp.Ws_gate.cpu(), inp.Ws_up.cpu(),
                                inp.Ws_down.cpu(), None, E=wl.E, F=wl.F, S=wl.S)
    err = rel_err(y, ref)
    print(f"decode {mode}: rel err {err:.3e}")
    assert err < Y_REL_TOL, err
