"""GPU parity of the FP8-weight path (moe_expert_ffn_fp8, moe_forward_fp8) through the C ABI.

The reference is the fp64 oracle run on the decoded FP8 weights (oracle.fp8_inputs:
E4M3 codes decoded from the format definition, times the block scales).  Shapes span
several tiles and ragged tails: d and d_ff that are not multiples of the 128- to
512-feature weight tiles, groups that are not multiples of the 16-token N step, more
than one token tile per group, two shared experts and none.  Both forms of the FP8
kernel run: the 1-SM form (the default) and the 2-SM pair (MOE_GEMM_TILES=swap_pair).
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_47_b200 as moe
import oracle
from gpu_helpers import Y_REL_TOL, dispatch_parity, oracle_rows, rel_err, route_parity
from workloads import WORKLOADS, Inputs, make_fp8, make_inputs, make_small, to_device

pytestmark = pytest.mark.gpu

FP8_SHAPES = [  # T, d, E, k, F, S, bias_scale
    (7, 128, 3, 2, 64, 1, 0.0),
    (64, 256, 16, 2, 128, 1, 0.0),
    (130, 320, 5, 3, 384, 2, 0.0),
    (300, 192, 64, 8, 192, 1, 0.5),
    (600, 256, 4, 2, 128, 1, 0.0),     # ~300 rows per expert: three token tiles each
    (40, 256, 8, 8, 128, 0, 0.0),      # k == E, no shared expert
]


def _ids(shapes):
    return ["T{}_d{}_E{}_k{}_F{}_S{}".format(*s[:6]) for s in shapes]


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def decoded_inputs(inp: Inputs, routed, shared) -> Inputs:
    """inp with its expert weights replaced by the oracle's decoding of the FP8 sets."""
    d = oracle.fp8_inputs(inp, routed, shared)
    return Inputs(inp.wl, inp.x, inp.W_router, inp.bias, _bf16(d.W_gate), _bf16(d.W_up),
                  _bf16(d.W_down), _bf16(d.Ws_gate), _bf16(d.Ws_up), _bf16(d.Ws_down))


def _forward_fp8(dev: Inputs, routed, shared):
    wl = dev.wl
    h = moe.moe_create(wl.d, wl.E, wl.k, wl.F, wl.S)
    ws = torch.empty(moe.moe_workspace_size(h, wl.T), dtype=torch.uint8, device="cuda")
    y = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward_fp8(h, dev.x, dev.W_router, dev.bias, routed, shared, y, ws)
    st, detail = moe.moe_device_status(h, wl.T, ws)
    assert st == moe.MOE_OK, hex(detail)
    return y.cpu(), {k: v.cpu() for k, v in moe.workspace_views(h, wl.T, ws).items()}


FORMS = ["pair", "swap"]


def _form(form, monkeypatch):
    if form == "pair":
        monkeypatch.setenv("MOE_GEMM_TILES", "swap_pair")
    else:
        monkeypatch.delenv("MOE_GEMM_TILES", raising=False)


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("shape", FP8_SHAPES, ids=_ids(FP8_SHAPES))
def test_fp8_expert_ffn_stage(shape, form, monkeypatch):
    """fp32 Y rows and the bf16 activations against the oracle on the decoded weights,
    given the oracle's dispatch."""
    _form(form, monkeypatch)
    T, d, E, k, F, S, bs = shape
    inp = make_small(T, d, E, k, F, S, seed=700 + T, bias_scale=bs)
    routed, shared = make_fp8(inp)
    ref_inp = decoded_inputs(inp, routed, shared)
    logits = oracle.router_logits(inp.x, inp.W_router, inp.bias)
    idx, w, _ = oracle.route(logits, k)
    counts, offsets, perm, pos = oracle.dispatch(idx, E)
    h = moe.moe_create(d, E, k, F, S)
    ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
    rows = T * k + S * T
    Y = torch.full((rows, d), float("nan"), dtype=torch.float32, device="cuda")
    moe.moe_expert_ffn_fp8(h, inp.x.cuda(), torch.from_numpy(perm).cuda(),
                           torch.from_numpy(offsets).cuda(), routed.to("cuda"),
                           shared.to("cuda"), Y, ws)
    st, detail = moe.moe_device_status(h, T, ws)
    assert st == moe.MOE_OK, hex(detail)
    H_ref, Y_ref = oracle_rows(ref_inp, idx, perm)
    Yg = Y.cpu().numpy()
    Hg = moe.workspace_views(h, T, ws)["h_act"].float().cpu().numpy()
    Yr = np.stack([Y_ref[r] for r in range(rows)])
    Hr = np.stack([H_ref[r] for r in range(rows)])
    assert np.isfinite(Yg).all()
    assert rel_err(Hg, Hr) < Y_REL_TOL, rel_err(Hg, Hr)
    assert rel_err(Yg, Yr) < Y_REL_TOL, rel_err(Yg, Yr)


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("shape", FP8_SHAPES, ids=_ids(FP8_SHAPES))
def test_fp8_forward_matches_oracle(shape, form, monkeypatch):
    _form(form, monkeypatch)
    T, d, E, k, F, S, bs = shape
    inp = make_small(T, d, E, k, F, S, seed=800 + T, bias_scale=bs)
    routed, shared = make_fp8(inp)
    y, v = _forward_fp8(to_device(inp, "cuda"), routed.to("cuda"), shared.to("cuda"))
    ref_inp = decoded_inputs(inp, routed, shared)
    logits = oracle.router_logits(inp.x, inp.W_router, inp.bias)
    exempt, idx_o, _ = route_parity(logits, v["topk_idx"].numpy(), v["topk_w"].numpy(), k)
    dispatch_parity(v["topk_idx"].numpy(), E, v["counts"], v["offsets"], v["perm"], v["pos"])
    idx_use = np.where(exempt[:, None], v["topk_idx"].numpy(), idx_o)
    ref = oracle.forward(ref_inp, idx_override=idx_use)
    assert rel_err(y.float().numpy(), ref["y"]) < Y_REL_TOL


@pytest.mark.parametrize("shape", FP8_SHAPES[1:5], ids=_ids(FP8_SHAPES[1:5]))
def test_fp8_path_equals_bf16_path_on_decoded_weights(shape, monkeypatch):
    """The FP8 kernels decode each weight exactly and then run the MMAs of the 1-SM
    weight-major bf16 kernel in the same order, so on the decoded weights the two GPU
    paths give bit-identical activations and outputs."""
    monkeypatch.setenv("MOE_GEMM_TILES", "swap")
    T, d, E, k, F, S, bs = shape
    inp = make_small(T, d, E, k, F, S, seed=900 + T, bias_scale=bs)
    routed, shared = make_fp8(inp)
    dec = to_device(decoded_inputs(inp, routed, shared), "cuda")
    y8, v8 = _forward_fp8(to_device(inp, "cuda"), routed.to("cuda"), shared.to("cuda"))
    h = moe.moe_create(d, E, k, F, S)
    ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
    y16 = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(h, dec.x, dec.W_router, dec.bias, dec.W_gate, dec.W_up, dec.W_down,
                    dec.Ws_gate, dec.Ws_up, dec.Ws_down, y16, ws)
    assert moe.moe_device_status(h, T, ws)[0] == moe.MOE_OK
    h16 = moe.workspace_views(h, T, ws)["h_act"].cpu()
    assert torch.equal(v8["h_act"].view(torch.int16), h16.view(torch.int16))
    assert torch.equal(y8.view(torch.int16), y16.cpu().view(torch.int16))


@pytest.mark.parametrize("name", ["decode_fp8", "batched_decode_fp8"])
def test_fp8_full_size_workload(name):
    """The Hy4-sized decode workloads with their FP8 checkpoint, in the launch configuration
    bench.py times; the output on a sample of tokens against the oracle (only the experts
    those tokens use are decoded on the host)."""
    wl = WORKLOADS[name]
    inp = make_inputs(wl, device="cuda")
    routed, shared = make_fp8(inp)
    y, v = _forward_fp8(inp, routed, shared)
    x_cpu = inp.x.cpu()
    logits = oracle.router_logits(x_cpu, inp.W_router.cpu(), None)
    idx_g = v["topk_idx"].numpy()
    exempt, idx_o, _ = route_parity(logits, idx_g, v["topk_w"].numpy(), wl.k)
    dispatch_parity(idx_g, wl.E, v["counts"], v["offsets"], v["perm"], v["pos"])
    yg = y.float().numpy()
    assert np.isfinite(yg).all()
    # decoding a routed expert on the host costs about a second, so the sample is 16 evenly
    # spaced tokens (all of them at T = 16) plus the last token of the most loaded expert
    idx_use = np.where(exempt[:, None], idx_g, idx_o)
    hottest = np.bincount(idx_g.reshape(-1)).argmax()
    last_hot = int(np.nonzero((idx_g == hottest).any(axis=1))[0][-1])
    tokens = np.unique(np.concatenate([
        np.linspace(0, wl.T - 1, min(16, wl.T)).round().astype(np.int32), [last_hot]]))
    w_use = oracle.renormalised_gates(logits, idx_use)
    used = sorted(set(idx_use[tokens].reshape(-1).tolist()))
    m = oracle.fp8_inputs(inp, routed, shared, experts=used)   # copies only those experts
    y_ref = oracle.moe_ffn_tokens(x_cpu, idx_use, w_use, m["W_gate"], m["W_up"], m["W_down"],
                                  m["Ws_gate"], m["Ws_up"], m["Ws_down"], tokens,
                                  E=wl.E, F=wl.F, S=wl.S)
    err = rel_err(yg[tokens], y_ref)
    print(f"{name}: exempt {int(exempt.sum())}, sampled {len(tokens)}, experts {len(used)}, "
          f"rel err {err:.3e}")
    assert err < Y_REL_TOL, err


SPECIAL_CODES = [0x00, 0x80, 0x01, 0x81, 0x07, 0x87, 0x08, 0x88, 0x7E, 0xFE, 0x38, 0xB8]


def test_fp8_special_codes_decode_exactly(monkeypatch):
    """Zero, negative zero, the smallest and largest subnormals, the smallest normal, +-448
    and +-1 planted across the gate, up and down weights (and a scale byte of 134, the
    largest the decoder accepts): the FP8 path must give exactly the bf16 path's result on
    the oracle's decoding, and match the oracle."""
    T, d, E, k, F, S = 64, 256, 4, 2, 128, 1
    inp = make_small(T, d, E, k, F, S, seed=31)
    routed, shared = make_fp8(inp)
    g = torch.Generator().manual_seed(5)
    codes = torch.tensor(SPECIAL_CODES, dtype=torch.uint8)
    for t in (routed.gate, routed.up, routed.down, shared.gate, shared.down):
        flat = t.view(-1)
        where = torch.randint(0, flat.numel(), (4096,), generator=g)
        flat[where] = codes[torch.randint(0, len(SPECIAL_CODES), (4096,), generator=g)]
    routed.gate_scale[0, 0, :8] = 134           # largest scale byte decoded exactly
    ref_inp = decoded_inputs(inp, routed, shared)
    monkeypatch.setenv("MOE_GEMM_TILES", "swap_pair")
    y8_pair, v8p = _forward_fp8(to_device(inp, "cuda"), routed.to("cuda"), shared.to("cuda"))
    ref_p = oracle.forward(ref_inp, idx_override=v8p["topk_idx"].numpy())
    assert rel_err(y8_pair.float().numpy(), ref_p["y"]) < Y_REL_TOL
    monkeypatch.setenv("MOE_GEMM_TILES", "swap")
    y8, v8 = _forward_fp8(to_device(inp, "cuda"), routed.to("cuda"), shared.to("cuda"))
    dec = to_device(ref_inp, "cuda")
    h = moe.moe_create(d, E, k, F, S)
    ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
    y16 = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(h, dec.x, dec.W_router, dec.bias, dec.W_gate, dec.W_up, dec.W_down,
                    dec.Ws_gate, dec.Ws_up, dec.Ws_down, y16, ws)
    assert moe.moe_device_status(h, T, ws)[0] == moe.MOE_OK
    assert torch.equal(y8.view(torch.int16), y16.cpu().view(torch.int16))
    ref = oracle.forward(ref_inp, idx_override=v8["topk_idx"].numpy())
    assert rel_err(y8.float().numpy(), ref["y"]) < Y_REL_TOL


@pytest.mark.parametrize("name", ["decode_fp8"])
def test_fp8_pair_and_single_forms_agree_at_full_size(name, monkeypatch):
    """The 2-SM and 1-SM FP8 kernels on the Hy4 decode workload: the same routing and
    outputs within the layer's tolerance of each other (the pair's M = 256 MMAs may order
    the tensor core's partial sums differently from two M = 128 ones)."""
    wl = WORKLOADS[name]
    inp = make_inputs(wl, device="cuda")
    routed, shared = make_fp8(inp)
    monkeypatch.setenv("MOE_GEMM_TILES", "swap_pair")
    y_pair, v_pair = _forward_fp8(inp, routed, shared)
    monkeypatch.delenv("MOE_GEMM_TILES", raising=False)
    y_one, v_one = _forward_fp8(inp, routed, shared)
    assert torch.equal(v_pair["topk_idx"], v_one["topk_idx"])
    err = rel_err(y_pair.float().numpy(), y_one.float().numpy())
    same = torch.equal(y_pair.view(torch.int16), y_one.view(torch.int16))
    print(f"{name}: pair vs 1-SM FP8 rel diff {err:.3e}, bit-identical {same}")
    assert err < Y_REL_TOL
