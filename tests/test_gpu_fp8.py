"""GPU parity of the FP8-weight path (moe_expert_ffn_fp8, moe_forward_fp8) through the C ABI.

The reference is the fp64 oracle run on the decoded FP8 weights (oracle.fp8_inputs:
E4M3 codes decoded from the format definition, times the block scales).  Shapes span
several tiles and ragged tails: d and d_ff that are not multiples of the 128- to
512-feature weight tiles, groups that are not multiples of the 16-token N step, more
than one token tile per group, two shared experts and none.  Every form of the FP8 path
runs: the tcgen05 kernel's 1-SM form (MOE_GEMM_TILES=swap, and the default above 16
tokens) and 2-SM pair (MOE_GEMM_TILES=swap_pair), and the warp-MMA form the default takes
at up to 16 tokens, whose shapes add K lengths of fewer 64-wide blocks than a CTA has warps,
groups of 1 to 8 tokens (one 8-token unit) and of 9 to 16 (two units).
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
    # up to 16 tokens: the default takes the warp-MMA form
    (16, 320, 5, 3, 384, 2, 0.0),      # K = 320 and 384: 5 and 6 blocks of 64 for 8 warps
    (1, 64, 1, 1, 64, 0, 0.0),         # one token, one expert, one K block: the smallest shape
    (12, 192, 64, 8, 192, 1, 0.5),     # most groups empty or of one token
    (13, 128, 2, 1, 128, 1, 0.0),      # routed groups of 6-7 tokens, the shared one of 13 (two units)
    (16, 64, 1024, 8, 64, 1, 0.0),     # 1024 experts: ~120 non-empty groups, the unit table's limit
    (16, 128, 8, 8, 64, 0, 0.0),       # k == E, no shared expert: every group two 8-token units
]
GEMV_SHAPES = [s for s in FP8_SHAPES if s[0] <= 16]


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


FORMS = ["pair", "swap", "auto"]


def _form(form, monkeypatch):
    """pair: the tensor-core kernel's 2-SM form; swap: its 1-SM form; auto: the default
    (the warp-MMA form at up to 16 tokens, else the tcgen05 kernel's 1-SM form)."""
    if form == "pair":
        monkeypatch.setenv("MOE_GEMM_TILES", "swap_pair")
    elif form == "swap":
        monkeypatch.setenv("MOE_GEMM_TILES", "swap")
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


@pytest.mark.parametrize("shape", FP8_SHAPES[1:5] + GEMV_SHAPES[:1],
                         ids=_ids(FP8_SHAPES[1:5] + GEMV_SHAPES[:1]))
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
def test_fp8_forms_agree_at_full_size(name, monkeypatch):
    """The three FP8 forms on the Hy4 decode workload: the same routing, and the 2-SM
    tcgen05 kernel and the warp-MMA form (the default at 16 tokens) each within the
    layer's tolerance of the 1-SM tensor-core kernel (the pair's M = 256 MMAs and the
    CUDA cores' lane-by-lane sums may order the fp32 additions differently)."""
    wl = WORKLOADS[name]
    inp = make_inputs(wl, device="cuda")
    routed, shared = make_fp8(inp)
    out = {}
    for form in FORMS:
        _form(form, monkeypatch)
        out[form] = _forward_fp8(inp, routed, shared)
    y_one, v_one = out["swap"]
    for form in ("pair", "auto"):
        y, v = out[form]
        assert torch.equal(v["topk_idx"], v_one["topk_idx"])
        err = rel_err(y.float().numpy(), y_one.float().numpy())
        same = torch.equal(y.view(torch.int16), y_one.view(torch.int16))
        print(f"{name}: {form} vs 1-SM FP8 rel diff {err:.3e}, bit-identical {same}")
        assert err < Y_REL_TOL


def _bf16_ulps(a: torch.Tensor, b: torch.Tensor) -> torch.Tensor:
    """Distance in bf16 steps between two bf16 tensors of finite values (sign-magnitude
    bit patterns mapped to a monotone integer line)."""
    def line(t):
        i = t.view(torch.int16).to(torch.int32)
        return torch.where(i < 0, -(i & 0x7FFF), i)
    return (line(a) - line(b)).abs()


@pytest.mark.parametrize("shape", GEMV_SHAPES, ids=_ids(GEMV_SHAPES))
def test_fp8_gemv_matches_tensor_core_form(shape, monkeypatch):
    """The warp-MMA form forms the same exact bf16 x bf16 products as the tcgen05
    kernel and adds them in fp32 in another order, so on the same dispatch its fp32 sums
    differ from the tensor core's by a few fp32 rounding steps: every bf16 activation is the
    tensor-core one or its neighbour, nearly all are equal, and the fp32 Y rows agree to far
    within the layer's tolerance."""
    T, d, E, k, F, S, bs = shape
    inp = make_small(T, d, E, k, F, S, seed=1700 + T, bias_scale=bs)
    routed, shared = make_fp8(inp)
    logits = oracle.router_logits(inp.x, inp.W_router, inp.bias)
    idx, _, _ = oracle.route(logits, k)
    _, offsets, perm, _ = oracle.dispatch(idx, E)
    rows = T * k + S * T
    res = {}
    for form in ("swap", "auto"):
        _form(form, monkeypatch)
        h = moe.moe_create(d, E, k, F, S)
        ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
        Y = torch.full((rows, d), float("nan"), dtype=torch.float32, device="cuda")
        moe.moe_expert_ffn_fp8(h, inp.x.cuda(), torch.from_numpy(perm).cuda(),
                               torch.from_numpy(offsets).cuda(), routed.to("cuda"),
                               shared.to("cuda"), Y, ws)
        assert moe.moe_device_status(h, T, ws)[0] == moe.MOE_OK
        res[form] = (moe.workspace_views(h, T, ws)["h_act"][:rows].cpu(), Y.cpu())
    (h_tc, y_tc), (h_cc, y_cc) = res["swap"], res["auto"]
    ulps = _bf16_ulps(h_cc, h_tc)
    assert int(ulps.max()) <= 1, int(ulps.max())
    assert float((ulps > 0).float().mean()) < 0.02
    assert torch.isfinite(y_cc).all()
    assert rel_err(y_cc.numpy(), y_tc.numpy()) < 1e-3


def test_fp8_gemv_special_codes(monkeypatch):
    """The special codes and the largest scale byte of test_fp8_special_codes_decode_exactly
    through the warp-MMA form (16 tokens): within the layer's tolerance of the oracle on
    the decoded weights."""
    T, d, E, k, F, S = 16, 256, 4, 2, 128, 1
    inp = make_small(T, d, E, k, F, S, seed=37)
    routed, shared = make_fp8(inp)
    g = torch.Generator().manual_seed(6)
    codes = torch.tensor(SPECIAL_CODES, dtype=torch.uint8)
    for t in (routed.gate, routed.up, routed.down, shared.gate, shared.up, shared.down):
        flat = t.view(-1)
        where = torch.randint(0, flat.numel(), (4096,), generator=g)
        flat[where] = codes[torch.randint(0, len(SPECIAL_CODES), (4096,), generator=g)]
    routed.gate_scale[0, 0, :8] = 134
    shared.down_scale[0, 0, :8] = 134
    monkeypatch.delenv("MOE_GEMM_TILES", raising=False)
    y8, v8 = _forward_fp8(to_device(inp, "cuda"), routed.to("cuda"), shared.to("cuda"))
    ref = oracle.forward(decoded_inputs(inp, routed, shared), idx_override=v8["topk_idx"].numpy())
    assert rel_err(y8.float().numpy(), ref["y"]) < Y_REL_TOL


@pytest.mark.parametrize("shape", [FP8_SHAPES[1], GEMV_SHAPES[0]], ids=_ids([FP8_SHAPES[1], GEMV_SHAPES[0]]))
def test_fp8_host_activations_match_the_device_call(shape):
    """moe_forward_fp8_host (pinned host x in, host y out) gives moe_forward_fp8's bits, for the
    tcgen05 form (64 tokens) and the warp-MMA form (7 tokens).  Calls are enqueued back to back
    without synchronising, each on its own input, so the staging slots alternate while earlier
    layers still run; every output is its own input's."""
    T, d, E, k, F, S, bs = shape
    inputs = [make_small(T, d, E, k, F, S, seed=1900 + T + i, bias_scale=bs) for i in range(3)]
    routed, shared = make_fp8(inputs[0])
    routed, shared = routed.to("cuda"), shared.to("cuda")
    dev = to_device(inputs[0], "cuda")
    h = moe.moe_create(d, E, k, F, S)
    ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
    want = []
    for inp in inputs:
        y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
        moe.moe_forward_fp8(h, inp.x.cuda(), dev.W_router, dev.bias, routed, shared, y, ws)
        want.append(y.cpu())
    xs = [inp.x.pin_memory() for inp in inputs]
    ys = [torch.full((T, d), float("nan"), dtype=torch.bfloat16).pin_memory() for _ in inputs]
    for _ in range(2):
        for x, y in zip(xs, ys):
            moe.moe_forward_fp8_host(h, x, dev.W_router, dev.bias, routed, shared, y, ws)
    torch.cuda.synchronize()
    st, detail = moe.moe_device_status(h, T, ws)
    assert st == moe.MOE_OK, hex(detail)
    for y, w in zip(ys, want):
        assert torch.equal(y.view(torch.int16), w.view(torch.int16))
