"""GPU parity of every step of the CUDA path against the fp64 oracle, through the C ABI.

Sizes span several tiles and ragged tails (groups not a multiple of the GEMMs'
128- or 256-row tiles or 16-token N step, d_ff not a multiple of the 128- or
256-feature gate/up tile, d not a multiple of the 256-feature down tile, dispatch
runs over more than one 4096-slot block) plus the degenerate cases (one token,
one expert, k = E, no shared expert, every token on one expert, an empty expert).
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_47_b200 as moe
import oracle
from gpu_helpers import (Y_REL_TOL, bad_index_routing, check_skipped_slots, dispatch_parity,
                         gpu_forward, oracle_rows, rel_err, route_parity)
from workloads import WORKLOADS, Inputs, make_inputs, make_small, to_device

pytestmark = pytest.mark.gpu

SHAPES = [  # T, d, E, k, F, S, bias_scale
    (1, 64, 1, 1, 64, 0, 0.0),
    (7, 128, 3, 2, 64, 1, 0.0),
    (64, 256, 16, 2, 128, 1, 0.0),
    (300, 192, 64, 8, 192, 1, 0.5),
    (130, 320, 5, 3, 384, 2, 0.0),
    (513, 512, 64, 8, 256, 1, 0.2),
    (40, 256, 8, 8, 128, 1, 0.0),      # k == E
    # T*k >= 96*E: the default 2-SM (cta_group::2) weight-major GEMM path
    (600, 256, 4, 2, 128, 1, 0.0),     # ~300 rows per expert: two pair tiles, ragged tail
    (200, 320, 2, 2, 192, 2, 0.0),     # k == E, every group 200 rows; two shared experts
    (1000, 128, 8, 2, 64, 1, 0.3),     # d_ff = 64: half of each gate/up tile masked
]


def _ids(shapes):
    return ["T{}_d{}_E{}_k{}_F{}_S{}".format(*s[:6]) for s in shapes]


@pytest.mark.parametrize("shape", SHAPES, ids=_ids(SHAPES))
def test_route_stage(shape):
    T, d, E, k, F, S, bs = shape
    inp = make_small(T, d, E, k, F, S, seed=100 + T, bias_scale=bs)
    dev = to_device(inp, "cuda")
    h = moe.moe_create(d, E, k, F, S)
    ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    moe.moe_route(h, dev.x, dev.W_router, dev.bias, idx, w, ws)
    torch.cuda.synchronize()
    logits = oracle.router_logits(inp.x, inp.W_router, inp.bias)
    route_parity(logits, idx.cpu().numpy(), w.cpu().numpy(), k)


ROUTER_SHAPES = [  # T, d, E, router init, bias scale
    (16, 6144, 256, "normal", 0.0),
    (513, 6144, 256, "uniform", 0.0),
    (300, 192, 64, "normal", 0.5),
    (70, 320, 5, "uniform", 0.0),
]


@pytest.mark.parametrize("path", ["tc", "ffma"])
@pytest.mark.parametrize("shape", ROUTER_SHAPES, ids=lambda s: "T{}_d{}_E{}_{}".format(*s[:4]))
def test_router_logit_accuracy(shape, path, monkeypatch):
    """Both score-GEMM paths (tensor cores with exact three-way bf16 split of W_r, and fp32
    FFMA) against the fp64 logits.  The bar is half the 1e-5 margin below which a token's
    routing is exempt, so no non-exempt token can change its experts through logit error."""
    monkeypatch.setenv("MOE_ROUTER", path)
    T, d, E, router, bs = shape
    inp = make_small(T, d, E, min(8, E), 64, 1, seed=400 + T, router=router, bias_scale=bs)
    dev = to_device(inp, "cuda")
    h = moe.moe_create(d, E, min(8, E), 64, 1)
    ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
    idx = torch.empty(T, h.k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, h.k, dtype=torch.float32, device="cuda")
    moe.moe_route(h, dev.x, dev.W_router, dev.bias, idx, w, ws)
    st, detail = moe.moe_device_status(h, T, ws)
    assert st == moe.MOE_OK, hex(detail)
    parts = moe.workspace_views(h, T, ws)["router_partials"].cpu().double().numpy()
    got = parts.sum(0)
    ref = oracle.router_logits(inp.x, inp.W_router, None)   # the bias is added by the top-k
    err = np.abs(got - ref).max()
    print(f"{path} T={T} d={d} E={E}: max |logit err| {err:.3e}, ksplit {parts.shape[0]}")
    assert err < 5e-6, err
    route_parity(oracle.router_logits(inp.x, inp.W_router, inp.bias), idx.cpu().numpy(),
                 w.cpu().numpy(), h.k)


TILINGS = ["single", "pair", "swap", "swap_pair"]


@pytest.mark.parametrize("tiles", TILINGS)
@pytest.mark.parametrize("shape", [(64, 256, 16, 2, 128, 1, 0.0), (600, 256, 4, 2, 128, 1, 0.0),
                                   (130, 320, 5, 3, 384, 2, 0.0)],
                         ids=lambda s: "T{}_d{}_E{}_k{}_F{}_S{}".format(*s[:6]))
def test_forward_all_gemm_tilings(shape, tiles, monkeypatch):
    """The row-tiled 1-SM (128-row) and 2-SM (256-row, cta_group::2) GEMMs and the
    weight-major GEMMs (weights on the MMA's M side; 1-SM token tiles of N <= 128, 2-SM
    token tiles of N <= 256) on the same inputs."""
    monkeypatch.setenv("MOE_GEMM_TILES", tiles)
    T, d, E, k, F, S, bs = shape
    inp = make_small(T, d, E, k, F, S, seed=500 + T, bias_scale=bs)
    y, v = gpu_forward(to_device(inp, "cuda"))
    logits = oracle.router_logits(inp.x, inp.W_router, inp.bias)
    exempt, idx_o, _ = route_parity(logits, v["topk_idx"].numpy(), v["topk_w"].numpy(), k)
    idx_use = np.where(exempt[:, None], v["topk_idx"].numpy(), idx_o)
    ref = oracle.forward(inp, idx_override=idx_use)
    assert rel_err(y.float().numpy(), ref["y"]) < Y_REL_TOL


@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (5, 3, 2), (64, 16, 2), (700, 64, 8),
                                   (1500, 256, 8), (2000, 1024, 32), (8192, 256, 8)])
def test_dispatch_stage(T, E, k):
    g = torch.Generator().manual_seed(T * 7 + E)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    h = moe.moe_create(64, E, k, 64, 1)
    ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    pos = torch.empty(T * k, dtype=torch.int32, device="cuda")
    moe.moe_dispatch(h, idx.cuda(), counts, offsets, perm, pos, ws)
    st, _ = moe.moe_device_status(h, T, ws)
    assert st == moe.MOE_OK
    dispatch_parity(idx.numpy(), E, counts.cpu(), offsets.cpu(), perm.cpu(), pos.cpu())


@pytest.mark.parametrize("T,E,k", [(10, 8, 2), (900, 64, 8), (64, 512, 8)])
def test_dispatch_flags_and_skips_out_of_range_index(T, E, k):
    """Out-of-range expert indices (one CTA path, three-kernel path, E > 256) are flagged
    MOE_ERR_BAD_INDEX, get pos = -1 and are left out of every segment."""
    idx = bad_index_routing(T, E, k, seed=T + E)
    h = moe.moe_create(64, E, k, 64, 1)
    ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
    out = [torch.full((n,), -7, dtype=torch.int32, device="cuda")
           for n in (E, E + 1, T * k, T * k)]
    moe.moe_dispatch(h, idx.cuda(), *out, ws)
    st, detail = moe.moe_device_status(h, T, ws)
    assert st == moe.MOE_ERR_BAD_INDEX and (detail >> 16) == 2
    check_skipped_slots(idx.numpy(), E, *[o.cpu().numpy() for o in out])


def test_combine_leaves_out_skipped_slots():
    """A slot with pos = -1 (an out-of-range index that dispatch skipped) adds nothing: the
    combine equals the oracle's with that slot's gate set to zero."""
    T, E, k, S, d = 40, 8, 2, 1, 256
    idx = bad_index_routing(T, E, k, seed=77)
    h = moe.moe_create(d, E, k, 64, S)
    ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
    out = [torch.empty(n, dtype=torch.int32, device="cuda") for n in (E, E + 1, T * k, T * k)]
    moe.moe_dispatch(h, idx.cuda(), *out, ws)
    pos = out[3]
    g = torch.Generator().manual_seed(5)
    Y = torch.randn(T * k + S * T, d, generator=g)
    w = torch.rand(T, k, generator=g)
    y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(h, Y.cuda(), w.cuda(), pos, y)
    torch.cuda.synchronize()
    pos_c = pos.cpu().numpy()
    skipped = pos_c < 0
    assert skipped.any()
    w_ref = w.double().numpy().reshape(-1).copy()
    w_ref[skipped] = 0.0
    pos_ref = np.where(skipped, 0, pos_c).astype(np.int32)
    ref = oracle.combine(Y.double().numpy(), w_ref.reshape(T, k), pos_ref, T, k, S)
    got = y.float().cpu().numpy()
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6)


@pytest.mark.parametrize("tiles", TILINGS)
@pytest.mark.parametrize("shape", SHAPES, ids=_ids(SHAPES))
def test_expert_ffn_stage(shape, tiles, monkeypatch):
    """Y rows (fp32) and the bf16 SwiGLU activations against the oracle, given the oracle's
    dispatch, for each GEMM tiling."""
    monkeypatch.setenv("MOE_GEMM_TILES", tiles)
    T, d, E, k, F, S, bs = shape
    inp = make_small(T, d, E, k, F, S, seed=200 + T, bias_scale=bs)
    dev = to_device(inp, "cuda")
    logits = oracle.router_logits(inp.x, inp.W_router, inp.bias)
    idx, w, _ = oracle.route(logits, k)
    counts, offsets, perm, pos = oracle.dispatch(idx, E)
    h = moe.moe_create(d, E, k, F, S)
    ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
    rows = T * k + S * T
    Y = torch.full((rows, d), float("nan"), dtype=torch.float32, device="cuda")
    moe.moe_expert_ffn(h, dev.x, torch.from_numpy(perm).cuda(), torch.from_numpy(offsets).cuda(),
                       dev.W_gate, dev.W_up, dev.W_down, dev.Ws_gate, dev.Ws_up, dev.Ws_down, Y,
                       ws)
    st, detail = moe.moe_device_status(h, T, ws)
    assert st == moe.MOE_OK, hex(detail)
    views = moe.workspace_views(h, T, ws)
    H_ref, Y_ref = oracle_rows(inp, idx, perm)
    Yg = Y.cpu().numpy()
    Hg = views["h_act"].float().cpu().numpy()
    Yr = np.stack([Y_ref[r] for r in range(rows)])
    Hr = np.stack([H_ref[r] for r in range(rows)])
    assert np.isfinite(Yg).all()
    assert rel_err(Hg, Hr) < Y_REL_TOL, rel_err(Hg, Hr)
    assert rel_err(Yg, Yr) < Y_REL_TOL, rel_err(Yg, Yr)


@pytest.mark.parametrize("T,k,S,d", [(1, 1, 0, 64), (64, 2, 1, 256), (33, 8, 2, 6144)])
def test_combine_stage(T, k, S, d):
    g = torch.Generator().manual_seed(T + k)
    rows = T * k + S * T
    Y = torch.randn(rows, d, generator=g)
    w = torch.rand(T, k, generator=g)
    w = w / w.sum(1, keepdim=True)
    pos = torch.randperm(T * k, generator=g).to(torch.int32)
    h = moe.moe_create(d, max(k, 2), k, 64, S)
    y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(h, Y.cuda(), w.cuda(), pos.cuda(), y)
    torch.cuda.synchronize()
    ref = oracle.combine(Y.double().numpy(), w.double().numpy(), pos.numpy(), T, k, S)
    got = y.float().cpu().numpy()
    # fp32 accumulation then one bf16 rounding: within 2^-8 relative of each element
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6)


@pytest.mark.parametrize("shape", SHAPES, ids=_ids(SHAPES))
def test_forward_matches_oracle(shape):
    T, d, E, k, F, S, bs = shape
    inp = make_small(T, d, E, k, F, S, seed=300 + T, bias_scale=bs)
    y, v = gpu_forward(to_device(inp, "cuda"))
    logits = oracle.router_logits(inp.x, inp.W_router, inp.bias)
    exempt, idx_o, _ = route_parity(logits, v["topk_idx"].numpy(), v["topk_w"].numpy(), k)
    dispatch_parity(v["topk_idx"].numpy(), E, v["counts"], v["offsets"], v["perm"], v["pos"])
    # exempt (near-tie) tokens are compared with the oracle rerun on the GPU's routing
    idx_use = np.where(exempt[:, None], v["topk_idx"].numpy(), idx_o)
    ref = oracle.forward(inp, idx_override=idx_use)
    assert rel_err(y.float().numpy(), ref["y"]) < Y_REL_TOL


def test_forward_tiny_workload():
    """The tiny workload (T=64, d=256, 16 experts top-2 + 1 shared, d_ff=128, seed 0)."""
    inp = make_inputs(WORKLOADS["tiny"], device="cpu")
    y, v = gpu_forward(to_device(inp, "cuda"))
    ref = oracle.forward(inp)
    exempt, _, _ = route_parity(ref["logits"], v["topk_idx"].numpy(), v["topk_w"].numpy(), 2)
    if not exempt.any():
        np.testing.assert_array_equal(v["offsets"].numpy(), ref["offsets"])
        np.testing.assert_array_equal(v["perm"].numpy(), ref["perm"])
    err = rel_err(y.float().numpy(), ref["y"])
    assert err < Y_REL_TOL, err


@pytest.mark.parametrize("tiles", ["single", "swap", "swap_pair"])
def test_every_token_on_one_expert_and_empty_experts(tiles, monkeypatch):
    """Dominant biases send all 300 tokens to experts 3 and 7 (3 M tiles of 128 rows each,
    3 token tiles of 112, 112 and 76 tokens, or 2 pair token tiles of 160 and 140); the
    other 14 experts stay empty."""
    monkeypatch.setenv("MOE_GEMM_TILES", tiles)
    T, d, E, k, F, S = 300, 128, 16, 2, 128, 1
    inp = make_small(T, d, E, k, F, S, seed=9)
    bias = torch.zeros(E)
    bias[3] = 50.0
    bias[7] = 40.0
    inp = Inputs(inp.wl, inp.x, inp.W_router, bias, inp.W_gate, inp.W_up, inp.W_down,
                 inp.Ws_gate, inp.Ws_up, inp.Ws_down)
    y, v = gpu_forward(to_device(inp, "cuda"))
    assert int(v["counts"][3]) == T and int(v["counts"][7]) == T
    assert int((v["counts"] == 0).sum()) == E - 2
    ref = oracle.forward(inp)
    route_parity(ref["logits"], v["topk_idx"].numpy(), v["topk_w"].numpy(), k)
    assert rel_err(y.float().numpy(), ref["y"]) < Y_REL_TOL


@pytest.mark.parametrize("tiles", ["pair", "swap_pair"])
def test_pair_tiles_hot_experts_and_empty_experts(tiles, monkeypatch):
    """2-SM paths: two experts take all 700 tokens (3 row tiles of 256, 256, 188 rows, or 3
    token tiles of 240, 240, 220) and the other two stay empty."""
    monkeypatch.setenv("MOE_GEMM_TILES", tiles)
    T, d, E, k, F, S = 700, 256, 4, 2, 128, 1
    inp = make_small(T, d, E, k, F, S, seed=19)
    bias = torch.tensor([0.0, 50.0, 0.0, 40.0])
    inp = Inputs(inp.wl, inp.x, inp.W_router, bias, inp.W_gate, inp.W_up, inp.W_down,
                 inp.Ws_gate, inp.Ws_up, inp.Ws_down)
    y, v = gpu_forward(to_device(inp, "cuda"))
    assert v["counts"].tolist() == [0, T, 0, T]
    ref = oracle.forward(inp)
    route_parity(ref["logits"], v["topk_idx"].numpy(), v["topk_w"].numpy(), k)
    assert rel_err(y.float().numpy(), ref["y"]) < Y_REL_TOL


def test_forward_is_deterministic_and_host_io_matches():
    inp = to_device(make_small(200, 256, 32, 4, 128, 1, seed=5), "cuda")
    wl = inp.wl
    h = moe.moe_create(wl.d, wl.E, wl.k, wl.F, wl.S)
    ws = torch.empty(moe.moe_workspace_size(h, wl.T), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(2):
        y = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device="cuda")
        moe.moe_forward(h, inp.x, inp.W_router, inp.bias, inp.W_gate, inp.W_up, inp.W_down,
                        inp.Ws_gate, inp.Ws_up, inp.Ws_down, y, ws)
        outs.append(y.cpu())
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    x_host = inp.x.cpu().pin_memory()
    y_host = torch.empty(wl.T, wl.d, dtype=torch.bfloat16).pin_memory()
    moe.moe_forward_host(h, x_host, inp.W_router, inp.bias, inp.W_gate, inp.W_up, inp.W_down,
                         inp.Ws_gate, inp.Ws_up, inp.Ws_down, y_host, ws)
    torch.cuda.synchronize()
    assert torch.equal(y_host.view(torch.int16), outs[0].view(torch.int16))


def test_bounded_wait_expires_with_a_status_and_the_device_stays_usable():
    """Failure detection without a GPU fault: a wait that nothing completes gives up after
    its limit (50 ms here), the host reads MOE_ERR_TIMEOUT, and the next forward is correct."""
    h = moe.moe_create(256, 16, 2, 128, 1)
    T = 64
    ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
    moe.moe_selftest_wait_timeout(ws, 50_000_000)
    st, detail = moe.moe_device_status(h, T, ws)
    assert st == moe.MOE_ERR_TIMEOUT and (detail >> 16) == 1, (st, hex(detail))
    inp = make_inputs(WORKLOADS["tiny"], device="cpu")
    y, v = gpu_forward(to_device(inp, "cuda"))          # status cleared, results correct
    ref = oracle.forward(inp)
    assert rel_err(y.float().numpy(), ref["y"]) < Y_REL_TOL


def test_zero_tokens_is_a_no_op():
    h = moe.moe_create(256, 16, 2, 128, 1)
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    x = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    W = make_small(1, 256, 16, 2, 128, 1)
    dev = to_device(W, "cuda")
    y = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(h, x, dev.W_router, None, dev.W_gate, dev.W_up, dev.W_down, dev.Ws_gate,
                    dev.Ws_up, dev.Ws_down, y, ws)
    torch.cuda.synchronize()


def test_back_to_back_host_calls_keep_each_input():
    """moe_forward_host calls enqueued without synchronising, each on its own pinned input:
    the input copies run ahead on the context's helper stream into two staging slots used in
    turn, so a slot must not be overwritten before the layer that reads it is done.  A long
    wait kernel on the stream first lets the copies run far ahead; every output must still
    equal moe_forward's on its own input."""
    wl_inp = make_small(96, 256, 16, 2, 128, 1, seed=61)
    dev = to_device(wl_inp, "cuda")
    wl = wl_inp.wl
    h = moe.moe_create(wl.d, wl.E, wl.k, wl.F, wl.S)
    ws = torch.empty(moe.moe_workspace_size(h, wl.T), dtype=torch.uint8, device="cuda")
    W = (dev.W_gate, dev.W_up, dev.W_down, dev.Ws_gate, dev.Ws_up, dev.Ws_down)
    g = torch.Generator().manual_seed(8)
    xs = [torch.randn(wl.T, wl.d, generator=g).to(torch.bfloat16).pin_memory() for _ in range(5)]
    ys = [torch.empty(wl.T, wl.d, dtype=torch.bfloat16).pin_memory() for _ in range(5)]
    torch.cuda.synchronize()
    torch.cuda._sleep(50_000_000)                    # ~25 ms of spinning on the stream
    for x, y in zip(xs, ys):
        moe.moe_forward_host(h, x, dev.W_router, dev.bias, *W, y, ws)
    torch.cuda.synchronize()
    for x, y in zip(xs, ys):
        ref = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device="cuda")
        moe.moe_forward(h, x.cuda(), dev.W_router, dev.bias, *W, ref, ws)
        torch.cuda.synchronize()
        assert torch.equal(ref.cpu().view(torch.int16), y.view(torch.int16))
    assert moe.moe_device_status(h, wl.T, ws)[0] == moe.MOE_OK


def test_host_calls_on_two_streams_each_with_its_own_workspace():
    """moe_forward_host calls alternating two streams, each with its own workspace and output
    buffer, enqueued without synchronising (as a serving loop that overlaps one call's output
    copy with the next call's layer): the calls may run at once, and every output must still
    equal moe_forward's on its own input."""
    wl_inp = make_small(160, 256, 16, 2, 128, 1, seed=67)
    dev = to_device(wl_inp, "cuda")
    wl = wl_inp.wl
    h = moe.moe_create(wl.d, wl.E, wl.k, wl.F, wl.S)
    size = moe.moe_workspace_size(h, wl.T)
    lanes = [(torch.cuda.current_stream(), torch.empty(size, dtype=torch.uint8, device="cuda")),
             (torch.cuda.Stream(), torch.empty(size, dtype=torch.uint8, device="cuda"))]
    W = (dev.W_gate, dev.W_up, dev.W_down, dev.Ws_gate, dev.Ws_up, dev.Ws_down)
    g = torch.Generator().manual_seed(9)
    xs = [torch.randn(wl.T, wl.d, generator=g).to(torch.bfloat16).pin_memory() for _ in range(7)]
    ys = [torch.empty(wl.T, wl.d, dtype=torch.bfloat16).pin_memory() for _ in range(7)]
    torch.cuda.synchronize()
    with torch.cuda.stream(lanes[0][0]):
        torch.cuda._sleep(20_000_000)                # the first stream starts late
    for i, (x, y) in enumerate(zip(xs, ys)):
        st, ws = lanes[i & 1]
        moe.moe_forward_host(h, x, dev.W_router, dev.bias, *W, y, ws, st)
    torch.cuda.synchronize()
    ws = lanes[0][1]
    for x, y in zip(xs, ys):
        ref = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device="cuda")
        moe.moe_forward(h, x.cuda(), dev.W_router, dev.bias, *W, ref, ws)
        torch.cuda.synchronize()
        assert torch.equal(ref.cpu().view(torch.int16), y.view(torch.int16))
    for _, ws in lanes:
        assert moe.moe_device_status(h, wl.T, ws)[0] == moe.MOE_OK
