"""Pins of the fp64 oracle against values fixed independently of it.

Each test checks the oracle against something other than itself: a
hand-derived closed form (tests/golden), a float64 library routine on a
special case that reduces to it, brute force on tiny inputs, or an invariant
the method guarantees.  Together they are chosen so that a dropped term, a
wrong sign or index, or a transposed operand in any oracle step fails one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import Inputs, Workload, make_small

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _sig(z):
    return 1.0 / (1.0 + math.exp(-z))


def _ev(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"sig": _sig, "exp": math.exp}))


def _bf16(a):
    return torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)


def _fixture_inputs(fx) -> Inputs:
    wl = Workload("hand", T=fx["T"], d=fx["d"], E=fx["E"], k=fx["k"], F=fx["F"], S=fx["S"])
    return Inputs(wl, _bf16(fx["x"]), torch.tensor(fx["W_router"], dtype=torch.float32), None,
                  _bf16(fx["W_gate"]), _bf16(fx["W_up"]), _bf16(fx["W_down"]),
                  _bf16(fx["Ws_gate"]), _bf16(fx["Ws_up"]), _bf16(fx["Ws_down"]))


def test_hand_worked_example():
    """Every stage of the oracle against the closed forms worked out by hand."""
    with open(os.path.join(GOLDEN, "hand_worked_T2_d3_E3_k2_F2_S1.json")) as f:
        fx = json.load(f)
    inp = _fixture_inputs(fx)
    out = oracle.forward(inp)
    ex = fx["expect"]
    np.testing.assert_array_equal(out["logits"], [[_ev(v) for v in r] for r in ex["logits"]])
    np.testing.assert_array_equal(out["idx"], ex["idx"])
    np.testing.assert_allclose(out["w"], [[_ev(v) for v in r] for r in ex["w"]], rtol=1e-14)
    np.testing.assert_array_equal(out["margin"], [_ev(v) for v in ex["margin"]])
    for key in ("counts", "offsets", "perm", "pos"):
        np.testing.assert_array_equal(out[key], ex[key], err_msg=key)
    np.testing.assert_allclose(out["y"], [[_ev(v) for v in r] for r in ex["y"]],
                               rtol=1e-14, atol=1e-15)
    h, y = oracle.expert_one(inp.x[0], inp.W_gate[1], inp.W_up[1], inp.W_down[1])
    np.testing.assert_allclose(h, [_ev(v) for v in ex["h_token0_e1"]], rtol=1e-14)
    np.testing.assert_allclose(y, [_ev(v) for v in ex["y_token0_e1"]], rtol=1e-14)
    # the combine step alone, fed the per-(slot, expert) rows in dispatch order
    T, k, S = fx["T"], fx["k"], fx["S"]
    rows = np.zeros((T * k + S * T, fx["d"]))
    for p, s in enumerate(ex["perm"]):
        t, i = divmod(s, k)
        e = ex["idx"][t][i]
        rows[p] = oracle.expert_one(inp.x[t], inp.W_gate[e], inp.W_up[e], inp.W_down[e])[1]
    for t in range(T):
        rows[T * k + t] = oracle.expert_one(inp.x[t], inp.Ws_gate[0], inp.Ws_up[0],
                                            inp.Ws_down[0])[1]
    yc = oracle.combine(rows, out["w"], out["pos"], T, k, S)
    np.testing.assert_allclose(yc, [[_ev(v) for v in r] for r in ex["y"]], rtol=1e-14,
                               atol=1e-15)


def test_router_logits_equal_float64_matmul():
    inp = make_small(T=37, d=96, E=11, k=3, F=64, S=1, seed=3, bias_scale=0.5)
    got = oracle.router_logits(inp.x, inp.W_router, inp.bias)
    ref = (inp.x.double() @ inp.W_router.double().T + inp.bias.double()).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-13)
    got_nb = oracle.router_logits(inp.x, inp.W_router, None)
    np.testing.assert_allclose(got_nb, (inp.x.double() @ inp.W_router.double().T).numpy(),
                               rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("E,k", [(1, 1), (5, 2), (16, 4), (64, 4), (64, 8), (9, 9)])
def test_topk_brute_force_with_ties(E, k):
    """Top-k equals a full sort by (logit desc, expert asc); ties are frequent here."""
    rng = np.random.default_rng(E * 100 + k)
    T = 200
    logits = rng.integers(-3, 4, size=(T, E)).astype(np.float64) * 0.25  # many exact ties
    idx, w, margin = oracle.route(logits, k)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-logits[t, e], e))
        assert list(idx[t]) == order[:k]
        if k < E:
            assert margin[t] == logits[t, order[k - 1]] - logits[t, order[k]]
        else:
            assert margin[t] == math.inf
        sel = logits[t, order[:k]]
        ref_w = np.exp(sel - sel.max()) / np.exp(sel - sel.max()).sum()  # softmax over the top-k
        np.testing.assert_allclose(w[t], ref_w, rtol=1e-13)


def test_k_equals_E_gives_full_softmax():
    from scipy.special import softmax
    rng = np.random.default_rng(1)
    logits = rng.normal(size=(50, 12))
    idx, w, margin = oracle.route(logits, 12)
    p = softmax(logits, axis=1)
    for t in range(50):
        np.testing.assert_allclose(w[t], p[t, idx[t]], rtol=1e-13)
        assert np.all(np.diff(logits[t, idx[t]]) <= 0)
    assert np.all(np.isinf(margin))


def test_gate_weights_properties():
    inp = make_small(T=300, d=64, E=64, k=8, F=64, S=1, seed=5)
    logits = oracle.router_logits(inp.x, inp.W_router)
    idx, w, margin = oracle.route(logits, 8)
    assert np.all(w >= 0)
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=1e-14)
    assert np.all(np.diff(w, axis=1) <= 0)          # non-increasing, like the logits
    assert np.all(margin >= 0)
    for t in range(300):
        assert len(set(idx[t])) == 8


def test_pages_example_64_experts_top4():
    """The explainer's example (section 2.2): 64 experts, K=4 -> 4 active, 60 idle per token."""
    inp = make_small(T=128, d=64, E=64, k=4, F=64, S=0, seed=7)
    logits = oracle.router_logits(inp.x, inp.W_router)
    idx, _, _ = oracle.route(logits, 4)
    for t in range(128):
        active = set(idx[t].tolist())
        assert len(active) == 4 and 64 - len(active) == 60
    counts, offsets, perm, pos = oracle.dispatch(idx, 64)
    assert counts.sum() == 128 * 4


@pytest.mark.parametrize("T,E,k", [(0, 4, 2), (1, 1, 1), (7, 3, 2), (300, 64, 8), (64, 16, 2)])
def test_dispatch_against_stable_argsort(T, E, k):
    rng = np.random.default_rng(T + E)
    idx = np.array([rng.permutation(E)[:k] for _ in range(T)], np.int32).reshape(T, k)
    counts, offsets, perm, pos = oracle.dispatch(idx, E)
    flat = idx.reshape(-1)
    np.testing.assert_array_equal(counts, np.bincount(flat, minlength=E))
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    np.testing.assert_array_equal(perm, np.argsort(flat, kind="stable"))
    assert counts.sum() == T * k and offsets[-1] == T * k and np.all(counts <= T)
    np.testing.assert_array_equal(perm[pos], np.arange(T * k))   # pos o perm = id
    np.testing.assert_array_equal(np.sort(perm), np.arange(T * k))  # bijection
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) > 0) and np.all(flat[seg] == e)


def _dense_swiglu_f64(x, Wg, Wu, Wd):
    """One dense SwiGLU FFN with torch float64 matmuls (the library routine)."""
    x = x.double()
    g = x @ Wg.double().T
    u = x @ Wu.double().T
    return (torch.nn.functional.silu(g) * u) @ Wd.double().T


def test_single_expert_reduces_to_dense_ffn():
    """E=1, k=1, S=0: the layer is one dense SwiGLU FFN (the dense first layer's form)."""
    inp = make_small(T=19, d=128, E=1, k=1, F=64, S=0, seed=11)
    out = oracle.forward(inp)
    assert np.all(out["idx"] == 0) and np.all(out["w"] == 1.0)
    ref = _dense_swiglu_f64(inp.x, inp.W_gate[0], inp.W_up[0], inp.W_down[0]).numpy()
    np.testing.assert_allclose(out["y"], ref, rtol=1e-12, atol=1e-12)


def test_single_expert_plus_shared_equals_concatenated_ffn():
    """E=1, k=1, S=1: routed + shared equals one dense FFN of width 2F (weights concatenated)."""
    inp = make_small(T=13, d=64, E=1, k=1, F=64, S=1, seed=12)
    out = oracle.forward(inp)
    Wg = torch.cat([inp.W_gate[0], inp.Ws_gate[0]], 0)
    Wu = torch.cat([inp.W_up[0], inp.Ws_up[0]], 0)
    Wd = torch.cat([inp.W_down[0], inp.Ws_down[0]], 1)
    ref = _dense_swiglu_f64(inp.x, Wg, Wu, Wd).numpy()
    np.testing.assert_allclose(out["y"], ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("seed,S", [(21, 1), (22, 0), (23, 2)])
def test_brute_force_all_experts_masked(seed, S):
    """Running every expert on every token and masking to the top-k gates gives the same y."""
    inp = make_small(T=24, d=64, E=6, k=3, F=64, S=S, seed=seed, bias_scale=0.3)
    out = oracle.forward(inp)
    x = inp.x.double()
    logits = x @ inp.W_router.double().T + inp.bias.double()
    p = torch.softmax(logits, dim=1)
    mask = torch.zeros_like(p)
    top = torch.tensor(out["idx"], dtype=torch.long)
    mask.scatter_(1, top, 1.0)
    gates = p * mask
    gates = gates / gates.sum(1, keepdim=True)
    ref = torch.zeros(inp.wl.T, inp.wl.d, dtype=torch.float64)
    for e in range(inp.wl.E):
        ref += gates[:, e:e + 1] * _dense_swiglu_f64(inp.x, inp.W_gate[e], inp.W_up[e],
                                                     inp.W_down[e])
    for s in range(S):
        ref += _dense_swiglu_f64(inp.x, inp.Ws_gate[s], inp.Ws_up[s], inp.Ws_down[s])
    # the top-k of the brute force is the full sort of the fp64 library logits
    for t in range(inp.wl.T):
        order = sorted(range(inp.wl.E), key=lambda e: (-logits[t, e].item(), e))
        assert list(out["idx"][t]) == order[:3]
    np.testing.assert_allclose(out["y"], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_token_independence_and_duplicates():
    inp = make_small(T=40, d=64, E=8, k=2, F=64, S=1, seed=31)
    full = oracle.forward(inp)
    sub = [39, 3, 17, 3]
    part = oracle.forward(inp, tokens=sub)
    np.testing.assert_array_equal(part["y"], full["y"][sub])
    np.testing.assert_array_equal(part["y"][1], part["y"][3])


def test_linearity_in_down_projection():
    inp = make_small(T=16, d=64, E=8, k=2, F=64, S=1, seed=41)
    y1 = oracle.forward(inp)["y"]
    inp2 = Inputs(inp.wl, inp.x, inp.W_router, inp.bias, inp.W_gate, inp.W_up, inp.W_down * 2,
                  inp.Ws_gate, inp.Ws_up, inp.Ws_down * 2)
    y2 = oracle.forward(inp2)["y"]
    np.testing.assert_array_equal(y2, 2 * y1)   # powers of two are exact in bf16 and fp64


def test_expert_relabelling_permutes_idx_and_keeps_y():
    inp = make_small(T=32, d=64, E=8, k=3, F=64, S=1, seed=51)
    out = oracle.forward(inp)
    pi = torch.randperm(8, generator=torch.Generator().manual_seed(0))  # new label j -> old pi[j]
    inp2 = Inputs(inp.wl, inp.x, inp.W_router[pi], None, inp.W_gate[pi], inp.W_up[pi],
                  inp.W_down[pi], inp.Ws_gate, inp.Ws_up, inp.Ws_down)
    out2 = oracle.forward(inp2)
    inv = torch.argsort(pi).numpy()   # old label -> new label
    np.testing.assert_array_equal(out2["idx"], inv[out["idx"]])
    np.testing.assert_allclose(out2["y"], out["y"], rtol=1e-13, atol=1e-13)


def test_override_idx_and_sparse_weight_mapping():
    inp = make_small(T=10, d=64, E=8, k=2, F=64, S=1, seed=61)
    out = oracle.forward(inp)
    # the same routing passed as an override gives the same result
    out2 = oracle.forward(inp, idx_override=out["idx"])
    np.testing.assert_allclose(out2["w"], out["w"], rtol=1e-14)
    np.testing.assert_allclose(out2["y"], out["y"], rtol=1e-13, atol=1e-14)
    # supplying only the experts the chosen tokens use
    toks = [2, 5]
    used = sorted(set(out["idx"][toks].reshape(-1).tolist()))
    sparse = {"W_gate": {e: inp.W_gate[e] for e in used}, "W_up": {e: inp.W_up[e] for e in used},
              "W_down": {e: inp.W_down[e] for e in used}}
    out3 = oracle.forward(inp, tokens=toks, weights=sparse)
    np.testing.assert_array_equal(out3["y"], out["y"][toks])
    missing = {"W_gate": {used[0]: inp.W_gate[used[0]]}, "W_up": {}, "W_down": {}}
    with pytest.raises(ValueError):
        oracle.forward(inp, tokens=toks, weights=missing)


def test_bad_arguments_rejected():
    with pytest.raises(ValueError):
        oracle.route(np.zeros((2, 3)), 4)          # k > E
    with pytest.raises(ValueError):
        oracle.dispatch(np.array([[0, 5]], np.int32), 4)   # expert id out of range


# ----------------------------------------------------------------------------
# FP8 expert weights: decode and block scales.
# ----------------------------------------------------------------------------
def test_e4m3_decode_matches_torch_float8_for_every_code():
    """All 256 codes against torch's float8_e4m3fn -> float64 conversion (a library
    implementation of the same OCP format, independent of the oracle's decoder)."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.E4M3_TABLE
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got)) and nan.sum() == 2   # 0x7F and 0xFF
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    # signed zeros are kept
    assert math.copysign(1.0, got[0x80]) == -1.0 and got[0x00] == 0.0


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6),
    (0x38, 1.0), (0x39, 1.125), (0x3F, 1.875), (0x40, 2.0), (0x7E, 448.0),
    (0xB8, -1.0), (0xFE, -448.0), (0x77, 240.0), (0x30, 0.5)])
def test_e4m3_values_from_the_format_definition(code, value):
    """Hand-derived values: (-1)^s * (1 + m/8) * 2^(e-7), subnormals m/8 * 2^-6."""
    assert oracle.e4m3_value(code) == value


def test_dequant_block_scales_and_layout():
    """Two experts, 3 rows, K = 64 (two 32-element blocks): scale byte of (expert e, block
    b, row r) = 120 + 4e + 2b + r, every code 0x38 (1.0) except row 1 of expert 0, whose
    codes are 0x40 (2.0); so w[e, r, j] = c * 2^(-7 + 4e + 2(j // 32) + r)."""
    n, rows, K = 2, 3, 64
    codes = np.full((n, rows, K), 0x38, np.uint8)
    codes[0, 1, :] = 0x40
    scales = np.zeros((n, K // 32, rows), np.uint8)
    for e in range(n):
        for b in range(K // 32):
            for r in range(rows):
                scales[e, b, r] = 120 + 4 * e + 2 * b + r
    w = oracle.dequant_fp8(codes, scales)
    for e in range(n):
        for r in range(rows):
            for j in (0, 31, 32, 63):
                c = 2.0 if (e, r) == (0, 1) else 1.0
                assert w[e, r, j] == c * 2.0 ** (-7 + 4 * e + 2 * (j // 32) + r), (e, r, j)


def test_fp8_checkpoint_round_trip_and_exact_bf16():
    """The workload's FP8 checkpoint decodes to within half an e4m3 step of the bf16 draws
    (relative 2^-4 of each value for normal codes, 2^-10 of the block maximum below the
    normal range), and the decoded weights are exact bf16 values."""
    from workloads import make_fp8
    inp = make_small(4, 128, 3, 2, 64, 1, seed=11)
    routed, shared = make_fp8(inp)
    for W, c, s in ((inp.W_gate, routed.gate, routed.gate_scale),
                    (inp.W_down, routed.down, routed.down_scale),
                    (inp.Ws_up, shared.up, shared.up_scale)):
        w = W.to(torch.float64).numpy()
        got = oracle.dequant_fp8(c, s)
        blocks = np.abs(w).reshape(w.shape[0], w.shape[1], -1, 32).max(-1)
        floor = np.repeat(blocks, 32, axis=2) * 2.0 ** -10
        assert np.all(np.abs(got - w) <= np.maximum(np.abs(w) * 2.0 ** -4, floor))
        bits = oracle.fp8_as_bf16(c, s)
        back = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64)
        np.testing.assert_array_equal(back.numpy(), got)


def test_fp8_layer_is_the_bf16_layer_on_decoded_weights():
    """The oracle's FP8 layer equals its bf16 layer run on weights that are already exactly
    the decoded values (both from the same seeded draws, via independent routes: the
    decoded bits versus torch's float8 -> bf16 cast of the same codes times the scales)."""
    from workloads import make_fp8
    inp = make_small(12, 128, 4, 2, 64, 1, seed=12)
    routed, shared = make_fp8(inp)
    via_oracle = oracle.forward(oracle.fp8_inputs(inp, routed, shared))["y"]

    def torch_dec(c, s):
        v = c.view(torch.float8_e4m3fn).to(torch.float32)
        m = torch.exp2(s.to(torch.float32) - 127.0).transpose(1, 2)
        return (v * m.repeat_interleave(32, dim=2)).to(torch.bfloat16)
    alt = Inputs(inp.wl, inp.x, inp.W_router, inp.bias,
                 torch_dec(routed.gate, routed.gate_scale), torch_dec(routed.up, routed.up_scale),
                 torch_dec(routed.down, routed.down_scale), torch_dec(shared.gate, shared.gate_scale),
                 torch_dec(shared.up, shared.up_scale), torch_dec(shared.down, shared.down_scale))
    np.testing.assert_array_equal(via_oracle, oracle.forward(alt)["y"])


def _slice(inp, f0, f1):
    """Rows f0:f1 of every W_gate / W_up and the matching columns of every W_down."""
    def rows(W):
        return W[:, f0:f1, :].contiguous()

    def cols(W):
        return W[:, :, f0:f1].contiguous()
    return (rows(inp.W_gate), rows(inp.W_up), cols(inp.W_down),
            rows(inp.Ws_gate), rows(inp.Ws_up), cols(inp.Ws_down))


def test_shard_of_one_expert_slice_is_the_dense_ffn_slice():
    """E=1, k=1, S=0: one d_ff slice's part is the dense SwiGLU FFN restricted to that slice
    (torch float64), and the parts of all slices add up to the dense FFN."""
    inp = make_small(T=11, d=128, E=1, k=1, F=256, S=0, seed=61)
    idx = np.zeros((11, 1), np.int32)
    w = np.ones((11, 1))
    total = np.zeros((11, 128))
    for f0 in range(0, 256, 64):
        Wg, Wu, Wd, _, _, _ = _slice(inp, f0, f0 + 64)
        part = oracle.shard_output(inp.x, idx, w, Wg, Wu, Wd)
        ref = _dense_swiglu_f64(inp.x, Wg[0], Wu[0], Wd[0]).numpy()
        np.testing.assert_allclose(part, ref, rtol=1e-12, atol=1e-12)
        total += part
    ref = _dense_swiglu_f64(inp.x, inp.W_gate[0], inp.W_up[0], inp.W_down[0]).numpy()
    np.testing.assert_allclose(total, ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("n_slices", [2, 4])
def test_d_ff_slices_add_up_to_the_layer(n_slices):
    """Tensor parallelism over d_ff: every shard holds a slice of every routed and shared
    expert; the parts add up to the whole layer."""
    inp = make_small(T=20, d=64, E=6, k=2, F=256, S=1, seed=62, bias_scale=0.2)
    full = oracle.forward(inp)
    width = 256 // n_slices
    total = np.zeros_like(full["y"])
    for r in range(n_slices):
        Wg, Wu, Wd, Sg, Su, Sd = _slice(inp, r * width, (r + 1) * width)
        total += oracle.shard_output(inp.x, full["idx"], full["w"], Wg, Wu, Wd, Sg, Su, Sd)
    np.testing.assert_allclose(total, full["y"], rtol=1e-11, atol=1e-12)


def test_expert_ranges_add_up_to_the_layer():
    """Expert parallelism: shards hold 3, 2 and 3 of 8 routed experts, the first one also the
    shared expert; the parts add up to the layer, and a part leaves out the other shards'
    experts (without the shared expert, a shard whose experts no token picked gives 0)."""
    inp = make_small(T=30, d=64, E=8, k=3, F=64, S=1, seed=63, bias_scale=0.3)
    full = oracle.forward(inp)
    total = np.zeros_like(full["y"])
    for r, (e0, n) in enumerate([(0, 3), (3, 2), (5, 3)]):
        sl = slice(e0, e0 + n)
        shared = (inp.Ws_gate, inp.Ws_up, inp.Ws_down) if r == 0 else (None, None, None)
        total += oracle.shard_output(inp.x, full["idx"], full["w"], inp.W_gate[sl],
                                     inp.W_up[sl], inp.W_down[sl], *shared, expert_begin=e0)
    np.testing.assert_allclose(total, full["y"], rtol=1e-11, atol=1e-12)
    idx = np.full_like(full["idx"], 7)
    idx[:, 1:] = 6
    none = oracle.shard_output(inp.x, idx, full["w"], inp.W_gate[:3], inp.W_up[:3],
                               inp.W_down[:3], expert_begin=0)
    assert np.all(none == 0.0)


def test_ihc_update_hand_worked():
    """Two streams, two features, one token, by hand:
    H = [[1, 2], [4, 8]] (stream 0, stream 1), B = [[0, 0.5], [0.25, 0]], gamma = [1, -2],
    y = [10, 20]:
      H'_0 = H_0 + 0 * H_0 + 0.5 * H_1 + 1 * y = [1 + 2 + 10, 2 + 4 + 20] = [13, 26]
      H'_1 = H_1 + 0.25 * H_0 + 0 * H_1 - 2 * y = [4 + 0.25 - 20, 8 + 0.5 - 40] = [-15.75, -31.5]
    and the layer input with alpha = [0.5, 0.25] is x = [0.5 + 1, 1 + 2] = [1.5, 3]."""
    H = np.array([[[1.0, 2.0], [4.0, 8.0]]])
    out = oracle.ihc_update(H, [[0.0, 0.5], [0.25, 0.0]], [1.0, -2.0], [[10.0, 20.0]])
    np.testing.assert_array_equal(out[0], [[13.0, 26.0], [-15.75, -31.5]])
    np.testing.assert_array_equal(oracle.ihc_mix_in(H, [0.5, 0.25]), [[1.5, 3.0]])


def test_ihc_with_one_stream_is_the_residual_connection():
    """n = 1, alpha = 1, B = 0, gamma = 1: H' = H + layer(H), the ordinary residual block."""
    inp = make_small(T=12, d=64, E=4, k=2, F=64, S=1, seed=71)
    H = inp.x.view(12, 1, 64)
    x = oracle.ihc_mix_in(H, [1.0])
    xf = torch.tensor(x).float().to(torch.bfloat16)
    assert torch.equal(xf.view(torch.int16), inp.x.view(torch.int16))   # exact: weight 1
    y = oracle.forward(inp)["y"]
    out = oracle.ihc_update(H, [[0.0]], [1.0], y)
    np.testing.assert_allclose(out[:, 0, :], inp.x.double().numpy() + y, rtol=0, atol=0)


def test_ihc_identity_path_and_stream_relabelling():
    """B = 0 keeps every stream: H'_i - H_i = gamma_i y exactly.  Relabelling the streams
    (alpha, the rows and columns of B, gamma, the stream axis of H) relabels the result,
    with an asymmetric B so a transposed exchange would fail."""
    g = torch.Generator().manual_seed(3)
    H = torch.randn(5, 4, 32, generator=g).to(torch.bfloat16)
    y = torch.randn(5, 32, generator=g).double().numpy()
    gamma = np.array([0.5, -1.0, 2.0, 0.25])
    out = oracle.ihc_update(H, np.zeros((4, 4)), gamma, y)
    Hf = H.double().numpy()
    for i in range(4):
        np.testing.assert_array_equal(out[:, i] - Hf[:, i], gamma[i] * y)
    B = np.arange(16, dtype=np.float64).reshape(4, 4) / 32.0
    alpha = np.array([0.1, 0.2, 0.3, 0.4])
    base = oracle.ihc_update(H, B, gamma, y)
    pi = np.array([2, 0, 3, 1])             # new stream i is old stream pi[i]
    perm = oracle.ihc_update(H[:, pi], B[np.ix_(pi, pi)], gamma[pi], y)
    np.testing.assert_allclose(perm, base[:, pi], rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(oracle.ihc_mix_in(H[:, pi], alpha[pi]),
                               oracle.ihc_mix_in(H, alpha), rtol=1e-15, atol=1e-15)
    # B against its transpose: stream 0 takes 1/32 of stream 1 in B, 4/32 in B^T
    bt = oracle.ihc_update(H, B.T, gamma, y)
    assert not np.allclose(bt, base)
