"""Shared helpers of the GPU parity tests: run the CUDA path through the C-ABI
binding, run the fp64 oracle on the same inputs, and compare as the layer's
contract states (indices bit-exact except near-tie tokens, dispatch bit-exact
given the same routing, outputs within max|gpu-ref|/max|ref| <= 1e-2)."""
from __future__ import annotations

import numpy as np
import torch

import mixture_experts_layer_47_b200 as moe
import oracle

MARGIN_EXEMPT = 1e-5      # 8th/9th logit margin below which a token's routing is exempt
Y_REL_TOL = 1e-2          # max|gpu - ref| / max|ref| for the layer output
W_ABS_TOL = 2e-6          # gate weights: fp32 softmax of fp32 logits vs fp64


def rel_err(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    denom = np.abs(ref).max()
    return float(np.abs(got - ref).max() / (denom if denom > 0 else 1.0))


def gpu_forward(inp, stream=None):
    """moe_forward on inp (device tensors); returns y and the workspace intermediates (CPU)."""
    wl = inp.wl
    h = moe.moe_create(wl.d, wl.E, wl.k, wl.F, wl.S)
    ws = torch.empty(moe.moe_workspace_size(h, wl.T), dtype=torch.uint8, device="cuda")
    y = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(h, inp.x, inp.W_router, inp.bias, inp.W_gate, inp.W_up, inp.W_down,
                    inp.Ws_gate, inp.Ws_up, inp.Ws_down, y, ws, stream)
    status, detail = moe.moe_device_status(h, wl.T, ws, stream)
    assert status == moe.MOE_OK, (status, hex(detail))
    views = {k: v.cpu() for k, v in moe.workspace_views(h, wl.T, ws).items()}
    return y.cpu(), views


def route_parity(logits_ref, idx_gpu, w_gpu, k):
    """Compare GPU routing with the oracle's.  Returns (exempt mask, oracle idx, oracle w)."""
    idx_o, w_o, margin = oracle.route(logits_ref, k)
    idx_g = np.asarray(idx_gpu)
    exempt = margin < MARGIN_EXEMPT
    T = idx_o.shape[0]
    for t in range(T):
        if exempt[t] or np.array_equal(idx_g[t], idx_o[t]):
            continue
        # an order swap inside the top-k is exempt where the swapped logits are within 1e-5
        assert sorted(idx_g[t]) == sorted(idx_o[t]), (t, idx_g[t], idx_o[t], margin[t])
        lg = logits_ref[t, idx_g[t]]
        lo = logits_ref[t, idx_o[t]]
        assert np.all(np.abs(lg - lo) < MARGIN_EXEMPT), (t, lg, lo)
    ok = ~exempt
    same = np.all(idx_g == idx_o, axis=1) & ok
    if same.any():
        np.testing.assert_allclose(np.asarray(w_gpu)[same], w_o[same], rtol=0, atol=W_ABS_TOL)
    return exempt, idx_o, w_o


def dispatch_parity(idx_gpu, E, counts, offsets, perm, pos):
    c_o, o_o, p_o, q_o = oracle.dispatch(np.asarray(idx_gpu, np.int32), E)
    np.testing.assert_array_equal(np.asarray(counts), c_o)
    np.testing.assert_array_equal(np.asarray(offsets), o_o)
    np.testing.assert_array_equal(np.asarray(perm), p_o)
    np.testing.assert_array_equal(np.asarray(pos), q_o)
    return c_o, o_o, p_o, q_o


def oracle_rows(inp, idx, perm, tokens_rows=None):
    """Oracle per-row expert outputs (h and y) in dispatch order, for the rows listed
    (default all): rows < T*k are routed slots perm[p]; the rest are shared rows."""
    wl = inp.wl
    T, k, S = wl.T, wl.k, wl.S
    nrows = T * k + S * T
    rows = range(nrows) if tokens_rows is None else tokens_rows
    x = inp.x.cpu()
    H, Y = {}, {}
    for r in rows:
        if r < T * k:
            s = int(perm[r])
            t, i = divmod(s, k)
            e = int(idx[t][i])
            Wg, Wu, Wd = inp.W_gate[e], inp.W_up[e], inp.W_down[e]
        else:
            s_idx, t = divmod(r - T * k, T)
            Wg, Wu, Wd = inp.Ws_gate[s_idx], inp.Ws_up[s_idx], inp.Ws_down[s_idx]
        h, y = oracle.expert_one(x[t], Wg.cpu(), Wu.cpu(), Wd.cpu())
        H[r], Y[r] = h, y
    return H, Y


def bad_index_routing(T, E, k, seed):
    """Random distinct experts per token with a few slots set out of range (E, E + 5, -1)."""
    g = torch.Generator().manual_seed(seed)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    flat = idx.view(-1)
    bad = torch.randperm(T * k, generator=g)[:max(2, T * k // 50)]
    for j, s in enumerate(bad.tolist()):
        flat[s] = (E, E + 5, -1)[j % 3]
    return idx


def check_skipped_slots(idx, E, counts, offsets, perm, pos):
    """Dispatch of routing with out-of-range slots: those slots are skipped (pos = -1), the
    valid ones are grouped exactly as a stable sort of the valid slots by expert."""
    flat = np.asarray(idx).reshape(-1)
    valid = (flat >= 0) & (flat < E)
    slots = np.nonzero(valid)[0]
    order = slots[np.argsort(flat[slots], kind="stable")]
    n = len(order)
    c = np.bincount(flat[valid], minlength=E)
    np.testing.assert_array_equal(np.asarray(counts), c)
    np.testing.assert_array_equal(np.asarray(offsets), np.concatenate([[0], np.cumsum(c)]))
    assert int(offsets[-1]) == n < flat.size
    np.testing.assert_array_equal(np.asarray(perm)[:n], order)
    exp_pos = np.full(flat.size, -1, np.int64)
    exp_pos[order] = np.arange(n)
    np.testing.assert_array_equal(np.asarray(pos), exp_pos)


def coverage_tokens(idx, T, n_even):
    """Tokens for a sampled full-size output check that reach every part of the grouped GEMMs:
    for every routed expert the last token routed to it (so each group's last, ragged token
    tile is checked), the first token of the most loaded expert, and n_even evenly spaced
    tokens.  The shared expert runs on all of them."""
    idx = np.asarray(idx)
    chosen = set(np.linspace(0, T - 1, min(n_even, T)).round().astype(np.int64).tolist())
    flat = idx.reshape(-1)
    k = idx.shape[1]
    last = {}
    for s in range(flat.size - 1, -1, -1):       # last slot per expert, scanning backwards
        e = int(flat[s])
        if e not in last:
            last[e] = s // k
    chosen.update(last.values())
    hottest = np.bincount(flat).argmax()
    chosen.add(int(np.nonzero((idx == hottest).any(axis=1))[0][0]))
    return np.array(sorted(chosen), dtype=np.int32)
