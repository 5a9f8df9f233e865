"""Full Hy4-sized workloads on the GPU, in the launch configuration bench.py times
(one moe_forward over the whole batch with the shared workspace).

Routing of every token is compared with the oracle (bit-exact indices except
near-tie tokens), dispatch bit-exactly given the GPU's routing (and end to end
when no token is exempt), and the layer output element by element on a sample
of tokens the fp64 oracle computes one by one, with only the experts those
tokens use copied to the host.  At decode the sample is every token; at the
larger batches it holds, for every routed expert, the last token routed to it
(the group's last, ragged token tile), the first token of the most loaded
expert, and 256 evenly spaced tokens.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (Y_REL_TOL, coverage_tokens, dispatch_parity, gpu_forward, rel_err,
                         route_parity)
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["decode", "batched_decode", "prefill", "skewed_prefill"])
def test_full_size_workload(name):
    wl = WORKLOADS[name]
    inp = make_inputs(wl, device="cuda")
    y, v = gpu_forward(inp)
    x_cpu = inp.x.cpu()
    bias = None if inp.bias is None else inp.bias.cpu()
    logits = oracle.router_logits(x_cpu, inp.W_router.cpu(), bias)
    idx_g = v["topk_idx"].numpy()
    exempt, idx_o, w_o = route_parity(logits, idx_g, v["topk_w"].numpy(), wl.k)
    c_o, o_o, _, _ = dispatch_parity(idx_g, wl.E, v["counts"], v["offsets"], v["perm"], v["pos"])
    assert c_o.sum() == wl.T * wl.k and c_o.max() <= wl.T
    if not exempt.any():
        np.testing.assert_array_equal(o_o, oracle.dispatch(idx_o, wl.E)[1])
    yg = y.float().numpy()
    assert np.isfinite(yg).all()

    idx_use = np.where(exempt[:, None], idx_g, idx_o)
    tokens = coverage_tokens(idx_g, wl.T, 256)
    assert len(set(idx_g[tokens].reshape(-1).tolist())) == int((c_o > 0).sum())
    w_use = oracle.renormalised_gates(logits, idx_use)
    used = sorted(set(idx_use[tokens].reshape(-1).tolist()))
    weights = {
        "W_gate": {e: inp.W_gate[e].cpu() for e in used},
        "W_up": {e: inp.W_up[e].cpu() for e in used},
        "W_down": {e: inp.W_down[e].cpu() for e in used},
    }
    y_ref = oracle.moe_ffn_tokens(x_cpu, idx_use, w_use, weights["W_gate"], weights["W_up"],
                                  weights["W_down"], inp.Ws_gate.cpu(), inp.Ws_up.cpu(),
                                  inp.Ws_down.cpu(), tokens, E=wl.E, F=wl.F, S=wl.S)
    err = rel_err(yg[tokens], y_ref)
    per_token = np.abs(yg[tokens] - y_ref).max(1) / np.abs(y_ref).max()
    print(f"{name}: exempt tokens {int(exempt.sum())}, sampled tokens {len(tokens)}, "
          f"experts used {len(used)}, max count {int(c_o.max())}, min count {int(c_o.min())}, "
          f"rel err {err:.3e} (worst token {int(tokens[per_token.argmax()])})")
    assert err < Y_REL_TOL, err
