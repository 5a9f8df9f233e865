"""moe_dispatch_noalloc: the dispatch for callers that cannot allocate device memory.

Such callers (a plug-in whose host application owns every device allocation,
or a loop that must not call cudaMalloc) cannot provide the workspace that
moe_dispatch uses for its scratch; this entry point uses a fixed array inside
the library instead.  The test calls it through the C ABI and checks that two
calls in a row -- the second one with different routing, so stale scratch
contents from the first would show -- give exactly what moe_dispatch gives.
Dispatch results are integers, so the comparison is bit-exact, as everywhere
else in these tests.  The file is collected last so that a run which stops at
the first failure has run every other test already.
"""
import pytest
import torch

import mixture_experts_layer_47_b200 as moe

pytestmark = pytest.mark.gpu


def _routing(T, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)


def _outputs(E, n):
    return [torch.full((m,), -1, dtype=torch.int32, device="cuda") for m in (E, E + 1, n, n)]


@pytest.mark.parametrize("T,E,k", [(16, 256, 8), (8192, 256, 8), (777, 64, 4)])
def test_noalloc_dispatch_matches_workspace_dispatch(T, E, k):
    h = moe.moe_create(64, E, k, 64, 1)
    ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
    for call, seed in enumerate((11, 12)):          # two calls in a row, different routing
        idx = _routing(T, E, k, seed + T).cuda()
        ref = _outputs(E, T * k)
        got = _outputs(E, T * k)
        moe.moe_dispatch(h, idx, *ref, ws)
        moe.moe_dispatch_noalloc(h, idx, *got)
        torch.cuda.synchronize()
        for name, a, b in zip(("counts", "offsets", "perm", "pos"), got, ref):
            assert torch.equal(a, b), (call, name)
        assert int(got[1][-1]) == T * k


def test_noalloc_dispatch_rejects_sizes_beyond_its_scratch():
    h = moe.moe_create(64, 256, 8, 64, 1)
    T = 65536 // 8 + 1                               # one token more than the fixed scratch holds
    idx = torch.zeros(T, 8, dtype=torch.int32, device="cuda")
    out = _outputs(256, T * 8)
    with pytest.raises(moe.MoEError) as e:
        moe.moe_dispatch_noalloc(h, idx, *out)
    assert e.value.status == moe.MOE_ERR_WORKSPACE
    assert torch.all(out[0] == -1)                   # nothing was enqueued
