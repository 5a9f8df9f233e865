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
from gpu_helpers import bad_index_routing, check_skipped_slots

pytestmark = pytest.mark.gpu


def _routing(T, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)


def _outputs(E, n):
    return [torch.full((m,), -1, dtype=torch.int32, device="cuda") for m in (E, E + 1, n, n)]


# E = 512 and E = 1024 take the three-kernel dispatch at few slots, and 1024 is the number
# of experts the fixed scratch is sized for.
@pytest.mark.parametrize("T,E,k", [(16, 256, 8), (8192, 256, 8), (777, 64, 4), (64, 1024, 8),
                                   (512, 512, 8), (2000, 1024, 32)])
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


def test_noalloc_dispatch_skips_out_of_range_index():
    """Out-of-range expert indices: the same skipped slots (pos = -1) and segments as
    moe_dispatch, although the status word is not readable through this entry point."""
    T, E, k = 900, 64, 8
    idx = bad_index_routing(T, E, k, seed=3).cuda()
    h = moe.moe_create(64, E, k, 64, 1)
    got = _outputs(E, T * k)
    moe.moe_dispatch_noalloc(h, idx, *got)
    torch.cuda.synchronize()
    check_skipped_slots(idx.cpu().numpy(), E, *[o.cpu().numpy() for o in got])
