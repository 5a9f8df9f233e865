"""Host-side checks of the C-ABI library: it builds for sm_100a, loads, exports
every entry point include/moe.h declares, and rejects bad arguments on the host
before anything reaches a device.  No kernel runs here."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import mixture_experts_layer_47_b200 as moe
from mixture_experts_layer_47_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.load_library()


def declared_symbols():
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:moe_status|size_t|int|const char \*)\s*(moe_\w+)\s*\(",
                                 text, re.M)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 12, names
    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (moe_\w+)", out))
    for n in names:
        assert n in exported, n
        assert hasattr(lib, n)
    assert set(names) == set(moe.EXPORTS)


def test_library_is_sm100a_only(lib):
    out = subprocess.run(["cuobjdump", "--list-elf", moe.LIB_PATH], capture_output=True,
                         text=True)
    if out.returncode != 0:
        pytest.skip("cuobjdump unavailable")
    archs = set(re.findall(r"sm_(\d+a?)", out.stdout))
    assert archs == {"100a"}, archs


def test_status_strings(lib):
    for code in range(0, 8):
        assert moe.status_string(code)
    assert moe.status_string(99) == "unknown status"


def _create(d, E, k, F, S):
    h = ctypes.c_void_p()
    rc = moe.load_library().moe_create(d, E, k, F, S, ctypes.byref(h))
    return rc, h


@pytest.mark.parametrize("args,code", [
    ((6144, 256, 8, 2048, 1), moe.MOE_OK),
    ((256, 16, 2, 128, 1), moe.MOE_OK),
    ((64, 1, 1, 64, 0), moe.MOE_OK),
    ((256, 16, 17, 128, 1), moe.MOE_ERR_INVALID_ARG),   # k > E
    ((256, 16, 0, 128, 1), moe.MOE_ERR_INVALID_ARG),    # k < 1
    ((0, 16, 2, 128, 1), moe.MOE_ERR_INVALID_ARG),
    ((256, 16, 2, 128, -1), moe.MOE_ERR_INVALID_ARG),
    ((250, 16, 2, 128, 1), moe.MOE_ERR_UNSUPPORTED),    # d not a multiple of 64
    ((256, 16, 2, 100, 1), moe.MOE_ERR_UNSUPPORTED),    # d_ff not a multiple of 64
    ((256, 2048, 2, 128, 1), moe.MOE_ERR_UNSUPPORTED),  # E > 1024
    ((256, 64, 33, 128, 1), moe.MOE_ERR_UNSUPPORTED),   # k > 32
    ((256, 16, 2, 128, 9), moe.MOE_ERR_UNSUPPORTED),    # S > 8
])
def test_create_validates_shape(lib, args, code):
    rc, h = _create(*args)
    assert rc == code
    assert (h.value is not None) == (code == moe.MOE_OK)
    if h.value:
        assert lib.moe_destroy(h) == moe.MOE_OK
    assert lib.moe_create(1, 1, 1, 1, 1, None) == moe.MOE_ERR_INVALID_ARG


def test_workspace_size_and_layout(lib):
    h = moe.moe_create(6144, 256, 8, 2048, 1)
    assert moe.moe_workspace_size(h, -1) == 0
    sizes = [moe.moe_workspace_size(h, T) for T in (1, 16, 256, 8192)]
    assert all(s > 0 for s in sizes) and sizes == sorted(sizes)
    # Hy4 prefill: X_perm 805 MB + H 302 MB + Y (bf16) 906 MB + two x staging slots and
    # the y staging (3 x 101 MB) + small
    assert 2.3e9 < sizes[-1] < 2.4e9
    for addr in (0, 1, 1000, 4096 + 16):
        L = moe.moe_get_workspace_layout(h, 16, addr)
        assert L["total"] <= moe.moe_workspace_size(h, 16)
        for key in ("status", "topk_idx", "topk_w", "counts", "offsets", "perm", "pos", "h_act",
                    "y_rows"):
            assert (addr + L[key]) % 1024 == 0, key
    assert lib.moe_workspace_size(None, 16) == 0


def test_host_side_argument_errors_need_no_device(lib):
    """Bad arguments are rejected before any CUDA call, so these never touch a device."""
    h = moe.moe_create(256, 16, 2, 128, 1)
    hv = h.value
    T = 64
    ws_size = moe.moe_workspace_size(h, T)
    A = 1 << 20  # a 16-byte aligned fake address; never dereferenced on these paths
    L = moe.load_library()
    # null handle / pointers
    assert L.moe_route(None, A, A, None, T, A, A, A, ws_size, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_route(hv, None, A, None, T, A, A, A, ws_size, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_route(hv, A, A, None, -1, A, A, A, ws_size, None) == moe.MOE_ERR_INVALID_ARG
    # misaligned x
    assert L.moe_route(hv, A + 2, A, None, T, A, A, A, ws_size, None) == moe.MOE_ERR_ALIGNMENT
    # workspace too small / missing
    assert L.moe_route(hv, A, A, None, T, A, A, A, ws_size - 1, None) == moe.MOE_ERR_WORKSPACE
    assert L.moe_route(hv, A, A, None, T, A, A, None, ws_size, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_dispatch(hv, None, T, A, A, A, A, A, ws_size, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_dispatch(hv, A, T, A, A, A, A, A, 10, None) == moe.MOE_ERR_WORKSPACE
    # expert FFN: missing shared weights when S = 1, misaligned weights
    assert L.moe_expert_ffn(hv, A, A, A, T, A, A, A, None, A, A, A, A, ws_size, None) == \
        moe.MOE_ERR_INVALID_ARG
    assert L.moe_expert_ffn(hv, A, A, A, T, A + 8, A, A, A, A, A, A, A, ws_size, None) == \
        moe.MOE_ERR_ALIGNMENT
    assert L.moe_combine(hv, None, A, A, T, A, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_combine(hv, A, A, A, T, A + 4, None) == moe.MOE_ERR_ALIGNMENT
    assert L.moe_forward(hv, A, A, None, A, A, A, A, A, A, T, A, A, ws_size - 1, None) == \
        moe.MOE_ERR_WORKSPACE
    assert L.moe_forward(hv, A, None, None, A, A, A, A, A, A, T, A, A, ws_size, None) == \
        moe.MOE_ERR_INVALID_ARG
    # T == 0 is a no-op that touches nothing
    assert L.moe_forward(hv, None, None, None, None, None, None, None, None, None, 0, None, None,
                         0, None) == moe.MOE_OK
    assert L.moe_dispatch(hv, None, 0, None, None, None, None, None, 0, None) == moe.MOE_OK
    assert L.moe_selftest_wait_timeout(None, 4096, 1000, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_selftest_wait_timeout(A, 4096, 0, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_selftest_wait_timeout(A, 4096, 3_000_000_000, None) == moe.MOE_ERR_INVALID_ARG
    # more rows than the supported envelope
    assert L.moe_route(hv, A, A, None, 1 << 23, A, A, A, 1 << 40, None) == \
        moe.MOE_ERR_UNSUPPORTED


def test_fp8_entry_points_validate_on_the_host(lib):
    """The FP8 calls: a missing or incomplete weight set, a missing shared set when S = 1,
    a misaligned code or scale pointer, and T = 0, all decided before any CUDA call."""
    h = moe.moe_create(256, 16, 2, 128, 1)
    hv = h.value
    T = 64
    ws_size = moe.moe_workspace_size(h, T)
    A = 1 << 20
    L = moe.load_library()
    full = moe.Fp8ExpertWeights(A, A, A, A, A, A)
    holed = moe.Fp8ExpertWeights(A, A, A, None, A, A)
    skew = moe.Fp8ExpertWeights(A, A, A, A, A, A + 8)
    ref = ctypes.byref
    assert L.moe_forward_fp8(hv, A, A, None, None, ref(full), T, A, A, ws_size, None) == \
        moe.MOE_ERR_INVALID_ARG
    assert L.moe_forward_fp8(hv, A, A, None, ref(holed), ref(full), T, A, A, ws_size, None) == \
        moe.MOE_ERR_INVALID_ARG
    assert L.moe_forward_fp8(hv, A, A, None, ref(full), None, T, A, A, ws_size, None) == \
        moe.MOE_ERR_INVALID_ARG
    assert L.moe_forward_fp8(hv, A, A, None, ref(skew), ref(full), T, A, A, ws_size, None) == \
        moe.MOE_ERR_ALIGNMENT
    assert L.moe_forward_fp8(hv, A, A, None, ref(full), ref(full), T, A, A, ws_size - 1,
                             None) == moe.MOE_ERR_WORKSPACE
    assert L.moe_forward_fp8_host(hv, A, None, None, ref(full), ref(full), T, A, A, ws_size,
                                  None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_expert_ffn_fp8(hv, A, A, A, T, ref(full), ref(skew), A, A, ws_size, None) == \
        moe.MOE_ERR_ALIGNMENT
    assert L.moe_expert_ffn_fp8(hv, A, None, A, T, ref(full), ref(full), A, A, ws_size,
                                None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_forward_fp8(hv, None, None, None, ref(full), None, 0, None, None, 0, None) == \
        moe.MOE_OK
    # no shared experts: the shared set may be NULL
    h0 = moe.moe_create(256, 16, 2, 128, 0)
    assert L.moe_forward_fp8(h0.value, A, A, None, ref(full), None, T, A, A, 10, None) == \
        moe.MOE_ERR_WORKSPACE


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_valid_call_without_device_reports_cuda_error(lib):
    """With valid arguments but no GPU, a launch returns MOE_ERR_CUDA instead of crashing."""
    h = moe.moe_create(256, 16, 2, 128, 1)
    T = 64
    ws = moe.moe_workspace_size(h, T)
    A = 1 << 20
    L = moe.load_library()
    assert L.moe_route(h.value, A, A, None, T, A, A, A, ws, None) == moe.MOE_ERR_CUDA


def test_python_binding_validates_tensors(lib):
    h = moe.moe_create(256, 16, 2, 128, 1)
    ws = torch.empty(16, dtype=torch.uint8)
    x = torch.zeros(4, 256, dtype=torch.float32)
    with pytest.raises(TypeError):
        moe.moe_route(h, x, torch.zeros(16, 256), None, torch.zeros(4, 2, dtype=torch.int32),
                      torch.zeros(4, 2), ws)


def test_tuning_overrides_are_fixed_when_the_context_is_created(lib, monkeypatch):
    """MOE_ROUTER / MOE_GEMM_TILES are read once by moe_create: changing the environment
    afterwards changes neither the workspace size nor the plan of an existing context.
    The two router paths carve the workspace differently (the tensor-core path keeps a
    split copy of W_router, the FFMA path more split-K partials), so the size shows which
    path a context took."""
    T = 64
    monkeypatch.setenv("MOE_ROUTER", "ffma")
    monkeypatch.setenv("MOE_GEMM_TILES", "single")
    h_ffma = moe.moe_create(6144, 256, 8, 2048, 1)
    size_ffma = moe.moe_workspace_size(h_ffma, T)
    monkeypatch.setenv("MOE_ROUTER", "tc")
    monkeypatch.setenv("MOE_GEMM_TILES", "swap_pair")
    assert moe.moe_workspace_size(h_ffma, T) == size_ffma
    h_tc = moe.moe_create(6144, 256, 8, 2048, 1)
    size_tc = moe.moe_workspace_size(h_tc, T)
    assert size_tc != size_ffma
    monkeypatch.delenv("MOE_ROUTER")
    assert moe.moe_workspace_size(h_tc, T) == size_tc
    assert moe.moe_workspace_size(h_ffma, T) == size_ffma


def test_shard_and_dense_entry_points_validate_on_the_host(lib):
    """moe_forward_partial (expert range, partial shared pointers, alignment, workspace),
    moe_reduce_partials (count, null or misaligned parts) and moe_dense_ffn (a context that is
    not the one-expert layer), all decided before any CUDA call."""
    L = moe.load_library()
    A = 1 << 20
    T = 32
    h = moe.moe_create(256, 16, 2, 128, 1)
    hv = h.value
    ws = moe.moe_workspace_size(h, T)
    fp = L.moe_forward_partial
    # expert range outside [0, E), empty range
    assert fp(hv, A, A, None, -1, 4, A, A, A, A, A, A, T, A, A, ws, None) == moe.MOE_ERR_INVALID_ARG
    assert fp(hv, A, A, None, 14, 4, A, A, A, A, A, A, T, A, A, ws, None) == moe.MOE_ERR_INVALID_ARG
    assert fp(hv, A, A, None, 0, 0, A, A, A, A, A, A, T, A, A, ws, None) == moe.MOE_ERR_INVALID_ARG
    # the shared experts' pointers all or none
    assert fp(hv, A, A, None, 0, 4, A, A, A, A, None, A, T, A, A, ws, None) == \
        moe.MOE_ERR_INVALID_ARG
    # misaligned part, small workspace, no output
    assert fp(hv, A, A, None, 0, 4, A, A, A, None, None, None, T, A + 4, A, ws, None) == \
        moe.MOE_ERR_ALIGNMENT
    assert fp(hv, A, A, None, 0, 4, A, A, A, None, None, None, T, A, A, ws - 1, None) == \
        moe.MOE_ERR_WORKSPACE
    assert fp(hv, A, A, None, 0, 4, A, A, A, None, None, None, T, None, A, ws, None) == \
        moe.MOE_ERR_INVALID_ARG
    assert fp(hv, None, None, None, 0, 4, None, None, None, None, None, None, 0, None, None, 0,
              None) == moe.MOE_OK
    # reduce: 1..16 parts, each non-null and aligned
    P = ctypes.c_void_p
    parts = (P * 17)(*([A] * 17))
    assert L.moe_reduce_partials(hv, parts, 0, T, A, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_reduce_partials(hv, parts, 17, T, A, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_reduce_partials(hv, None, 2, T, A, None) == moe.MOE_ERR_INVALID_ARG
    holed = (P * 2)(A, None)
    assert L.moe_reduce_partials(hv, holed, 2, T, A, None) == moe.MOE_ERR_INVALID_ARG
    skew = (P * 2)(A, A + 4)
    assert L.moe_reduce_partials(hv, skew, 2, T, A, None) == moe.MOE_ERR_ALIGNMENT
    assert L.moe_reduce_partials(hv, parts, 2, T, A + 2, None) == moe.MOE_ERR_ALIGNMENT
    assert L.moe_reduce_partials(hv, parts, 2, 0, A, None) == moe.MOE_OK
    # dense layer: only the E=1, k=1, S=0 context
    assert L.moe_dense_ffn(hv, A, A, A, A, T, A, A, ws, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_dense_ffn_kernel_count(hv, T) == -1
    hd = moe.moe_create(256, 1, 1, 640, 0)
    wsd = moe.moe_workspace_size(hd, T)
    assert L.moe_dense_ffn(hd.value, A, A, A + 2, A, T, A, A, wsd, None) == moe.MOE_ERR_ALIGNMENT
    assert L.moe_dense_ffn(hd.value, A, A, A, A, T, A, A, wsd - 1, None) == moe.MOE_ERR_WORKSPACE
    assert L.moe_dense_ffn(hd.value, None, None, None, None, 0, None, None, 0, None) == moe.MOE_OK
    # the host-activation form takes the same checks
    assert L.moe_dense_ffn_host(hv, A, A, A, A, T, A, A, ws, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_dense_ffn_host(hd.value, A, A, A + 2, A, T, A, A, wsd, None) == \
        moe.MOE_ERR_ALIGNMENT
    assert L.moe_dense_ffn_host(hd.value, A, A, A, A, T, A, A, wsd - 1, None) == \
        moe.MOE_ERR_WORKSPACE
    assert L.moe_dense_ffn_host(hd.value, A, A, A, A, T, None, A, wsd, None) == \
        moe.MOE_ERR_INVALID_ARG
    assert L.moe_dense_ffn_host(hd.value, None, None, None, None, 0, None, None, 0, None) == \
        moe.MOE_OK
    # the weight-major GEMMs build the one-group schedule, and the K ranges of the split down
    # projection (up to 128 tokens) add their parts in the kernel while the output tiles'
    # counters fit (32): two launches; wider layers take the separate sum (three)
    assert L.moe_dense_ffn_kernel_count(hd.value, 16) == 2
    assert L.moe_dense_ffn_kernel_count(hd.value, 4096) == 2
    hw = moe.moe_create(8448, 1, 1, 640, 0)
    assert L.moe_dense_ffn_kernel_count(hw.value, 16) == 3
    assert L.moe_dense_ffn_kernel_count(hw.value, 4096) == 2


def test_fused_combine_option_is_fixed_at_create(lib, monkeypatch):
    """MOE_FUSED_COMBINE=1 at moe_create takes the combine out of moe_forward's launch list
    where it applies; the count of another context is unchanged (no device is needed to
    count).  Without a GPU the occupancy check cannot pass, so the fused form is not chosen
    and the counts agree."""
    monkeypatch.delenv("MOE_FUSED_COMBINE", raising=False)
    h0 = moe.moe_create(6144, 256, 8, 2048, 1)
    monkeypatch.setenv("MOE_FUSED_COMBINE", "1")
    h1 = moe.moe_create(6144, 256, 8, 2048, 1)
    monkeypatch.delenv("MOE_FUSED_COMBINE")
    n0 = moe.moe_forward_kernel_count(h0, 16)
    n1 = moe.moe_forward_kernel_count(h1, 16)
    assert n0 == 7
    assert n1 in (n0, n0 - 1)
    if not torch.cuda.is_available():
        assert n1 == n0
