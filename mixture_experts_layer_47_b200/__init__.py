"""B200 (sm_100a) forward pass of one Hy4-shaped mixture-of-experts FFN layer.

A thin ctypes binding over ``libmoe.so`` (declared in ``include/moe.h``).  The
functions carry the C names and only marshal arguments: check dtype, shape,
device and contiguity of torch tensors, pass their device pointers and the
current CUDA stream.  Every step of the layer runs in the library's kernels;
there is no CPU or PyTorch fallback.  If the library is missing the import
of any entry point raises.

    import mixture_experts_layer_47_b200 as moe
    h = moe.moe_create(6144, 256, 8, 2048, 1)
    ws = torch.empty(moe.moe_workspace_size(h, T), dtype=torch.uint8, device="cuda")
    moe.moe_forward(h, x, W_router, None, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down, y, ws)
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_TIMEOUT = 5
MOE_ERR_BAD_INDEX = 6
MOE_ERR_ALIGNMENT = 7

# Every symbol include/moe.h declares.
EXPORTS = ("moe_create", "moe_destroy", "moe_workspace_size", "moe_get_workspace_layout",
           "moe_route", "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_forward",
           "moe_forward_host", "moe_device_status", "moe_set_stage_events",
           "moe_dispatch_noalloc", "moe_selftest_wait_timeout", "moe_forward_kernel_count",
           "moe_status_string", "moe_expert_ffn_fp8", "moe_forward_fp8", "moe_forward_fp8_host",
           "moe_forward_partial", "moe_reduce_partials", "moe_dense_ffn", "moe_dense_ffn_host",
           "moe_dense_ffn_kernel_count", "moe_ihc_mix", "moe_forward_ihc")
MOE_STAGE_EVENTS = 7
STAGE_NAMES = ("router", "dispatch", "gather", "gate_up_gemm", "down_gemm", "combine")


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


class _Layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("status", "topk_idx", "topk_w", "counts", "offsets", "perm", "pos", "h_act",
                 "y_rows", "total", "router_partials", "router_ksplit")]


class Fp8ExpertWeights(ctypes.Structure):
    """struct moe_fp8_expert_weights: E4M3 codes and K-block-major scale bytes of one set."""
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("gate", "gate_scale", "up", "up_scale", "down", "down_scale")]


_lib = None


def load_library() -> ctypes.CDLL:
    """Load libmoe.so from this package's directory (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing; build it with `python -m mixture_experts_layer_47_b200.build`"
            " (the MoE layer has no fallback path)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    sig = {
        "moe_create": ([I, I, I, I, I, ctypes.POINTER(P)], I),
        "moe_destroy": ([P], I),
        "moe_workspace_size": ([P, I], Z),
        "moe_get_workspace_layout": ([P, I, ctypes.c_size_t, ctypes.POINTER(_Layout)], I),
        "moe_route": ([P, P, P, P, I, P, P, P, Z, P], I),
        "moe_dispatch": ([P, P, I, P, P, P, P, P, Z, P], I),
        "moe_expert_ffn": ([P, P, P, P, I, P, P, P, P, P, P, P, P, Z, P], I),
        "moe_combine": ([P, P, P, P, I, P, P], I),
        "moe_forward": ([P, P, P, P, P, P, P, P, P, P, I, P, P, Z, P], I),
        "moe_forward_host": ([P, P, P, P, P, P, P, P, P, P, I, P, P, Z, P], I),
        "moe_device_status": ([P, I, P, P, ctypes.POINTER(ctypes.c_int32)], I),
        "moe_set_stage_events": ([P, ctypes.POINTER(P), I], I),
        "moe_dispatch_noalloc": ([P, P, I, P, P, P, P, P], I),
        "moe_selftest_wait_timeout": ([P, Z, ctypes.c_ulonglong, P], I),
        "moe_forward_kernel_count": ([P, I], I),
        "moe_status_string": ([I], ctypes.c_char_p),
        "moe_expert_ffn_fp8": ([P, P, P, P, I, ctypes.POINTER(Fp8ExpertWeights),
                                ctypes.POINTER(Fp8ExpertWeights), P, P, Z, P], I),
        "moe_forward_fp8": ([P, P, P, P, ctypes.POINTER(Fp8ExpertWeights),
                             ctypes.POINTER(Fp8ExpertWeights), I, P, P, Z, P], I),
        "moe_forward_fp8_host": ([P, P, P, P, ctypes.POINTER(Fp8ExpertWeights),
                                  ctypes.POINTER(Fp8ExpertWeights), I, P, P, Z, P], I),
        "moe_forward_partial": ([P, P, P, P, I, I, P, P, P, P, P, P, I, P, P, Z, P], I),
        "moe_reduce_partials": ([P, ctypes.POINTER(P), I, I, P, P], I),
        "moe_dense_ffn": ([P, P, P, P, P, I, P, P, Z, P], I),
        "moe_dense_ffn_host": ([P, P, P, P, P, I, P, P, Z, P], I),
        "moe_dense_ffn_kernel_count": ([P, I], I),
        "moe_ihc_mix": ([P, P, I, P, I, P, P], I),
        "moe_forward_ihc": ([P, P, I, P, P, P, P, P, P, P, P, P, P, P, I, P, P, Z, P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().moe_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != MOE_OK:
        raise MoEError(status, what)


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor], dtype: torch.dtype, name: str, shape=None,
         device_kind: str = "cuda") -> Optional[int]:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.device.type != device_kind:
        raise ValueError(f"{name}: expected a {device_kind} tensor, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr()


class Handle:
    """A layer context (``moe_create``) that remembers its shape."""

    def __init__(self, d_model: int, n_experts: int, top_k: int, d_ff: int, n_shared: int):
        lib = load_library()
        h = ctypes.c_void_p()
        _check(lib.moe_create(d_model, n_experts, top_k, d_ff, n_shared, ctypes.byref(h)),
               "moe_create")
        self._h = h
        self.d, self.E, self.k, self.F, self.S = d_model, n_experts, top_k, d_ff, n_shared

    @property
    def value(self):
        return self._h

    def close(self):
        if self._h is not None and self._h.value:
            load_library().moe_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_create(d_model: int, n_experts: int, top_k: int, d_ff: int, n_shared: int) -> Handle:
    return Handle(d_model, n_experts, top_k, d_ff, n_shared)


def moe_destroy(h: Handle) -> None:
    h.close()


def moe_workspace_size(h: Handle, T: int) -> int:
    return int(load_library().moe_workspace_size(h.value, int(T)))


def moe_get_workspace_layout(h: Handle, T: int, workspace_addr: int = 0) -> dict:
    out = _Layout()
    _check(load_library().moe_get_workspace_layout(h.value, int(T), int(workspace_addr),
                                                   ctypes.byref(out)), "moe_get_workspace_layout")
    return {name: getattr(out, name) for name, _ in _Layout._fields_}


def _ws(workspace: torch.Tensor):
    if workspace.dtype != torch.uint8 or workspace.device.type != "cuda":
        raise TypeError("workspace must be a CUDA uint8 tensor")
    return workspace.data_ptr(), workspace.numel()


def moe_route(h: Handle, x, W_router, bias, topk_idx, topk_w, workspace, stream=None) -> None:
    T = x.shape[0]
    wp, wn = _ws(workspace)
    _check(load_library().moe_route(
        h.value, _ptr(x, torch.bfloat16, "x", (T, h.d)),
        _ptr(W_router, torch.float32, "W_router", (h.E, h.d)),
        _ptr(bias, torch.float32, "bias", (h.E,)), T,
        _ptr(topk_idx, torch.int32, "topk_idx", (T, h.k)),
        _ptr(topk_w, torch.float32, "topk_w", (T, h.k)), wp, wn, _stream(stream)), "moe_route")


def moe_dispatch(h: Handle, topk_idx, counts, offsets, perm, pos, workspace, stream=None) -> None:
    T = topk_idx.shape[0]
    n = T * h.k
    wp, wn = _ws(workspace)
    _check(load_library().moe_dispatch(
        h.value, _ptr(topk_idx, torch.int32, "topk_idx", (T, h.k)), T,
        _ptr(counts, torch.int32, "counts", (h.E,)),
        _ptr(offsets, torch.int32, "offsets", (h.E + 1,)),
        _ptr(perm, torch.int32, "perm", (n,)), _ptr(pos, torch.int32, "pos", (n,)), wp, wn,
        _stream(stream)), "moe_dispatch")


def moe_dispatch_noalloc(h: Handle, topk_idx, counts, offsets, perm, pos, stream=None) -> None:
    """moe_dispatch without a workspace, for callers that cannot allocate device memory
    (the library's fixed scratch is used instead; see include/moe.h for its limits)."""
    T = topk_idx.shape[0]
    n = T * h.k
    _check(load_library().moe_dispatch_noalloc(
        h.value, _ptr(topk_idx, torch.int32, "topk_idx", (T, h.k)), T,
        _ptr(counts, torch.int32, "counts", (h.E,)),
        _ptr(offsets, torch.int32, "offsets", (h.E + 1,)),
        _ptr(perm, torch.int32, "perm", (n,)), _ptr(pos, torch.int32, "pos", (n,)),
        _stream(stream)), "moe_dispatch_noalloc")


def _weights(h: Handle, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down):
    return (_ptr(W_gate, torch.bfloat16, "W_gate", (h.E, h.F, h.d)),
            _ptr(W_up, torch.bfloat16, "W_up", (h.E, h.F, h.d)),
            _ptr(W_down, torch.bfloat16, "W_down", (h.E, h.d, h.F)),
            _ptr(Ws_gate, torch.bfloat16, "Ws_gate", (h.S, h.F, h.d)) if h.S else None,
            _ptr(Ws_up, torch.bfloat16, "Ws_up", (h.S, h.F, h.d)) if h.S else None,
            _ptr(Ws_down, torch.bfloat16, "Ws_down", (h.S, h.d, h.F)) if h.S else None)


def moe_expert_ffn(h: Handle, x, perm, offsets, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down,
                   Y, workspace, stream=None) -> None:
    T = x.shape[0]
    rows = T * h.k + h.S * T
    wp, wn = _ws(workspace)
    _check(load_library().moe_expert_ffn(
        h.value, _ptr(x, torch.bfloat16, "x", (T, h.d)),
        _ptr(perm, torch.int32, "perm", (T * h.k,)),
        _ptr(offsets, torch.int32, "offsets", (h.E + 1,)), T,
        *_weights(h, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down),
        _ptr(Y, torch.float32, "Y", (rows, h.d)), wp, wn, _stream(stream)), "moe_expert_ffn")


def _fp8_set(h: Handle, fs, n: int, name: str):
    """A Fp8ExpertWeights for an object with uint8 tensors gate, gate_scale, up, up_scale,
    down, down_scale (e.g. ``workloads.Fp8Set``); None when n == 0."""
    if n == 0:
        return None
    if fs is None:
        raise ValueError(f"{name}: FP8 weights required")
    d, F = h.d, h.F
    shapes = dict(gate=(n, F, d), gate_scale=(n, d // 32, F), up=(n, F, d),
                  up_scale=(n, d // 32, F), down=(n, d, F), down_scale=(n, F // 32, d))
    return Fp8ExpertWeights(**{k: _ptr(getattr(fs, k), torch.uint8, f"{name}.{k}", shp)
                               for k, shp in shapes.items()})


def _byref(s):
    return None if s is None else ctypes.byref(s)


def moe_expert_ffn_fp8(h: Handle, x, perm, offsets, routed, shared, Y, workspace,
                       stream=None) -> None:
    """moe_expert_ffn with FP8 expert weights (``routed``/``shared``: see ``_fp8_set``)."""
    T = x.shape[0]
    rows = T * h.k + h.S * T
    wp, wn = _ws(workspace)
    r, sh = _fp8_set(h, routed, h.E, "routed"), _fp8_set(h, shared, h.S, "shared")
    _check(load_library().moe_expert_ffn_fp8(
        h.value, _ptr(x, torch.bfloat16, "x", (T, h.d)),
        _ptr(perm, torch.int32, "perm", (T * h.k,)),
        _ptr(offsets, torch.int32, "offsets", (h.E + 1,)), T, _byref(r), _byref(sh),
        _ptr(Y, torch.float32, "Y", (rows, h.d)), wp, wn, _stream(stream)),
        "moe_expert_ffn_fp8")


def moe_forward_fp8(h: Handle, x, W_router, bias, routed, shared, y, workspace,
                    stream=None) -> None:
    T = x.shape[0]
    wp, wn = _ws(workspace)
    r, sh = _fp8_set(h, routed, h.E, "routed"), _fp8_set(h, shared, h.S, "shared")
    _check(load_library().moe_forward_fp8(
        h.value, _ptr(x, torch.bfloat16, "x", (T, h.d)),
        _ptr(W_router, torch.float32, "W_router", (h.E, h.d)),
        _ptr(bias, torch.float32, "bias", (h.E,)), _byref(r), _byref(sh), T,
        _ptr(y, torch.bfloat16, "y", (T, h.d)), wp, wn, _stream(stream)), "moe_forward_fp8")


def moe_forward_fp8_host(h: Handle, x_host, W_router, bias, routed, shared, y_host, workspace,
                         stream=None) -> None:
    """x_host / y_host: CPU bf16 tensors (pinned for asynchronous copies)."""
    T = x_host.shape[0]
    wp, wn = _ws(workspace)
    r, sh = _fp8_set(h, routed, h.E, "routed"), _fp8_set(h, shared, h.S, "shared")
    _check(load_library().moe_forward_fp8_host(
        h.value, _ptr(x_host, torch.bfloat16, "x_host", (T, h.d), "cpu"),
        _ptr(W_router, torch.float32, "W_router", (h.E, h.d)),
        _ptr(bias, torch.float32, "bias", (h.E,)), _byref(r), _byref(sh), T,
        _ptr(y_host, torch.bfloat16, "y_host", (T, h.d), "cpu"), wp, wn, _stream(stream)),
        "moe_forward_fp8_host")


def moe_combine(h: Handle, Y, topk_w, pos, y, stream=None) -> None:
    T = topk_w.shape[0]
    rows = T * h.k + h.S * T
    _check(load_library().moe_combine(
        h.value, _ptr(Y, torch.float32, "Y", (rows, h.d)),
        _ptr(topk_w, torch.float32, "topk_w", (T, h.k)),
        _ptr(pos, torch.int32, "pos", (T * h.k,)), T,
        _ptr(y, torch.bfloat16, "y", (T, h.d)), _stream(stream)), "moe_combine")


def moe_forward(h: Handle, x, W_router, bias, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down, y,
                workspace, stream=None) -> None:
    T = x.shape[0]
    wp, wn = _ws(workspace)
    _check(load_library().moe_forward(
        h.value, _ptr(x, torch.bfloat16, "x", (T, h.d)),
        _ptr(W_router, torch.float32, "W_router", (h.E, h.d)),
        _ptr(bias, torch.float32, "bias", (h.E,)),
        *_weights(h, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down), T,
        _ptr(y, torch.bfloat16, "y", (T, h.d)), wp, wn, _stream(stream)), "moe_forward")


def moe_forward_host(h: Handle, x_host, W_router, bias, W_gate, W_up, W_down, Ws_gate, Ws_up,
                     Ws_down, y_host, workspace, stream=None) -> None:
    """x_host / y_host: CPU bf16 tensors (pinned for asynchronous copies)."""
    T = x_host.shape[0]
    wp, wn = _ws(workspace)
    _check(load_library().moe_forward_host(
        h.value, _ptr(x_host, torch.bfloat16, "x_host", (T, h.d), "cpu"),
        _ptr(W_router, torch.float32, "W_router", (h.E, h.d)),
        _ptr(bias, torch.float32, "bias", (h.E,)),
        *_weights(h, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down), T,
        _ptr(y_host, torch.bfloat16, "y_host", (T, h.d), "cpu"), wp, wn, _stream(stream)),
        "moe_forward_host")


def moe_forward_partial(h: Handle, x, W_router, bias, expert_begin: int, W_gate, W_up, W_down,
                        Ws_gate, Ws_up, Ws_down, y_partial, workspace, stream=None) -> None:
    """One shard's fp32 part of the layer output (tensor parallelism over d_ff: the handle's
    d_ff is the slice width; expert parallelism: W_* hold experts expert_begin ... of the
    layer).  Ws_* are all None when this shard adds no shared-expert term."""
    T = x.shape[0]
    n_local = W_gate.shape[0]
    wp, wn = _ws(workspace)
    shared = Ws_gate is not None and h.S > 0
    _check(load_library().moe_forward_partial(
        h.value, _ptr(x, torch.bfloat16, "x", (T, h.d)),
        _ptr(W_router, torch.float32, "W_router", (h.E, h.d)),
        _ptr(bias, torch.float32, "bias", (h.E,)), int(expert_begin), int(n_local),
        _ptr(W_gate, torch.bfloat16, "W_gate", (n_local, h.F, h.d)),
        _ptr(W_up, torch.bfloat16, "W_up", (n_local, h.F, h.d)),
        _ptr(W_down, torch.bfloat16, "W_down", (n_local, h.d, h.F)),
        _ptr(Ws_gate, torch.bfloat16, "Ws_gate", (h.S, h.F, h.d)) if shared else None,
        _ptr(Ws_up, torch.bfloat16, "Ws_up", (h.S, h.F, h.d)) if shared else None,
        _ptr(Ws_down, torch.bfloat16, "Ws_down", (h.S, h.d, h.F)) if shared else None, T,
        _ptr(y_partial, torch.float32, "y_partial", (T, h.d)), wp, wn, _stream(stream)),
        "moe_forward_partial")


def moe_dense_ffn(h: Handle, x, W_gate, W_up, W_down, y, workspace, stream=None) -> None:
    """The dense SwiGLU FFN layer (h created with n_experts=1, top_k=1, n_shared=0).
    W_gate, W_up: [F, d] or [1, F, d]; W_down: [d, F] or [1, d, F]."""
    T = x.shape[0]
    wp, wn = _ws(workspace)
    Wg, Wu, Wd = (W.reshape(W.shape[-2:]) if W.dim() == 3 else W
                  for W in (W_gate, W_up, W_down))
    _check(load_library().moe_dense_ffn(
        h.value, _ptr(x, torch.bfloat16, "x", (T, h.d)),
        _ptr(Wg, torch.bfloat16, "W_gate", (h.F, h.d)),
        _ptr(Wu, torch.bfloat16, "W_up", (h.F, h.d)),
        _ptr(Wd, torch.bfloat16, "W_down", (h.d, h.F)), T,
        _ptr(y, torch.bfloat16, "y", (T, h.d)), wp, wn, _stream(stream)), "moe_dense_ffn")


def moe_dense_ffn_host(h: Handle, x_host, W_gate, W_up, W_down, y_host, workspace,
                       stream=None) -> None:
    """moe_dense_ffn with x_host / y_host CPU bf16 tensors (pinned for asynchronous copies)."""
    T = x_host.shape[0]
    wp, wn = _ws(workspace)
    Wg, Wu, Wd = (W.reshape(W.shape[-2:]) if W.dim() == 3 else W
                  for W in (W_gate, W_up, W_down))
    _check(load_library().moe_dense_ffn_host(
        h.value, _ptr(x_host, torch.bfloat16, "x_host", (T, h.d), "cpu"),
        _ptr(Wg, torch.bfloat16, "W_gate", (h.F, h.d)),
        _ptr(Wu, torch.bfloat16, "W_up", (h.F, h.d)),
        _ptr(Wd, torch.bfloat16, "W_down", (h.d, h.F)), T,
        _ptr(y_host, torch.bfloat16, "y_host", (T, h.d), "cpu"), wp, wn, _stream(stream)),
        "moe_dense_ffn_host")


def moe_reduce_partials(h: Handle, partials, y, stream=None) -> None:
    """y = bf16(sum of the fp32 partial outputs, added in list order)."""
    T = y.shape[0]
    arr = (ctypes.c_void_p * len(partials))(
        *[_ptr(p, torch.float32, f"partials[{i}]", (T, h.d)) for i, p in enumerate(partials)])
    _check(load_library().moe_reduce_partials(
        h.value, arr, len(partials), T, _ptr(y, torch.bfloat16, "y", (T, h.d)),
        _stream(stream)), "moe_reduce_partials")


def moe_device_status(h: Handle, T: int, workspace, stream=None) -> tuple:
    """Synchronise the stream; return (status, raw device word) of the workspace."""
    detail = ctypes.c_int32(0)
    st = load_library().moe_device_status(h.value, int(T), workspace.data_ptr(), _stream(stream),
                                          ctypes.byref(detail))
    return int(st), int(detail.value)


def moe_set_stage_events(h: Handle, events) -> None:
    """Record the given 7 torch.cuda.Events at the stage boundaries of later forwards
    (None switches it off).  Each event must have been recorded once already so that
    its CUDA handle exists."""
    lib = load_library()
    if events is None:
        _check(lib.moe_set_stage_events(h.value, None, 0), "moe_set_stage_events")
        return
    arr = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
    _check(lib.moe_set_stage_events(h.value, arr, len(events)), "moe_set_stage_events")


def moe_selftest_wait_timeout(workspace, timeout_ns: int, stream=None) -> None:
    """Run a kernel whose bounded wait is made to expire (see include/moe.h)."""
    wp, wn = _ws(workspace)
    _check(load_library().moe_selftest_wait_timeout(wp, wn, int(timeout_ns), _stream(stream)),
           "moe_selftest_wait_timeout")


def moe_forward_kernel_count(h: Handle, T: int) -> int:
    return int(load_library().moe_forward_kernel_count(h.value, int(T)))


def moe_ihc_mix(h: Handle, H, alpha, x, stream=None) -> None:
    """x = bf16(sum_j alpha[j] H[:, j]) for streams H [T, n, d] (bf16) and alpha [n] (fp32)."""
    T, n = H.shape[0], H.shape[1]
    _check(load_library().moe_ihc_mix(
        h.value, _ptr(H, torch.bfloat16, "H", (T, n, h.d)), n,
        _ptr(alpha, torch.float32, "alpha", (n,)), T, _ptr(x, torch.bfloat16, "x", (T, h.d)),
        _stream(stream)), "moe_ihc_mix")


def moe_forward_ihc(h: Handle, H, alpha, B, gamma, W_router, bias, W_gate, W_up, W_down,
                    Ws_gate, Ws_up, Ws_down, H_out, workspace, stream=None) -> None:
    """The layer inside n residual streams: H_out[:, i] = H[:, i] + sum_j B[i, j] H[:, j]
    + gamma[i] * layer(sum_j alpha[j] H[:, j])."""
    T, n = H.shape[0], H.shape[1]
    wp, wn = _ws(workspace)
    _check(load_library().moe_forward_ihc(
        h.value, _ptr(H, torch.bfloat16, "H", (T, n, h.d)), n,
        _ptr(alpha, torch.float32, "alpha", (n,)), _ptr(B, torch.float32, "B", (n, n)),
        _ptr(gamma, torch.float32, "gamma", (n,)),
        _ptr(W_router, torch.float32, "W_router", (h.E, h.d)),
        _ptr(bias, torch.float32, "bias", (h.E,)),
        *_weights(h, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down), T,
        _ptr(H_out, torch.bfloat16, "H_out", (T, n, h.d)), wp, wn, _stream(stream)),
        "moe_forward_ihc")


def moe_dense_ffn_kernel_count(h: Handle, T: int) -> int:
    return int(load_library().moe_dense_ffn_kernel_count(h.value, int(T)))


def moe_status_string(status: int) -> str:
    return status_string(status)


def workspace_views(h: Handle, T: int, workspace: torch.Tensor) -> dict:
    """Typed views of the intermediates moe_forward leaves in the workspace."""
    L = moe_get_workspace_layout(h, T, workspace.data_ptr())
    rows = T * h.k + h.S * T

    def view(off, n, dtype):
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        return workspace[off:off + nbytes].view(dtype)

    ks = L["router_ksplit"]
    return dict(
        status=view(L["status"], 1, torch.int32),
        router_partials=view(L["router_partials"], ks * T * h.E, torch.float32).view(ks, T, h.E),
        topk_idx=view(L["topk_idx"], T * h.k, torch.int32).view(T, h.k),
        topk_w=view(L["topk_w"], T * h.k, torch.float32).view(T, h.k),
        counts=view(L["counts"], h.E, torch.int32),
        offsets=view(L["offsets"], h.E + 1, torch.int32),
        perm=view(L["perm"], T * h.k, torch.int32),
        pos=view(L["pos"], T * h.k, torch.int32),
        h_act=view(L["h_act"], rows * h.F, torch.bfloat16).view(rows, h.F),
        y_rows=view(L["y_rows"], rows * h.d, torch.bfloat16).view(rows, h.d),
    )


class MoELayer:
    """Convenience owner of a context, its weights and a workspace sized for up to max_T."""

    def __init__(self, inputs, max_T: Optional[int] = None, device="cuda"):
        wl = inputs.wl
        self.inputs = inputs
        self.h = moe_create(wl.d, wl.E, wl.k, wl.F, wl.S)
        self.max_T = max_T or wl.T
        self.workspace = torch.empty(moe_workspace_size(self.h, self.max_T), dtype=torch.uint8,
                                     device=device)

    def weights(self):
        i = self.inputs
        return (i.W_gate, i.W_up, i.W_down, i.Ws_gate, i.Ws_up, i.Ws_down)

    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, stream=None):
        if x.shape[0] > self.max_T:
            raise ValueError("more tokens than the workspace was sized for")
        if y is None:
            y = torch.empty_like(x)
        i = self.inputs
        moe_forward(self.h, x, i.W_router, i.bias, *self.weights(), y, self.workspace, stream)
        return y
