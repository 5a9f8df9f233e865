"""fp64 CPU oracle of the MoE FFN layer forward -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA path
(``mixture_experts_layer_47_b200``) and neither imports the other; the only
common module is ``workloads`` (seeded input draws, no layer arithmetic).

The arithmetic lives in ``moe_oracle.c`` (plain C, fp64, OpenMP over tokens);
this file builds it with gcc and marshals numpy / CPU torch arrays.  Each step
follows the pages' statement of the layer (m.xxqk.cn Hy4-preview MoE explainer
section 2.1 "FFN split" and 2.2 "router mechanism"; ZAKER Hy4 Preview release
news, MoE paragraph) with the readings written at the top of ``moe_oracle.c``.

FP8 expert weights (the format the Hy4 pages' FP8 checkpoint implies but does
not specify; the stated choice is described in ``workloads``): ``e4m3_value``
decodes one code from the OCP FP8 E4M3 definition, ``dequant_fp8`` applies the
per-32-element power-of-two scales, and ``fp8_as_bf16`` hands the decoded
weights to the bf16 layer above as exact bf16 bit patterns (every decoded
weight has at most 4 significant bits, so the conversion is exact; it is
checked, not assumed).

Pinning: every function here is checked in ``tests/test_oracle.py`` against
values fixed independently of it (hand-derived closed forms in
``tests/golden/``, numpy/torch float64 library routines on special cases,
brute force, and invariants).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Mapping, Optional, Sequence, Union

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmoe_oracle.so")
_lib = None

_ERRORS = {1: "bad argument", 2: "out of memory", 3: "missing expert weights"}


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so next to it (gcc, -O2, OpenMP).

    -O2 without -ffast-math keeps every floating-point sum in source order.
    """
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_router_logits.argtypes = [P, P, P, I, I, I, P]
        lib.oracle_route.argtypes = [P, I, I, I, P, P, P]
        lib.oracle_dispatch.argtypes = [P, I, I, I, P, P, P, P]
        lib.oracle_moe_ffn_tokens.argtypes = [P, I, I, I, I, I, I, P, P, P, P, P, P, P, P,
                                              P, I, P]
        lib.oracle_expert_one.argtypes = [P, I, I, P, P, P, P, P]
        lib.oracle_num_threads.argtypes = []
        lib.oracle_combine.argtypes = [P, P, P, I, I, I, I, P]
        for f in ("oracle_router_logits", "oracle_route", "oracle_dispatch",
                  "oracle_moe_ffn_tokens", "oracle_expert_one", "oracle_num_threads",
                  "oracle_combine"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {what}: {_ERRORS.get(rc, rc)}")


def _np(a, dtype) -> np.ndarray:
    """A C-contiguous numpy array of ``dtype``; bf16 torch tensors become uint16 bit patterns."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach()
            if a.device.type != "cpu":
                a = a.cpu()
            if a.dtype == torch.bfloat16:
                a = a.contiguous().view(torch.int16).numpy().view(np.uint16)
            else:
                a = a.contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def num_threads() -> int:
    return _load().oracle_num_threads()


def router_logits(x, W_router, bias=None) -> np.ndarray:
    """logits[t, e] = sum_j x[t, j] W_router[e, j] + bias[e], in fp64."""
    x = _np(x, np.uint16)
    Wr = _np(W_router, np.float32)
    b = None if bias is None else _np(bias, np.float32)
    T, d = x.shape
    E = Wr.shape[0]
    assert Wr.shape == (E, d)
    out = np.empty((T, E), np.float64)
    _check(_load().oracle_router_logits(_ptr(x), _ptr(Wr), _ptr(b), T, d, E, _ptr(out)),
           "router_logits")
    return out


def route(logits: np.ndarray, k: int):
    """Softmax gate, top-k by (p desc, expert asc), renormalised weights.

    Returns idx [T, k] int32, w [T, k] fp64, margin [T] fp64 (l_(k) - l_(k+1)).
    """
    logits = np.ascontiguousarray(logits, dtype=np.float64)
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    margin = np.empty((T,), np.float64)
    _check(_load().oracle_route(_ptr(logits), T, E, k, _ptr(idx), _ptr(w), _ptr(margin)),
           "route")
    return idx, w, margin


def dispatch(idx, E: int):
    """Stable counting sort of the T*k slots by expert: counts, offsets, perm, pos."""
    idx = _np(idx, np.int32)
    T, k = idx.shape
    counts = np.empty((E,), np.int32)
    offsets = np.empty((E + 1,), np.int32)
    perm = np.empty((T * k,), np.int32)
    pos = np.empty((T * k,), np.int32)
    _check(_load().oracle_dispatch(_ptr(idx), T, E, k, _ptr(counts), _ptr(offsets), _ptr(perm),
                                   _ptr(pos)), "dispatch")
    return counts, offsets, perm, pos


ExpertWeights = Union["np.ndarray", Mapping[int, "np.ndarray"], Sequence]


def _expert_ptr_array(W, n: int, shape) -> tuple:
    """Array of n per-expert pointers from a stacked [n, r, c] array or a {e: [r, c]} mapping.

    Returns (ctypes array, list of arrays kept alive)."""
    keep = []
    arr = (ctypes.c_void_p * max(n, 1))()
    if isinstance(W, Mapping):
        for e, We in W.items():
            a = _np(We, np.uint16).reshape(shape)
            keep.append(a)
            arr[int(e)] = a.ctypes.data
    else:
        a = _np(W, np.uint16)
        assert a.shape == (n,) + tuple(shape), (a.shape, n, shape)
        keep.append(a)
        step = a.strides[0]
        for e in range(n):
            arr[e] = a.ctypes.data + e * step
    return arr, keep


def moe_ffn_tokens(x, idx, w, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down,
                   tokens: Optional[Sequence[int]] = None, *, E: int, F: int, S: int) -> np.ndarray:
    """y for the chosen tokens: sum of shared experts + sum_i w_i * expert_{idx_i}, fp64.

    Expert weights may be stacked arrays ([E, F, d] / [E, d, F]) or mappings
    {expert: [F, d] / [d, F]} holding only the experts the chosen tokens use.
    """
    x = _np(x, np.uint16)
    T, d = x.shape
    idx = _np(idx, np.int32)
    k = idx.shape[1]
    w = np.ascontiguousarray(w, dtype=np.float64)
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    g_arr, k1 = _expert_ptr_array(W_gate, E, (F, d))
    u_arr, k2 = _expert_ptr_array(W_up, E, (F, d))
    d_arr, k3 = _expert_ptr_array(W_down, E, (d, F))
    sg_arr, k4 = _expert_ptr_array(Ws_gate, S, (F, d))
    su_arr, k5 = _expert_ptr_array(Ws_up, S, (F, d))
    sd_arr, k6 = _expert_ptr_array(Ws_down, S, (d, F))
    y = np.empty((len(tokens), d), np.float64)
    rc = _load().oracle_moe_ffn_tokens(
        _ptr(x), T, d, E, k, F, S, _ptr(idx), _ptr(w),
        ctypes.cast(g_arr, ctypes.c_void_p), ctypes.cast(u_arr, ctypes.c_void_p),
        ctypes.cast(d_arr, ctypes.c_void_p), ctypes.cast(sg_arr, ctypes.c_void_p),
        ctypes.cast(su_arr, ctypes.c_void_p), ctypes.cast(sd_arr, ctypes.c_void_p),
        _ptr(tokens), len(tokens), _ptr(y))
    del k1, k2, k3, k4, k5, k6
    _check(rc, "moe_ffn_tokens")
    return y


def expert_one(xrow, W_gate_e, W_up_e, W_down_e):
    """h = silu(Wg x) * (Wu x) and y = Wd h for one token and one expert, fp64."""
    xr = _np(xrow, np.uint16).reshape(-1)
    d = xr.shape[0]
    Wg = _np(W_gate_e, np.uint16)
    Wu = _np(W_up_e, np.uint16)
    Wd = _np(W_down_e, np.uint16)
    F = Wg.shape[0]
    assert Wg.shape == (F, d) and Wu.shape == (F, d) and Wd.shape == (d, F)
    h = np.empty((F,), np.float64)
    y = np.empty((d,), np.float64)
    _check(_load().oracle_expert_one(_ptr(xr), d, F, _ptr(Wg), _ptr(Wu), _ptr(Wd), _ptr(h),
                                     _ptr(y)), "expert_one")
    return h, y


def combine(Y_rows, w, pos, T: int, k: int, S: int) -> np.ndarray:
    """y[t] = sum_s Y_rows[T*k + s*T + t] + sum_i w[t, i] * Y_rows[pos[t*k + i]], fp64."""
    Yr = np.ascontiguousarray(Y_rows, dtype=np.float64)
    w = np.ascontiguousarray(w, dtype=np.float64)
    pos = _np(pos, np.int32)
    d = Yr.shape[1]
    assert Yr.shape[0] == T * k + S * T and w.shape == (T, k) and pos.size == T * k
    y = np.empty((T, d), np.float64)
    _check(_load().oracle_combine(_ptr(Yr), _ptr(w), _ptr(pos), T, k, S, d, _ptr(y)), "combine")
    return y


def forward(inp, tokens: Optional[Sequence[int]] = None, idx_override=None,
            weights: Optional[dict] = None) -> dict:
    """The whole layer for ``workloads.Inputs`` ``inp`` (CPU tensors or numpy).

    Routing (logits, idx, w, margin) and dispatch (counts, offsets, perm, pos)
    cover every token; y covers ``tokens`` (default: all).  ``idx_override``
    replaces the oracle's own top-k choice (the gate weights are then the
    softmax renormalised over the given experts, in the given order).
    ``weights`` optionally supplies per-expert mappings in place of the stacked
    weights of ``inp`` (keys 'W_gate', 'W_up', 'W_down', 'Ws_gate', 'Ws_up', 'Ws_down').
    """
    wl = inp.wl
    logits = router_logits(inp.x, inp.W_router, inp.bias)
    idx, w, margin = route(logits, wl.k)
    if idx_override is not None:
        idx = _np(idx_override, np.int32).copy()
        w = renormalised_gates(logits, idx)
    counts, offsets, perm, pos = dispatch(idx, wl.E)
    W = dict(W_gate=inp.W_gate, W_up=inp.W_up, W_down=inp.W_down,
             Ws_gate=inp.Ws_gate, Ws_up=inp.Ws_up, Ws_down=inp.Ws_down)
    if weights:
        W.update(weights)
    y = moe_ffn_tokens(inp.x, idx, w, W["W_gate"], W["W_up"], W["W_down"], W["Ws_gate"],
                       W["Ws_up"], W["Ws_down"], tokens, E=wl.E, F=wl.F, S=wl.S)
    return dict(logits=logits, idx=idx, w=w, margin=margin, counts=counts, offsets=offsets,
                perm=perm, pos=pos, y=y,
                tokens=np.arange(wl.T) if tokens is None else np.asarray(tokens))


def shard_output(x, idx, w, W_gate, W_up, W_down, Ws_gate=None, Ws_up=None, Ws_down=None,
                 expert_begin: int = 0, tokens: Optional[Sequence[int]] = None) -> np.ndarray:
    """One shard's part of the layer output, fp64, for the sharded deployments the pages name
    (gpuvram.cloud "Tencent Hy4 preview" model card: vLLM TP8 on eight GPUs; pgsm.cn Hy4
    preview hands-on, vLLM section: expert parallelism for MoE).  A shard holds routed experts
    expert_begin .. expert_begin + n - 1 (W_gate, W_up [n, F, d], W_down [n, d, F], possibly
    only a slice of d_ff: rows of W_gate/W_up and the matching columns of W_down) and, if
    Ws_* are given, the shared experts (or their slices):

        part[t] = sum_s FFN_s(x_t) + sum over i with expert_begin <= idx[t, i] < expert_begin + n
                  of w[t, i] * FFN_{idx[t, i]}(x_t)

    summed in that order, each FFN term computed by ``expert_one``.  Summing the parts of
    all shards gives the layer (SwiGLU acts feature by feature, and every slot's expert lives
    on exactly one shard)."""
    xs = _np(x, np.uint16)
    idx = np.asarray(idx)
    w = np.asarray(w, np.float64)
    T, d = xs.shape
    n = W_gate.shape[0]
    toks = range(T) if tokens is None else [int(t) for t in tokens]
    out = np.zeros((len(toks), d), np.float64)
    for row, t in enumerate(toks):
        if Ws_gate is not None:
            for s in range(Ws_gate.shape[0]):
                out[row] += expert_one(xs[t], Ws_gate[s], Ws_up[s], Ws_down[s])[1]
        for i in range(idx.shape[1]):
            e = int(idx[t, i]) - expert_begin
            if 0 <= e < n:
                out[row] += w[t, i] * expert_one(xs[t], W_gate[e], W_up[e], W_down[e])[1]
    return out


# ----------------------------------------------------------------------------
# iHC: the layer inside four parallel residual streams.  ZAKER "Tencent releases and
# open-sources Hy4 Preview", iHC paragraphs: identity Hyper-Connections widen the single
# residual stream to 4 parallel streams that are recombined at every layer, and keep a stable
# identity path under the learned exchange between streams.  The pages give no formula; the
# reading (static hyper-connections with the identity term kept exactly):
#   layer input   x[t]     = sum_j alpha[j] * H[t, j]
#   stream update H'[t, i] = H[t, i] + sum_j B[i, j] * H[t, j] + gamma[i] * y[t]
# with y = the MoE layer on x, and alpha [n], B [n, n], gamma [n] the learned coefficients.
# ----------------------------------------------------------------------------
def ihc_mix_in(H, alpha) -> np.ndarray:
    """x[t] = sum_j alpha[j] * H[t, j] in fp64, j in order.  H: [T, n, d] bf16 (uint16 bits
    or a CPU bf16 tensor) or float; returns [T, d] fp64."""
    Hf = _as_f64(H)
    alpha = np.asarray(alpha, np.float64)
    T, n, d = Hf.shape
    x = np.zeros((T, d), np.float64)
    for j in range(n):
        x += alpha[j] * Hf[:, j, :]
    return x


def ihc_update(H, B, gamma, y) -> np.ndarray:
    """H'[t, i] = H[t, i] + sum_j B[i, j] * H[t, j] + gamma[i] * y[t] in fp64: the identity
    path, then the exchange terms j in order, then the layer's output."""
    Hf = _as_f64(H)
    B = np.asarray(B, np.float64)
    gamma = np.asarray(gamma, np.float64)
    y = np.asarray(y, np.float64)
    T, n, d = Hf.shape
    out = np.empty_like(Hf)
    for i in range(n):
        acc = Hf[:, i, :].copy()
        for j in range(n):
            acc += B[i, j] * Hf[:, j, :]
        out[:, i, :] = acc + gamma[i] * y
    return out


def _as_f64(a) -> np.ndarray:
    """bf16 bit patterns (uint16) or a bf16 tensor -> exact fp64; float arrays as they are."""
    if hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        a = a.view(dtype=__import__("torch").int16).numpy().view(np.uint16)
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def renormalised_gates(logits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """Gate weights for a given expert choice: softmax over all logits, renormalised over idx."""
    logits = np.asarray(logits, np.float64)
    T, E = logits.shape
    k = idx.shape[1]
    w = np.empty((T, k), np.float64)
    # Same two steps as the C routine: p = softmax(l), w_i = p_{e_i} / sum_j p_{e_j}.
    for t in range(T):
        l = logits[t]
        p = np.exp(l - l.max())
        p = p / p.sum()
        sel = p[idx[t]]
        w[t] = sel / sel.sum()
    return w


# ----------------------------------------------------------------------------
# FP8 (E4M3) expert weights with power-of-two block scales.
# ----------------------------------------------------------------------------
FP8_BLOCK = 32


def e4m3_value(code: int) -> float:
    """The number an FP8 E4M3 code stands for (OCP 8-bit floating point specification,
    E4M3 row): bit 7 sign, bits 6-3 exponent with bias 7, bits 2-0 mantissa; exponent
    field 0 is subnormal (m/8 * 2^-6); all-ones exponent and mantissa is NaN; there is no
    infinity."""
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def dequant_fp8(codes, scales) -> np.ndarray:
    """fp64 weights from codes [n, rows, K] (uint8) and scales [n, K/32, rows] (uint8):
    w[e, r, j] = e4m3(codes[e, r, j]) * 2^(scales[e, j // 32, r] - 127)."""
    c = _np(codes, np.uint8)
    sc = _np(scales, np.uint8)
    n, rows, K = c.shape
    assert K % FP8_BLOCK == 0 and sc.shape == (n, K // FP8_BLOCK, rows), (c.shape, sc.shape)
    mult = np.exp2(sc.astype(np.float64) - 127.0)           # [n, K/32, rows]
    mult = np.repeat(np.transpose(mult, (0, 2, 1)), FP8_BLOCK, axis=2)   # [n, rows, K]
    return E4M3_TABLE[c] * mult


def fp8_as_bf16(codes, scales) -> np.ndarray:
    """The dequantised weights as bf16 bit patterns (uint16), for the bf16 layer routines.
    Raises if any weight is not exactly a bf16 value."""
    w = dequant_fp8(codes, scales)
    if not np.all(np.isfinite(w)):
        raise ValueError("NaN code in FP8 weights")
    f32 = w.astype(np.float32)
    if not np.array_equal(f32.astype(np.float64), w):
        raise ValueError("FP8 weight not representable in fp32")
    bits = f32.view(np.uint32)
    if np.any(bits & 0xFFFF):
        raise ValueError("FP8 weight not representable in bf16")
    return (bits >> 16).astype(np.uint16)


def fp8_inputs(inp, routed, shared, experts: Optional[Sequence[int]] = None):
    """``inp`` with its expert weights replaced by the decoded FP8 sets (``workloads.Fp8Set``).

    With ``experts`` given, only those routed experts are decoded and returned as a
    mapping for ``forward(..., weights=...)``; otherwise a full copy of ``inp`` is
    returned."""
    def dec(c, s):
        return fp8_as_bf16(c, s)
    sh = {k: dec(getattr(shared, k), getattr(shared, k + "_scale"))
          for k in ("gate", "up", "down")}
    if experts is not None:
        m = {"W_gate": {}, "W_up": {}, "W_down": {}}
        for e in experts:
            for k in ("gate", "up", "down"):
                c = _np(getattr(routed, k)[e:e + 1], np.uint8)
                s = _np(getattr(routed, k + "_scale")[e:e + 1], np.uint8)
                m["W_" + k][int(e)] = dec(c, s)[0]
        m.update(Ws_gate=sh["gate"], Ws_up=sh["up"], Ws_down=sh["down"])
        return m
    import copy
    out = copy.copy(inp)
    out.W_gate = dec(routed.gate, routed.gate_scale)
    out.W_up = dec(routed.up, routed.up_scale)
    out.W_down = dec(routed.down, routed.down_scale)
    out.Ws_gate, out.Ws_up, out.Ws_down = sh["gate"], sh["up"], sh["down"]
    return out
