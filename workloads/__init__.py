"""Seeded synthetic inputs for the Hy4-shaped MoE FFN layer.

This module is shared by the fp64 oracle's tests and by the CUDA path's tests
and benchmark.  It draws numbers and nothing else: it holds none of the layer's
arithmetic (no routing, no FFN, no combine).  The one derived input, the
per-expert router bias of the skewed workload, is read from a text table that
``tests/golden/make_zipf_bias.py`` writes with the oracle's router.

Shapes come from the Hy4-preview pages: hidden size 6144 (ZAKER release news,
"wider internal dimension" paragraph), 256 routed experts top-8 plus 1 shared
expert (same article, MoE paragraph; gpuvram.cloud "Tencent Hy4 preview" model
card).  The expert width d_ff = 2048 is not printed on any page; it is the
stated assumption of this layer (770B total / 49B active is consistent with it).

Draw order (CPU ``torch.Generator`` seeded with ``seed``): x, W_router, bias,
then the expert weights shared W_gate, W_up, W_down and routed W_gate, W_up,
W_down.  Expert weights of the Hy4-sized workloads (about 19.4 GB of bf16) are
drawn on the target device with a generator of that device seeded with
``seed``, in the same order, expert by expert; the tiny workload draws
everything on the CPU so that CPU-only and GPU tests see identical values.
"""
from __future__ import annotations

import math
import os
from dataclasses import dataclass, field, replace
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_REPO = os.path.dirname(_HERE)
ZIPF_BIAS_DIR = os.path.join(_REPO, "tests", "golden")


@dataclass(frozen=True)
class Workload:
    """One layer configuration and its input recipe."""

    name: str
    T: int            # tokens
    d: int            # d_model
    E: int            # routed experts
    k: int            # top-k
    F: int            # expert d_ff
    S: int            # shared experts (always on, weight 1)
    router: str = "normal"        # "normal": N(0, 1/sqrt(d)); "uniform": U(-1/sqrt(d), 1/sqrt(d))
    zipf_s: Optional[float] = None  # per-expert bias making expert popularity ~ Zipf(s)
    seed: int = 0
    description: str = ""
    weights: str = "bf16"           # "bf16", or "fp8": the same draws stored as e4m3 + block scales
    layer: str = "moe"              # "moe"; "dense": the dense FFN layer (E = 1, k = 1, S = 0);
                                    # "ihc": the MoE layer inside n_streams residual streams
    n_streams: int = 0              # iHC streams (the pages' model: 4)

    @property
    def slots(self) -> int:
        return self.T * self.k

    @property
    def rows(self) -> int:
        """Rows the expert FFN processes: T*k routed slots plus S*T shared rows."""
        return self.T * self.k + self.S * self.T

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload(
        "tiny", T=64, d=256, E=16, k=2, F=128, S=1, router="normal", seed=0,
        description="Tiny MoE layer: T=64, d_model=256, 16 routed experts top-2 + 1 shared, "
                    "SwiGLU d_ff=128; x ~N(0,1), expert W ~N(0,1/sqrt(fan_in)), router ~N(0,1/sqrt(d))"),
    "decode": Workload(
        "decode", T=16, d=6144, E=256, k=8, F=2048, S=1, router="normal", seed=0,
        description="Hy4-shaped decode: T=16, d_model=6144, 256 experts top-8 + 1 shared, d_ff=2048"),
    "batched_decode": Workload(
        "batched_decode", T=256, d=6144, E=256, k=8, F=2048, S=1, router="uniform", seed=0,
        description="Hy4-shaped batched decode: T=256, uniform router init (balanced load)"),
    "prefill": Workload(
        "prefill", T=8192, d=6144, E=256, k=8, F=2048, S=1, router="uniform", seed=0,
        description="Hy4-shaped prefill: T=8192, uniform router init (balanced load)"),
    "skewed_prefill": Workload(
        "skewed_prefill", T=8192, d=6144, E=256, k=8, F=2048, S=1, router="uniform",
        zipf_s=1.2, seed=0,
        description="Skewed-load prefill: T=8192, router logits plus a per-expert bias "
                    "calibrated so expert popularity follows Zipf s=1.2"),
    "decode_fp8": Workload(
        "decode_fp8", T=16, d=6144, E=256, k=8, F=2048, S=1, router="normal", seed=0,
        weights="fp8",
        description="the decode workload with its expert weights stored as FP8 (e4m3 codes, one "
                    "power-of-two scale per 32 K elements of a row)"),
    "batched_decode_fp8": Workload(
        "batched_decode_fp8", T=256, d=6144, E=256, k=8, F=2048, S=1, router="uniform", seed=0,
        weights="fp8",
        description="the batched decode workload with FP8 expert weights"),
    # The MoE layer inside the iHC wrapper's four residual streams (ZAKER release news, iHC
    # paragraphs); streams H ~ N(0, 1), alpha ~ U(0.1, 0.5), B ~ N(0, 0.1^2), gamma ~ U(0.5, 1.5)
    # drawn after the layer's inputs (make_ihc).
    "decode_ihc": Workload(
        "decode_ihc", T=16, d=6144, E=256, k=8, F=2048, S=1, router="normal", seed=0,
        layer="ihc", n_streams=4,
        description="the decode workload inside four iHC residual streams"),
    # The model's first layer is a standard dense FFN (ZAKER release news, architecture
    # paragraph); its width is not printed.  Reading: SwiGLU of width (8 + 1) * 2048 = 18432,
    # the FFN width one token passes through in an MoE layer (8 routed + 1 shared experts).
    "dense_decode": Workload(
        "dense_decode", T=16, d=6144, E=1, k=1, F=18432, S=0, router="normal", seed=0,
        layer="dense",
        description="the dense first layer at decode: T=16, d_model=6144, SwiGLU d_ff=18432"),
    "dense_prefill": Workload(
        "dense_prefill", T=8192, d=6144, E=1, k=1, F=18432, S=0, router="normal", seed=0,
        layer="dense",
        description="the dense first layer at prefill: T=8192, d_model=6144, SwiGLU d_ff=18432"),
}

# Reduced cases of the same kernels for profiler captures that must stay a few GB on the
# device: the Hy4 hidden and expert widths with 32 routed experts (2.4 GB of weights).
PROFILE_WORKLOADS = {
    "profile_decode_e32": Workload(
        "profile_decode_e32", T=16, d=6144, E=32, k=8, F=2048, S=1, router="normal", seed=0,
        description="decode-shaped profiling case: T=16, d=6144, 32 experts top-8 + 1 shared"),
    "profile_prefill_e32": Workload(
        "profile_prefill_e32", T=1024, d=6144, E=32, k=8, F=2048, S=1, router="uniform", seed=0,
        description="prefill-shaped profiling case: T=1024 (256 rows per expert), d=6144, "
                    "32 experts top-8 + 1 shared"),
    "profile_router_prefill": Workload(
        "profile_router_prefill", T=8192, d=6144, E=256, k=8, F=64, S=1, router="uniform",
        seed=0,
        description="the prefill router at full size (T=8192, d=6144, 256 experts top-8) with "
                    "64-wide experts, so the case holds about 1 GB on the device"),
    "profile_decode_fp8_e32": Workload(
        "profile_decode_fp8_e32", T=16, d=6144, E=32, k=8, F=2048, S=1, router="normal", seed=0,
        weights="fp8",
        description="decode-shaped profiling case with FP8 expert weights (1.2 GB of codes)"),
}
ALL_WORKLOADS = {**WORKLOADS, **PROFILE_WORKLOADS}


def zipf_bias_path(wl: Workload) -> str:
    return os.path.join(
        ZIPF_BIAS_DIR,
        f"zipf_bias_E{wl.E}_k{wl.k}_d{wl.d}_T{wl.T}_s{wl.zipf_s}_seed{wl.seed}.txt")


def load_zipf_bias(wl: Workload) -> torch.Tensor:
    """Read the calibrated per-expert bias table (one float per line, '#' comments)."""
    path = zipf_bias_path(wl)
    vals = []
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                vals.append(float(line))
    if len(vals) != wl.E:
        raise ValueError(f"{path}: expected {wl.E} values, found {len(vals)}")
    return torch.tensor(vals, dtype=torch.float32)


def zipf_targets(E: int, s: float, perm: torch.Tensor) -> torch.Tensor:
    """Target popularity share q_e proportional to (perm[e]+1)^-s (sums to 1)."""
    ranks = perm.to(torch.float64) + 1.0
    q = ranks.pow(-s)
    return q / q.sum()


def zipf_permutation(wl: Workload) -> torch.Tensor:
    """Seeded permutation that assigns popularity ranks to experts."""
    g = torch.Generator().manual_seed(wl.seed + 7919)
    return torch.randperm(wl.E, generator=g)


@dataclass
class Inputs:
    wl: Workload
    x: torch.Tensor            # [T, d] bf16
    W_router: torch.Tensor     # [E, d] fp32
    bias: Optional[torch.Tensor]  # [E] fp32 or None
    W_gate: torch.Tensor       # [E, F, d] bf16
    W_up: torch.Tensor         # [E, F, d] bf16
    W_down: torch.Tensor       # [E, d, F] bf16
    Ws_gate: torch.Tensor      # [S, F, d] bf16
    Ws_up: torch.Tensor        # [S, F, d] bf16
    Ws_down: torch.Tensor      # [S, d, F] bf16
    extra: dict = field(default_factory=dict)


def make_x(wl: Workload, gen: torch.Generator, T: Optional[int] = None) -> torch.Tensor:
    T = wl.T if T is None else T
    return torch.randn(T, wl.d, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def make_router(wl: Workload, gen: torch.Generator) -> torch.Tensor:
    bound = 1.0 / math.sqrt(wl.d)
    if wl.router == "normal":
        return torch.randn(wl.E, wl.d, generator=gen, dtype=torch.float32) * bound
    if wl.router == "uniform":
        return (torch.rand(wl.E, wl.d, generator=gen, dtype=torch.float32) * 2.0 - 1.0) * bound
    raise ValueError(f"unknown router init {wl.router!r}")


def _fill_normal_bf16(out: torch.Tensor, std: float, gen: torch.Generator, chunk_rows: int) -> None:
    """Fill a [n, r, c] bf16 tensor with N(0, std^2) values, chunk_rows leading rows at a time."""
    n = out.shape[0]
    for i in range(0, n, chunk_rows):
        j = min(n, i + chunk_rows)
        tmp = torch.randn((j - i,) + tuple(out.shape[1:]), generator=gen,
                          dtype=torch.float32, device=out.device)
        out[i:j].copy_((tmp * std).to(torch.bfloat16))
        del tmp


def make_inputs(wl: Workload, device: str | torch.device = "cpu",
                weights_on: Optional[str | torch.device] = None) -> Inputs:
    """Draw every input of ``wl``.

    x, W_router and bias are drawn on the CPU and moved to ``device``.  Expert
    weights are drawn on ``weights_on`` (default: the CPU for the tiny
    workload, ``device`` otherwise) so that 19.4 GB of weights never pass
    through host memory.
    """
    device = torch.device(device)
    gen = torch.Generator().manual_seed(wl.seed)
    x = make_x(wl, gen)
    W_router = make_router(wl, gen)
    bias = load_zipf_bias(wl) if wl.zipf_s is not None else None

    n_weights = 3 * (wl.E + wl.S) * wl.F * wl.d
    if weights_on is None:
        weights_on = "cpu" if n_weights <= (1 << 26) else device
    wdev = torch.device(weights_on)
    if wdev.type == "cpu":
        wgen = gen
    else:
        wgen = torch.Generator(device=wdev).manual_seed(wl.seed)

    def empty(*shape):
        return torch.empty(*shape, dtype=torch.bfloat16, device=wdev)

    std_in = 1.0 / math.sqrt(wl.d)
    std_dn = 1.0 / math.sqrt(wl.F)
    Ws_gate, Ws_up, Ws_down = empty(wl.S, wl.F, wl.d), empty(wl.S, wl.F, wl.d), empty(wl.S, wl.d, wl.F)
    W_gate, W_up, W_down = empty(wl.E, wl.F, wl.d), empty(wl.E, wl.F, wl.d), empty(wl.E, wl.d, wl.F)
    chunk = max(1, (1 << 26) // (wl.F * wl.d))  # about 64M elements (256 MB fp32) per draw
    _fill_normal_bf16(Ws_gate, std_in, wgen, chunk)
    _fill_normal_bf16(Ws_up, std_in, wgen, chunk)
    _fill_normal_bf16(Ws_down, std_dn, wgen, chunk)
    _fill_normal_bf16(W_gate, std_in, wgen, chunk)
    _fill_normal_bf16(W_up, std_in, wgen, chunk)
    _fill_normal_bf16(W_down, std_dn, wgen, chunk)

    def mv(t):
        return None if t is None else t.to(device)

    return Inputs(wl, mv(x), mv(W_router), mv(bias),
                  mv(W_gate), mv(W_up), mv(W_down), mv(Ws_gate), mv(Ws_up), mv(Ws_down))


def make_small(T: int, d: int, E: int, k: int, F: int, S: int, seed: int = 0,
               router: str = "normal", device="cpu", bias_scale: float = 0.0) -> Inputs:
    """Arbitrary small shapes for parity sweeps (all drawn on the CPU).

    ``bias_scale`` > 0 adds a N(0, bias_scale^2) per-expert router bias drawn
    after W_router.
    """
    wl = Workload(f"small_T{T}_d{d}_E{E}_k{k}_F{F}_S{S}_seed{seed}", T=T, d=d, E=E, k=k,
                  F=F, S=S, router=router, seed=seed)
    gen = torch.Generator().manual_seed(seed)
    x = make_x(wl, gen)
    W_router = make_router(wl, gen)
    bias = None
    if bias_scale > 0:
        bias = torch.randn(E, generator=gen, dtype=torch.float32) * bias_scale
    std_in, std_dn = 1.0 / math.sqrt(d), 1.0 / math.sqrt(F)

    def nrm(shape, std):
        return (torch.randn(*shape, generator=gen, dtype=torch.float32) * std).to(torch.bfloat16)

    Ws_gate, Ws_up, Ws_down = nrm((S, F, d), std_in), nrm((S, F, d), std_in), nrm((S, d, F), std_dn)
    W_gate, W_up, W_down = nrm((E, F, d), std_in), nrm((E, F, d), std_in), nrm((E, d, F), std_dn)
    inp = Inputs(wl, x, W_router, bias, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down)
    if torch.device(device).type != "cpu":
        inp = to_device(inp, device)
    return inp


def to_device(inp: Inputs, device) -> Inputs:
    def mv(t):
        return None if t is None else t.to(device)
    return Inputs(inp.wl, mv(inp.x), mv(inp.W_router), mv(inp.bias), mv(inp.W_gate),
                  mv(inp.W_up), mv(inp.W_down), mv(inp.Ws_gate), mv(inp.Ws_up),
                  mv(inp.Ws_down), dict(inp.extra))


# ----------------------------------------------------------------------------
# FP8 expert weights (an input format, not part of the layer's arithmetic).
#
# The Hy4 pages mention an official FP8 checkpoint but print no scaling scheme;
# this layer's stated choice is the OCP microscaling layout: every weight is an
# FP8 E4M3 code (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no
# infinities, S.1111.111 = NaN, largest finite 448), and each run of 32
# consecutive K elements of a weight row shares one power-of-two scale stored
# as a biased exponent byte (value 2^(byte - 127)).  Scales are stored
# K-block-major, scale[n][K/32][rows], so the scales of 128 consecutive rows
# for one K block are contiguous.  The FP8 checkpoint of a workload is made
# from the same seeded bf16 draws: per block the smallest power of two 2^e with
# max|w| / 2^e <= 448, codes = e4m3(w / 2^e) rounded to nearest even.
# ----------------------------------------------------------------------------
FP8_BLOCK = 32
FP8_E4M3_MAX = 448.0


@dataclass
class Fp8Set:
    """FP8 weights of one set of experts (routed or shared)."""
    gate: torch.Tensor         # [n, F, d] uint8 e4m3 codes
    gate_scale: torch.Tensor   # [n, d/32, F] uint8 biased exponents
    up: torch.Tensor           # [n, F, d]
    up_scale: torch.Tensor     # [n, d/32, F]
    down: torch.Tensor         # [n, d, F]
    down_scale: torch.Tensor   # [n, F/32, d]

    def to(self, device) -> "Fp8Set":
        return Fp8Set(*(t.to(device) for t in (self.gate, self.gate_scale, self.up,
                                               self.up_scale, self.down, self.down_scale)))


def quantize_fp8(W: torch.Tensor, chunk: int = 8) -> tuple:
    """[n, rows, K] weights -> (codes [n, rows, K] uint8, scales [n, K/32, rows] uint8).

    Works on W's device, ``chunk`` leading slices at a time."""
    n, rows, K = W.shape
    if K % FP8_BLOCK:
        raise ValueError("K must be a multiple of 32")
    codes = torch.empty((n, rows, K), dtype=torch.uint8, device=W.device)
    scales = torch.empty((n, K // FP8_BLOCK, rows), dtype=torch.uint8, device=W.device)
    for i in range(0, n, chunk):
        j = min(n, i + chunk)
        w = W[i:j].to(torch.float32).reshape(j - i, rows, K // FP8_BLOCK, FP8_BLOCK)
        amax = w.abs().amax(dim=-1)
        e = torch.ceil(torch.log2(amax / FP8_E4M3_MAX))
        e = torch.where(amax > 0, e, torch.full_like(e, -127.0)).clamp(-127.0, 127.0)
        q = (w / torch.exp2(e).unsqueeze(-1)).to(torch.float8_e4m3fn)
        codes[i:j] = q.view(torch.uint8).reshape(j - i, rows, K)
        scales[i:j] = (e + 127.0).to(torch.uint8).transpose(1, 2)
        del w, amax, e, q
    return codes, scales


def make_fp8(inp: Inputs) -> tuple:
    """(routed, shared) FP8 sets made from the bf16 expert weights of ``inp``."""
    def one(Wg, Wu, Wd):
        g, gs = quantize_fp8(Wg)
        u, us = quantize_fp8(Wu)
        dn, ds = quantize_fp8(Wd)
        return Fp8Set(g, gs, u, us, dn, ds)
    return one(inp.W_gate, inp.W_up, inp.W_down), one(inp.Ws_gate, inp.Ws_up, inp.Ws_down)


def make_ihc(wl: Workload, device="cpu") -> tuple:
    """(H [T, n, d] bf16, alpha [n], B [n, n], gamma [n] fp32) for an iHC workload, drawn with
    a CPU generator seeded with seed + 17: H ~ N(0, 1), alpha ~ U(0.1, 0.5),
    B ~ N(0, 0.1^2), gamma ~ U(0.5, 1.5)."""
    n = wl.n_streams
    g = torch.Generator().manual_seed(wl.seed + 17)
    H = torch.randn(wl.T, n, wl.d, generator=g).to(torch.bfloat16)
    alpha = (0.1 + 0.4 * torch.rand(n, generator=g)).float()
    B = (0.1 * torch.randn(n, n, generator=g)).float()
    gamma = (0.5 + torch.rand(n, generator=g)).float()
    return tuple(t.to(device) for t in (H, alpha, B, gamma))
