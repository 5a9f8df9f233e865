"""Benchmark of the B200 MoE FFN layer forward (tokens/s), one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode]
                    [--workloads all|none|name,name]
    python bench.py --impl reference ...      # the fp64 CPU oracle arm

A step is one moe_forward over one batch of T tokens: router, dispatch,
gather, gate/up GEMM + SwiGLU, down GEMM, combine.  The headline is the
decode workload (T = 16); every other configuration of the layer (batched
decode, prefill, skewed prefill, and the two FP8-weight decodes) is timed in
the same run the same way and reported under "workloads" in the same line.
With N GPUs (one process per GPU; `--gpus N` starts them through torchrun
when the script is not already running under it) every rank runs its own
replica of the layer on its own batch (the layer has no exchange between
token batches): "scaling": "weak", value = tokens of all ranks / the slowest
rank's time.

Timing: W untimed warm-up steps, then exactly K steps.  Before each step a
1 GB buffer (eight times L2) is written on the same stream, outside the timed
interval, so every step starts with a cold L2; each step is bracketed by CUDA
events on the launching stream; a barrier and synchronisation bracket the
timed loop; the per-rank total is max-reduced over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import ALL_WORKLOADS, Workload, make_fp8, make_ihc, make_inputs  # noqa: E402

DEFAULT_WORKLOAD = "decode"


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ----------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ----------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clocks_setting": 0x100,
    }

    def __init__(self, device: torch.device, period_s: float = 0.01):
        self.period = period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            p = torch.cuda.get_device_properties(device)
            try:   # NVML indices ignore CUDA_VISIBLE_DEVICES: find the GPU by its PCI address
                bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device.index or 0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - NVML missing
            self._nvml = None
            self.error = str(e)

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(self.period)

    def __enter__(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self) -> dict:
        if self._nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "NVML unavailable"}
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ----------------------------------------------------------------------------
# distributed plumbing (barrier, max over ranks); no collective on the data path
# ----------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, local, world


def init_dist(world: int, backend: str):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend=backend,
                                             timeout=datetime.timedelta(seconds=120))


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


def rank_batch(wl: Workload, rank: int) -> torch.Tensor:
    """The token batch of a replica rank > 0 (rank 0 uses the workload's own x): every rank
    holds the same weights and draws its own T tokens from seed + 1000 * rank."""
    g = torch.Generator().manual_seed(wl.seed + 1000 * rank)
    return torch.randn(wl.T, wl.d, generator=g).to(torch.bfloat16)


def max_over_ranks(value: float, world: int, device) -> float:
    if world == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int, device) -> float:
    if world == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


# ----------------------------------------------------------------------------
# algorithmic work of one forward (counts only touched expert weights, W_r, x, y)
# ----------------------------------------------------------------------------
def weight_bytes_per_element(wl: Workload) -> float:
    """bf16: 2 bytes; FP8: 1 byte of code plus 1/32 byte of block scale."""
    return 1.0 + 1.0 / 32 if wl.weights == "fp8" else 2.0


def algorithmic_work(wl: Workload, counts: np.ndarray) -> dict:
    touched = int((counts > 0).sum())
    bpe = weight_bytes_per_element(wl)
    per_expert_w = int(3 * wl.F * wl.d * bpe)
    w_bytes = (touched + wl.S) * per_expert_w
    rows = wl.T * wl.k + wl.S * wl.T
    gate_up_bytes = int((touched + wl.S) * 2 * wl.F * wl.d * bpe)
    down_bytes = int((touched + wl.S) * wl.F * wl.d * bpe)
    dense = wl.layer == "dense"     # no router: weights, x and y only
    act = wl.n_streams if wl.layer == "ihc" else 1   # iHC: n streams in and out
    return {
        "touched_experts": touched,
        "layer_bytes": w_bytes + (0 if dense else wl.E * wl.d * 4) + 2 * act * wl.T * wl.d * 2,
        "expert_flops": 6 * wl.d * wl.F * rows,
        "router_flops": 0 if dense else 2 * wl.T * wl.d * wl.E,
        "gate_up_bytes": gate_up_bytes,
        "gate_up_flops": 4 * wl.d * wl.F * rows,
        "down_bytes": down_bytes,
        "down_flops": 2 * wl.d * wl.F * rows,
    }


def fp8_form(T: int) -> str:
    """Which FP8 expert GEMM the library runs for a T-token batch: the warp-MMA form
    (expert_gemv_fp8.cu) up to 16 tokens unless MOE_GEMM_TILES picks a tiling, else the
    tcgen05 kernel (expert_gemm_fp8.cu)."""
    return "fp8_mma" if T <= 16 and not os.environ.get("MOE_GEMM_TILES") else "fp8"


def measured_traffic(kernel: str, bound: str, units: int, weights: str = "bf16",
                     d_model: int = 6144, d_ff: int = 2048, T: int = 16, layer: str = "moe"):
    """DRAM bytes per launch of ``kernel`` scaled from the committed ncu capture
    (profiles/traffic.json) by the touched experts, or None when there is none, when the
    experts' shape differs from the captured one (per-expert bytes do not carry over), or
    when the kernel source has changed since the counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    key = f"{kernel}/{bound}" + ("/" + fp8_form(T) if weights == "fp8" else "") + \
        ("/dense" if layer == "dense" else "")
    with open(path) as f:
        entry = json.load(f).get(key)
    if not entry or entry.get("bound") != bound:
        return None
    if entry.get("d_model", d_model) != d_model or entry.get("d_ff", d_ff) != d_ff:
        return None
    src = os.path.join(ROOT, "mixture_experts_layer_47_b200", "csrc",
                       entry.get("kernel_source", "expert_gemm.cu"))
    if not os.path.exists(src):
        return None
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != entry["kernel_source_sha256"]:
            return None
    return int(entry["bytes_per_touched_expert"] * units)


def hbm_bound(wl: Workload, work: dict, peaks: dict) -> bool:
    """Arithmetic intensity of the gate/up GEMM against the machine balance."""
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    return work["gate_up_flops"] / work["gate_up_bytes"] < ridge


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------
# Every workload of the layer's configurations is timed in one run: the headline
# (--workload, decode by default) and, in "workloads", the others.  Each is created,
# timed and freed before the next (19.4 GB of weights each).
EXTRA_WORKLOADS = ("batched_decode", "prefill", "skewed_prefill", "decode_fp8",
                   "batched_decode_fp8", "dense_decode", "dense_prefill", "decode_ihc")


def time_workload(wl: Workload, args, rank: int, world: int, device, cpu_seconds: float,
                  cpu_tokens: int) -> dict:
    """This rank's raw timings of one workload on its GPU (nothing reduced over ranks yet).

    Keys: step_ms (K device-timed steps), stage_ms (mean per stage of K evented steps),
    e2e_ms (K host-timed steps through moe_forward_host), counts (realised expert loads),
    clocks, kernels_per_step, h2d/d2h bytes per step, fp8, and on rank 0 of a one-GPU run
    cpu_baseline."""
    import mixture_experts_layer_47_b200 as moe

    inp = make_inputs(wl, device=device)
    if rank > 0:
        inp.x = rank_batch(wl, rank).to(device)
    h = moe.moe_create(wl.d, wl.E, wl.k, wl.F, wl.S)
    ws = torch.empty(moe.moe_workspace_size(h, wl.T), dtype=torch.uint8, device=device)
    y = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device=device)
    # 1 GB: eight times L2, and long enough (~0.2 ms) for the host to queue the whole
    # step behind it, so no launch latency falls inside the timed interval
    flush = torch.empty(1 << 30, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    fp8 = None
    if wl.weights == "fp8":
        fp8 = make_fp8(inp)   # the FP8 checkpoint of the same draws
        inp.W_gate = inp.W_up = inp.W_down = None   # the bf16 copies are not used
        inp.Ws_gate = inp.Ws_up = inp.Ws_down = None
        torch.cuda.empty_cache()
    weights = (inp.W_gate, inp.W_up, inp.W_down, inp.Ws_gate, inp.Ws_up, inp.Ws_down)
    dense = wl.layer == "dense"
    ihc = make_ihc(wl, device) if wl.layer == "ihc" else None
    x_stage = y_stage = None
    if ihc is not None:   # the activations are the residual streams H [T, n, d]
        inp.x = ihc[0]
        y = torch.empty_like(ihc[0])
        x_stage, y_stage = torch.empty_like(ihc[0]), torch.empty_like(ihc[0])

    def forward(x_arg, y_arg, host=False, lane=None):
        # lane: (stream, workspace, iHC staging buffers) of an end-to-end step
        st, w_s, stage = lane if lane is not None else (stream, ws, (x_stage, y_stage))
        if ihc is not None:   # the layer inside iHC streams; host streams copied around it
            H_in, H_out = stage if host else (x_arg, y_arg)
            with torch.cuda.stream(st):
                if host:
                    H_in.copy_(x_arg, non_blocking=True)
                moe.moe_forward_ihc(h, H_in, ihc[1], ihc[2], ihc[3], inp.W_router, inp.bias,
                                    *weights, H_out, w_s, st)
                if host:
                    y_arg.copy_(H_out, non_blocking=True)
        elif dense:   # the dense FFN layer
            f = moe.moe_dense_ffn_host if host else moe.moe_dense_ffn
            f(h, x_arg, inp.W_gate, inp.W_up, inp.W_down, y_arg, w_s, st)
        elif fp8 is not None:
            f = moe.moe_forward_fp8_host if host else moe.moe_forward_fp8
            f(h, x_arg, inp.W_router, inp.bias, fp8[0], fp8[1], y_arg, w_s, st)
        else:
            f = moe.moe_forward_host if host else moe.moe_forward
            f(h, x_arg, inp.W_router, inp.bias, *weights, y_arg, w_s, st)

    def step():
        forward(inp.x, y)

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize(device)
    st, detail = moe.moe_device_status(h, wl.T, ws, stream)
    if st != moe.MOE_OK:
        raise RuntimeError(f"{wl.name}: device status {st} ({detail:#x}) after warm-up")
    counts = (np.array([wl.T]) if dense else
              moe.workspace_views(h, wl.T, ws)["counts"].cpu().numpy())

    # ---- the timed steps (headline): events around each whole forward only ----
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(device)
    with ClockSampler(device) as clocks:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)      # cold L2 for every step, outside the timed interval
            starts[i].record(stream)
            step()
            ends[i].record(stream)
            ends[i].synchronize()
        torch.cuda.synchronize(device)
    barrier(world)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    st, detail = moe.moe_device_status(h, wl.T, ws, stream)
    if st != moe.MOE_OK:
        raise RuntimeError(f"{wl.name}: device status {st} ({detail:#x}) after the timed loop")

    # ---- stage times for the roofline: the same steps again with an event at every
    # stage boundary (the events serialise the kernels, so this loop is not the headline) ----
    stage_ev = [torch.cuda.Event(enable_timing=True) for _ in range(moe.MOE_STAGE_EVENTS)]
    for ev in stage_ev:
        ev.record(stream)
    moe.moe_set_stage_events(h, stage_ev)
    stage_ms = np.zeros((args.steps, moe.MOE_STAGE_EVENTS - 1))
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        step()
        stage_ev[-1].synchronize()
        for j in range(moe.MOE_STAGE_EVENTS - 1):
            stage_ms[i, j] = stage_ev[j].elapsed_time(stage_ev[j + 1])
    moe.moe_set_stage_events(h, None)

    # ---- end to end: every step copies its x in from pinned host memory and its y back
    # out, through the host-activation call.  The steps are enqueued back to back, as a
    # serving loop issues them, on two streams in turn, each with its own workspace and
    # host output buffer, so a step's output copy (on its own stream, after its layer)
    # overlaps the next step's layer, and its input copy the previous step's.  The whole
    # run is timed on the host clock, synchronised on both sides.  Every step streams GBs
    # of weights, far more than L2, so no flush separates them. ----
    x_host = inp.x.cpu().pin_memory()
    lanes = [(stream, ws, (x_stage, y_stage)),
             (torch.cuda.Stream(device), torch.empty_like(ws),
              (torch.empty_like(x_stage), torch.empty_like(y_stage)) if ihc is not None
              else (None, None))]
    y_hosts = [torch.empty(y.shape, dtype=torch.bfloat16).pin_memory() for _ in lanes]
    for i in range(max(2, args.warmup + (args.warmup & 1))):   # even: each lane keeps a slot
        forward(x_host, y_hosts[i & 1], host=True, lane=lanes[i & 1])
    torch.cuda.synchronize(device)
    barrier(world)
    t0 = time.perf_counter()
    for i in range(args.steps):
        forward(x_host, y_hosts[i & 1], host=True, lane=lanes[i & 1])
    torch.cuda.synchronize(device)
    e2e_ms = [(time.perf_counter() - t0) * 1e3 / args.steps] * args.steps
    barrier(world)
    del lanes

    raw = {"step_ms": step_ms, "stage_ms": stage_ms.mean(0).tolist(), "e2e_ms": e2e_ms,
           "counts": counts, "clocks": clocks.summary(),
           "kernels_per_step": (moe.moe_dense_ffn_kernel_count(h, wl.T) if dense
                                else moe.moe_forward_kernel_count(h, wl.T)
                                + (1 if ihc is not None else 0)),   # + the iHC mix
           "h2d_bytes": int(x_host.numel() * x_host.element_size()),
           "d2h_bytes": int(y_hosts[0].numel() * y_hosts[0].element_size()),
           "fp8": fp8 is not None}
    if rank == 0 and world == 1 and cpu_seconds > 0 and ihc is None:
        raw["cpu_baseline"] = cpu_baseline(inp, cpu_seconds, fp8, cpu_tokens)
    if hbm_bound(wl, algorithmic_work(wl, counts), load_peaks()):
        raw["read_only_gbs"] = read_only_peak(device)
    del inp, fp8, weights, ws, y, flush, x_host, y_hosts, x_stage, y_stage, ihc
    moe.moe_destroy(h)
    torch.cuda.synchronize(device)
    torch.cuda.empty_cache()
    return raw


def read_only_peak(device) -> float:
    """GB/s of a read-only stream on this GPU, measured live: a max-reduction over a 4 GiB
    int64 buffer (reads only, one value written; of the reductions tried on B200 the fastest
    reader), best of 5 with CUDA events.  The HBM-bound kernels here mostly read, so this is
    shown beside the copy peak (read + write) that MEASURED_PEAKS.json holds."""
    buf = torch.ones(1 << 29, dtype=torch.int64, device=device)
    best = 0.0
    for _ in range(6):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        buf.max()
        b.record()
        b.synchronize()
        best = max(best, buf.numel() * 8 / (a.elapsed_time(b) / 1e3) / 1e9)
    del buf
    torch.cuda.empty_cache()
    return round(best, 1)


def roofline(wl: Workload, work: dict, stage_mean: dict, peaks: dict) -> dict:
    """Roofline of the dominant kernel (the slower of the two expert GEMMs) from its live
    stage time: algorithmic bytes against the HBM peak below the machine balance,
    algorithmic FLOPs against the bf16 peak (burst and sustained) above it."""
    dominant = max(("gate_up_gemm", "down_gemm"), key=lambda n: stage_mean[n])
    dom_ms = stage_mean[dominant]
    key = "gate_up" if dominant == "gate_up_gemm" else "down"
    if hbm_bound(wl, work, peaks):
        achieved = work[key + "_bytes"] / (dom_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4)}
        if peaks.get("read_only_gbs"):
            roof["peak_read_only"] = peaks["read_only_gbs"]
            roof["frac_read_only"] = round(achieved / peaks["read_only_gbs"], 4)
    else:
        achieved = work[key + "_flops"] / (dom_ms / 1e3) / 1e12
        peak = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "peak_sustained": peaks["bf16_tflops_sustained"],
                "frac_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4)}
    traffic = measured_traffic(dominant, roof["bound"], work["touched_experts"] + wl.S,
                               wl.weights, wl.d, wl.F, wl.T, wl.layer)
    roof.update({"kernel": dominant, "traffic": traffic, "peak_source": peaks["source"],
                 "algorithmic_per_launch": work[key + ("_bytes" if roof["bound"] == "hbm"
                                                       else "_flops")],
                 "launch_ms": round(dom_ms, 4)})
    return roof


def workload_config(wl: Workload, world: int) -> dict:
    """The "config" of a bench line (the same for both arms)."""
    return {"workload": wl.name, "T": wl.T, "d_model": wl.d, "n_experts": wl.E,
            "top_k": wl.k, "d_ff": wl.F, "n_shared": wl.S, "router": wl.router,
            "zipf_s": wl.zipf_s, "weights": wl.weights, "layer": wl.layer,
            "global_batch": wl.T * world, "parallelism": f"replicas{world}",
            "l2": "flushed before every step (1 GB write, outside the timed interval)"}


def e2e_api(wl: Workload, fp8: bool) -> str:
    """The call the end-to-end number goes through."""
    if wl.layer == "dense":
        api = "moe_dense_ffn_host (pinned host x in, host y out)"
    elif wl.layer == "ihc":
        api = "moe_forward_ihc between pinned host copies of the streams"
    else:
        api = ("moe_forward_fp8_host" if fp8 else "moe_forward_host") + \
            " (pinned host x in, host y out)"
    return api + ("; steps enqueued back to back on two streams in turn, each with its own "
                  "workspace (a step's output copy overlaps the next step's layer)")


def report_workload(wl: Workload, raw: dict, args, world: int, device, stage_names) -> dict:
    """Reduce one workload's raw timings over ranks (the slowest rank sets every time) and
    derive tokens/s, the end-to-end number, the roofline and the layer's rates."""
    total_ms = max_over_ranks(sum(raw["step_ms"]), world, device)
    ms_per_step = total_ms / args.steps
    tokens_all = wl.T * world * args.steps
    stage_mean = {n: max_over_ranks(float(v), world, device)
                  for n, v in zip(stage_names, raw["stage_ms"])}
    e2e_total = max_over_ranks(sum(raw["e2e_ms"]), world, device)
    peaks = dict(load_peaks(), read_only_gbs=raw.get("read_only_gbs"))
    counts = raw["counts"]
    work = algorithmic_work(wl, counts)
    layer = {
        "tflops": round((work["expert_flops"] + work["router_flops"]) / (ms_per_step / 1e3)
                        / 1e12, 2),
        "gbs": round(work["layer_bytes"] / (ms_per_step / 1e3) / 1e9, 1),
        "touched_experts": work["touched_experts"],
        "hbm_frac": round(work["layer_bytes"] / (ms_per_step / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
        "tensor_frac": round(work["expert_flops"] / (ms_per_step / 1e3) / 1e12
                             / peaks["bf16_tflops"], 4),
        "stage_ms": {n: round(v, 4) for n, v in stage_mean.items()},
        "max_expert_rows": int(counts.max()), "min_expert_rows": int(counts.min()),
    }
    entry = {
        "value": round(tokens_all / (total_ms / 1e3), 1), "unit": "tokens/s",
        "ms_per_step": round(ms_per_step, 4),
        "config": workload_config(wl, world),
        "e2e": {"value": round(tokens_all / (e2e_total / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": raw["h2d_bytes"], "d2h_bytes_per_step": raw["d2h_bytes"],
                "api": e2e_api(wl, raw["fp8"]),
                "l2": "not flushed between the back-to-back steps (each streams GBs of "
                      "weights)"},
        "gpu_launches": raw["kernels_per_step"] * args.steps,
        "roofline": roofline(wl, work, stage_mean, peaks),
        "layer": layer,
        "clocks": raw["clocks"],
    }
    if raw["fp8"]:
        entry["weights"] = ("fp8: E4M3 codes, one power-of-two scale per 32 K elements of a "
                            "row, decoded to bf16 on the SMs; bf16 tensor-core MMAs")
    if "cpu_baseline" in raw:
        entry["cpu_baseline"] = raw["cpu_baseline"]
    return entry


def run_ours(args, rank, local, world, device=None, timer=time_workload, stage_names=None):
    """Time the headline workload and the extra ones on every rank; rank 0 prints the line.
    ``timer`` produces one rank's raw timings of one workload (the GPU work)."""
    if device is None:
        device = torch.device("cuda", local)
        torch.cuda.set_device(device)
    if stage_names is None:
        import mixture_experts_layer_47_b200 as moe
        stage_names = moe.STAGE_NAMES
    head_wl = ALL_WORKLOADS[args.workload]
    raw = timer(head_wl, args, rank, world, device, args.cpu_seconds, 16)
    head = report_workload(head_wl, raw, args, world, device, stage_names)
    extras = {}
    names = [] if args.workloads == "none" else \
        [n for n in (EXTRA_WORKLOADS if args.workloads == "all" else args.workloads.split(","))
         if n != args.workload]
    for name in names:
        wl = ALL_WORKLOADS[name]
        raw = timer(wl, args, rank, world, device, args.extra_cpu_seconds, 4)
        extras[name] = report_workload(wl, raw, args, world, device, stage_names)
    out = {
        "metric": "MoE-layer tokens/s", "value": head["value"], "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, random-init weights)",
        "config": head["config"], "e2e": head["e2e"], "gpu_launches": head["gpu_launches"],
        "roofline": head["roofline"], "layer": head["layer"], "clocks": head["clocks"],
    }
    for key in ("weights", "cpu_baseline"):
        if key in head:
            out[key] = head[key]
    if extras:
        out["workloads"] = extras
    if rank == 0:
        print(json.dumps(out), flush=True)
    return out


# ----------------------------------------------------------------------------
# the fp64 oracle on the host cores (CPU baseline and reference arm)
# ----------------------------------------------------------------------------
def _oracle_sample(inp, tokens: np.ndarray, fp8=None):
    """Host copies the oracle needs for these tokens: x, router, bias, used experts (for an
    FP8 checkpoint, those experts decoded by the oracle once, like loading a checkpoint)."""
    import oracle
    x = inp.x.cpu()
    Wr = inp.W_router.cpu()
    b = None if inp.bias is None else inp.bias.cpu()
    logits = oracle.router_logits(x[tokens], Wr, b)
    idx, _, _ = oracle.route(logits, inp.wl.k)
    used = sorted(set(idx.reshape(-1).tolist()))
    if fp8 is not None:
        return x[tokens].contiguous(), Wr, b, oracle.fp8_inputs(inp, fp8[0], fp8[1], used)
    W = {"W_gate": {e: inp.W_gate[e].cpu() for e in used},
         "W_up": {e: inp.W_up[e].cpu() for e in used},
         "W_down": {e: inp.W_down[e].cpu() for e in used},
         "Ws_gate": inp.Ws_gate.cpu(), "Ws_up": inp.Ws_up.cpu(), "Ws_down": inp.Ws_down.cpu()}
    return x[tokens].contiguous(), Wr, b, W


def _oracle_pass(x, Wr, b, W, wl) -> None:
    """One oracle forward of the sampled tokens: route, dispatch, experts, combine."""
    import oracle
    logits = oracle.router_logits(x, Wr, b)
    idx, w, _ = oracle.route(logits, wl.k)
    oracle.dispatch(idx, wl.E)
    oracle.moe_ffn_tokens(x, idx, w, W["W_gate"], W["W_up"], W["W_down"], W["Ws_gate"],
                          W["Ws_up"], W["Ws_down"], None, E=wl.E, F=wl.F, S=wl.S)


def _sample_tokens(wl: Workload, n: int = 16) -> np.ndarray:
    n = min(wl.T, n)
    return np.unique(np.linspace(0, wl.T - 1, n).round().astype(np.int64))


def cpu_baseline(inp, seconds: float, fp8=None, n_tokens: int = 16) -> dict:
    import oracle
    wl = inp.wl
    tokens = _sample_tokens(wl, n_tokens)
    x, Wr, b, W = _oracle_sample(inp, tokens, fp8)
    passes, t0 = 0, time.perf_counter()
    while True:
        _oracle_pass(x, Wr, b, W, wl)
        passes += 1
        el = time.perf_counter() - t0
        if el >= seconds or passes >= 1000:
            break
    return {"value": round(passes * len(tokens) / el, 3), "unit": "tokens/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{len(tokens)} of the {wl.T} tokens (evenly spaced) through the whole "
                      f"fp64 layer, {passes} passes in {el:.1f} s"}


def run_reference(args, rank, local, world):
    if rank != 0:
        return
    import oracle
    wl = ALL_WORKLOADS[args.workload]
    device = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    inp = make_inputs(wl, device=device)
    fp8 = make_fp8(inp) if wl.weights == "fp8" else None
    tokens = _sample_tokens(wl)
    x, Wr, b, W = _oracle_sample(inp, tokens, fp8)
    for _ in range(args.warmup):
        _oracle_pass(x, Wr, b, W, wl)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_pass(x, Wr, b, W, wl)
    el = time.perf_counter() - t0
    value = args.steps * len(tokens) / el
    sample = (f"each step: {len(tokens)} of the {wl.T} tokens (evenly spaced) through the "
              f"whole fp64 layer")
    out = {
        "impl": "reference", "metric": "MoE-layer tokens/s", "value": round(value, 3),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, random-init weights)",
        "config": workload_config(wl, world),
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s",
                         "cores": oracle.num_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


# ----------------------------------------------------------------------------
# sharded arm (--parallel tp|ep): one layer over N GPUs, the parts added by collective
# ----------------------------------------------------------------------------
def shard_plan(parallel: str, rank: int, world: int, E: int, F: int) -> dict:
    """What rank holds of the layer.  tp: rows [f0, f1) of every routed and shared expert's
    W_gate / W_up and the matching columns of W_down (F / world each); ep: routed experts
    [e0, e0 + n) (E / world each, full d_ff) and, on rank 0 only, the shared experts."""
    if parallel == "tp":
        if F % world or (F // world) % 64:
            raise ValueError(f"d_ff {F} does not split into {world} slices of a multiple of 64")
        w = F // world
        return {"e0": 0, "n": E, "f0": rank * w, "f1": (rank + 1) * w, "shared": True}
    if parallel == "ep":
        if E % world:
            raise ValueError(f"{E} experts do not split over {world} ranks")
        n = E // world
        return {"e0": rank * n, "n": n, "f0": 0, "f1": F, "shared": rank == 0}
    raise ValueError(parallel)


def shard_weights(inp, plan: dict) -> tuple:
    """This rank's contiguous copies (or views) of its expert weights."""
    e0, e1, f0, f1 = plan["e0"], plan["e0"] + plan["n"], plan["f0"], plan["f1"]

    def rows(W, a, b):
        return W[a:b, f0:f1, :].contiguous()

    def cols(W, a, b):
        return W[a:b, :, f0:f1].contiguous()
    routed = (rows(inp.W_gate, e0, e1), rows(inp.W_up, e0, e1), cols(inp.W_down, e0, e1))
    S = inp.Ws_gate.shape[0]
    shared = ((rows(inp.Ws_gate, 0, S), rows(inp.Ws_up, 0, S), cols(inp.Ws_down, 0, S))
              if plan["shared"] else (None, None, None))
    return routed, shared


def gather_parts(part: torch.Tensor, world: int) -> list:
    """Every rank's fp32 part, in rank order (one all-gather; none at world 1)."""
    if world == 1:
        return [part]
    n = part.shape[0]
    buf = torch.empty((world * n,) + tuple(part.shape[1:]), dtype=part.dtype, device=part.device)
    torch.distributed.all_gather_into_tensor(buf, part)
    return [buf[r * n:(r + 1) * n] for r in range(world)]


def run_sharded(args, rank, local, world):
    """One layer over the ranks: every rank routes all T tokens (x is the same on every
    rank), computes its shard's fp32 part (moe_forward_partial), the parts are all-gathered
    (NCCL) and every rank adds them in rank order (moe_reduce_partials): "scaling": "strong"
    (the same T tokens whatever the number of GPUs)."""
    import mixture_experts_layer_47_b200 as moe
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    wl = ALL_WORKLOADS[args.workload]
    if wl.weights != "bf16":
        raise SystemExit("--parallel tp|ep takes a bf16-weight workload")
    plan = shard_plan(args.parallel, rank, world, wl.E, wl.F)
    inp = make_inputs(wl, device=device)      # same seed, so the same x and router everywhere
    (Wg, Wu, Wd), (Sg, Su, Sd) = shard_weights(inp, plan)
    inp.W_gate = inp.W_up = inp.W_down = inp.Ws_gate = inp.Ws_up = inp.Ws_down = None
    torch.cuda.empty_cache()
    F_local = plan["f1"] - plan["f0"]
    h = moe.moe_create(wl.d, wl.E, wl.k, F_local, wl.S)
    ws = torch.empty(moe.moe_workspace_size(h, wl.T), dtype=torch.uint8, device=device)
    part = torch.empty(wl.T, wl.d, dtype=torch.float32, device=device)
    y = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device=device)
    flush = torch.empty(1 << 30, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step(x_in):
        moe.moe_forward_partial(h, x_in, inp.W_router, inp.bias, plan["e0"], Wg, Wu, Wd, Sg, Su,
                                Sd, part, ws, stream)
        moe.moe_reduce_partials(h, gather_parts(part, world), y, stream)

    for _ in range(args.warmup):
        flush.fill_(1)
        step(inp.x)
    torch.cuda.synchronize(device)
    st, detail = moe.moe_device_status(h, wl.T, ws, stream)
    if st != moe.MOE_OK:
        raise RuntimeError(f"device status {st} ({detail:#x}) after warm-up")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(device)
    with ClockSampler(device) as clocks:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            starts[i].record(stream)
            step(inp.x)
            ends[i].record(stream)
            ends[i].synchronize()
    barrier(world)
    total_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(starts, ends)), world,
                              device)
    # end to end: pinned host x in, y out, every step
    x_host = inp.x.cpu().pin_memory()
    y_host = torch.empty(wl.T, wl.d, dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(inp.x)
    barrier(world)
    e2e_ms = []
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        torch.cuda.synchronize(device)
        t0 = time.perf_counter()
        x_dev.copy_(x_host, non_blocking=True)
        step(x_dev)
        y_host.copy_(y, non_blocking=True)
        stream.synchronize()
        e2e_ms.append((time.perf_counter() - t0) * 1e3)
    barrier(world)
    e2e_total = max_over_ranks(sum(e2e_ms), world, device)
    ms = total_ms / args.steps
    out = {
        "metric": "MoE-layer tokens/s", "value": round(wl.T * args.steps / (total_ms / 1e3), 1),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, random-init weights)",
        "config": dict(workload_config(wl, 1), parallelism=f"{args.parallel}{world}"),
        "e2e": {"value": round(wl.T * args.steps / (e2e_total / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": wl.T * wl.d * 2, "d2h_bytes_per_step": wl.T * wl.d * 2,
                "api": "moe_forward_partial + all-gather + moe_reduce_partials"},
        "gpu_launches": (moe.moe_forward_kernel_count(h, wl.T) + 1) * args.steps,
        "shard": plan, "clocks": clocks.summary(),
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    return out


def _free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_command(n: int, argv, port: int) -> list:
    """The torchrun command that starts n ranks of this script with the same arguments."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={n}", "--master-addr=127.0.0.1", f"--master-port={port}",
            os.path.abspath(__file__), *argv]


def spawn_ranks(n: int, argv, visible: int) -> int:
    """--gpus N without a torchrun environment: start N ranks, one per visible GPU.
    Fails before starting anything when fewer than N GPUs are visible."""
    if visible < n:
        raise SystemExit(f"bench.py: --gpus {n} asked for, but {visible} CUDA device(s) are "
                         "visible")
    import subprocess
    # bounded: each rank's process group times out after 120 s; this is the last bound above
    cmd = ["timeout", "-k", "60", "3600", *launch_command(n, argv, _free_port())]
    return subprocess.run(cmd).returncode


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(ALL_WORKLOADS))
    ap.add_argument("--workloads", default="all",
                    help="extra workloads timed in the same run: 'all' (every configuration "
                         "of the layer), 'none', or a comma-separated list")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--extra-cpu-seconds", type=float, default=3.0)
    ap.add_argument("--parallel", default="replicas", choices=["replicas", "tp", "ep"],
                    help="replicas: every GPU runs the whole layer on its own tokens (weak "
                         "scaling); tp / ep: one layer over the GPUs, d_ff slices or expert "
                         "ranges per GPU, parts added after an all-gather (strong scaling)")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        ap.error("at least 3 warm-up steps are required")
    if args.workloads not in ("all", "none"):
        for n in args.workloads.split(","):
            if n not in ALL_WORKLOADS:
                ap.error(f"unknown workload {n}")
    if args.no_cpu_baseline:
        args.cpu_seconds = args.extra_cpu_seconds = 0.0
    return args


def main():
    args = parse_args()
    rank, local, world = dist_env()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        visible = torch.cuda.device_count() if torch.cuda.is_available() else 0
        sys.exit(spawn_ranks(args.gpus, sys.argv[1:], visible))
    if world > 1 and args.gpus not in (1, world):
        raise SystemExit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}")
    if args.impl == "reference":
        run_reference(args, rank, local, world)   # rank 0 only; no process group needed
        return
    init_dist(world, "nccl")
    try:
        if args.parallel == "replicas":
            run_ours(args, rank, local, world)
        else:
            run_sharded(args, rank, local, world)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
