"""Benchmark of the B200 BitLinear forward (W1.58A8) -- one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--workload decode|prefill|sweep|chain] [--impl ours|reference]

Metric: decode GEMV weight GB/s (packed 2-bit weight bytes streamed per
second) and prefill GEMM int8 TOPS (2*M*N*K per second), each against the
B200 roofline.  The default run measures both: the decode GEMV is the line's
own value, and the prefill GEMM (M=4096, K=2560, N=6912) its "prefill"
object, each with its roofline, CPU oracle baseline, end-to-end figure and
clocks.

Every timed region is one replay of a CUDA graph holding one untimed step
and then the K timed steps, with CUDA events recorded inside the graph around
the timed ones: the start event on a side branch after the untimed step, so
the first timed step overlaps its predecessor (programmatic dependent launch)
like every later one, and the events bracket K steps of the steady state,
free of the graph's start-up and the host's launch latency (the same per-step
time for --steps 20 as for --steps 2000).  A spin kernel ahead of the replay
keeps the GPU busy while the host submits the graph.

A step is one pass of the BitLinear forward over one batch of synthetic,
seeded input: per-token activation quantisation, the ternary x int8
contraction with int32 accumulation, the gamma/s rescale and the bf16 store.
The default workload is the decode GEMV (M = 1 token, K = N = 2560, bf16 in
and out); each step uses the next of R copies of the packed weights, R sized
so the copies span more than 3x the L2 cache, so no step reads its weights
from a warm L2.  The timed steps run back to back from a CUDA graph (the
launches use programmatic dependent launch, so a step may stream its weights
while the previous step finishes; its activations are read only after the
previous step has completed).

With --gpus N (one process per GPU, launched by torch.distributed.run) every
rank runs the same workload on its own GPU: replicas with no data-path
collective (weak scaling); the time is the max over ranks.

--impl reference times the CPU oracle (plain C) on the host cores on a
bounded sample of the same workload (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W1.58A8 decode GEMV weight GB/s & prefill GEMM int8 TOPS, % of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_PER_BF16 = 2.0  # nominal dense int8 / bf16 tensor throughput ratio on B200 (4.5 / 2.25 PF)


# ------------------------------------------------------------------ helpers
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_hash(*files) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(key: str, files) -> int | None:
    """DRAM bytes per launch of a kernel from the committed ncu summary, or
    None if there is none or the kernel source changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        table = json.load(f)
    ent = table.get(key)
    if not ent or ent.get("source_hash") != source_hash(*files):
        return None
    return int(ent["dram_bytes_per_launch"])


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle", 0x10: "sync_boost"}

    def __init__(self, index):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            try:
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(index)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.nv = None

    def _sample(self):
        nv = self.nv
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
            fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            self.reasons |= int(fn(self.h))
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self._sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()
            self._sample()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def max_over_ranks(x: float, dist, device) -> float:
    """Max of a per-rank number over all ranks (every rank calls it)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world: int, units_per_step: float, steps: int, seconds: float,
                    scale: float) -> float:
    """Whole-job throughput: every rank processes the same per-step work
    (replicas), timed as the slowest rank."""
    return world * units_per_step * steps / seconds * scale


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ------------------------------------------------------------------ workloads
class Workload:
    """Common shape of a benchmarked workload."""
    name = ""
    unit = "GB/s"
    bound = "hbm"


def workload_identity(workload: str, sweep_m: int = 8, layers: int = 30) -> dict:
    """What a workload is (shapes, distributions, dtypes), shared by both arms' JSON lines."""
    if workload == "decode":
        return {"workload": "decode GEMV M=1 K=2560 N=2560, bf16 activations N(0,1) with 0.1% "
                            "x20 outliers, absmean ternary weights from N(0,0.02), bf16 out",
                "M": 1, "K": 2560, "N": 2560, "x_dtype": "bf16", "y_dtype": "bf16"}
    if workload == "sweep":
        return {"workload": f"decode sweep M={sweep_m}: one decoder layer's BitLinears, qkv "
                            "2560->3840, o 2560->2560, up 2560->6912 + ReLU^2, down 6912->2560; "
                            "Student-t(3) bf16 activations, absmean ternary weights from "
                            "N(0,0.02), bf16 out",
                "M": sweep_m, "x_dtype": "bf16", "y_dtype": "bf16"}
    if workload == "prefill":
        return {"workload": "prefill GEMM M=4096 K=2560 N=6912, bf16 activations N(0,1) "
                            "per-token absmax int8, ternary weights from N(0,0.02), int32 "
                            "accumulation, bf16 out",
                "M": 4096, "K": 2560, "N": 6912, "x_dtype": "bf16", "y_dtype": "bf16"}
    if workload == "chain":
        return {"workload": f"{layers}-layer decode chain, M=1, per layer qkv 2560->3840, "
                            "o 2560->2560, up 2560->6912 + ReLU^2, down 6912->2560, rms norm",
                "M": 1, "layers": layers, "x_dtype": "bf16", "y_dtype": "bf16"}
    raise ValueError(workload)


def make_decode(tw, torch, dev, l2_bytes, table_lookup=False):
    import synth
    d = synth.config_inputs("decode")
    W = torch.from_numpy(d["W"]).to(dev)
    packed, gamma = tw.bitnet_quantize_weights(W)
    del W
    wbytes = packed.numel()
    R = max(4, -(-3 * l2_bytes // wbytes))
    copies = torch.empty((R,) + tuple(packed.shape), dtype=torch.uint8, device=dev)
    copies[:] = packed
    views = list(copies)  # one tensor per copy, made once (not a new view every call)
    X = torch.from_numpy(d["x_bits"].view(np.int16)).to(dev).view(torch.bfloat16)
    Y = torch.empty((1, d["N"]), dtype=torch.bfloat16, device=dev)

    def step(i, stream=None):
        tw.bitnet_w158a8_matmul(X, copies[i % R], gamma, Y=Y, weights_static=True,
                                table_lookup=table_lookup, stream=stream)

    return dict(
        step=step, kernel_step=step, units_per_step=wbytes, unit="GB/s", scale=1e-9, bound="hbm",
        launches_per_step=1, X=X, Y=Y, rotate=R, extra=dict(packed=copies, gamma=gamma),
        config={**workload_identity("decode"),
                "l2": f"inputs larger than L2: {R} rotating weight copies, "
                      f"{R * wbytes / 1e6:.0f} MB >= 3x L2",
                "timing": "CUDA graph of the timed steps, programmatic dependent launch, "
                          "weights flagged static",
                **({"kernel": "table-lookup comparison kernel"} if table_lookup else {})},
        kernel_key=None if table_lookup else "decode_gemv_M1_K2560_N2560",
        kernel_files=["ternary_weight_linear_token_b200/csrc/gemv_rows.cu",
                      "ternary_weight_linear_token_b200/csrc/common.cuh"],
        e2e_inputs=lambda: (d["x_bits"].view(np.int16), 2 * d["K"], 2 * d["N"]),
        # end to end: one host-to-host call per step, through a plan per weight copy
        # (the table-lookup comparison goes through the device entry point, the host
        # one takes no flags)
        e2e_plans=None if table_lookup else (
            lambda xh, yh, stream=None: [tw.HostMatmulPlan(xh, v, gamma, X, Y, yh,
                                                           weights_static=True, stream=stream)
                                         for v in views]),
    )


def make_sweep(tw, torch, dev, l2_bytes, M=8, table_lookup=False):
    """Decode sweep: one step is one decoder layer's four projections (qkv,
    o, up + ReLU^2, down) at M tokens, each a dependent call."""
    import synth
    projs = []
    for p in range(4):
        d = synth.config_inputs("sweep", M=M, proj=p)
        packed, gamma = tw.bitnet_quantize_weights(torch.from_numpy(d["W"]).to(dev))
        X = torch.from_numpy(d["x_bits"].view(np.int16)).to(dev).view(torch.bfloat16)
        Y = torch.empty((M, d["N"]), dtype=torch.bfloat16, device=dev)
        need = tw.bitnet_w158a8_matmul_workspace_size(M, d["N"], d["K"], torch.bfloat16)
        ws = torch.empty(max(1, need), dtype=torch.uint8, device=dev)
        projs.append(dict(packed=packed, gamma=gamma, X=X, Y=Y, ws=ws, relu2=d["relu2"], d=d))
    wbytes = sum(q["packed"].numel() for q in projs)
    R = max(4, -(-3 * l2_bytes // wbytes))
    for q in projs:  # rotating copies: every step streams its weights from HBM
        q["copies"] = torch.empty((R,) + tuple(q["packed"].shape), dtype=torch.uint8, device=dev)
        q["copies"][:] = q["packed"]

    def step(i, stream=None):
        for q in projs:
            tw.bitnet_w158a8_matmul(q["X"], q["copies"][i % R], q["gamma"], relu2=q["relu2"],
                                    Y=q["Y"], workspace=q["ws"], weights_static=True,
                                    table_lookup=table_lookup, stream=stream)

    d0 = projs[0]["d"]
    # 4 tokens and more: quantiser + product per projection (the table-lookup
    # kernel quantises inside, like the fused one)
    launches = 4 if (M <= 3 or table_lookup) else 8
    return dict(
        step=step, kernel_step=step, units_per_step=wbytes, unit="GB/s", scale=1e-9, bound="hbm",
        launches_per_step=launches, X=projs[0]["X"], Y=projs[3]["Y"], rotate=R,
        config={**workload_identity("sweep", sweep_m=M),
                "l2": f"inputs larger than L2: {R} rotating copies of the layer's weights, "
                      f"{R * wbytes / 1e6:.0f} MB >= 3x L2",
                "timing": "CUDA graph of the timed steps, programmatic dependent launch, "
                          "weights flagged static",
                **({"kernel": "table-lookup comparison kernel"} if table_lookup else {})},
        kernel_key=None, kernel_files=[],
        e2e_inputs=lambda: (d0["x_bits"].view(np.int16), 2 * M * d0["K"], 2 * M * 2560),
    )


def make_prefill(tw, torch, dev, l2_bytes, prep_in_kernel=False):
    import synth
    d = synth.config_inputs("prefill")
    M, N, K = d["M"], d["N"], d["K"]
    W = torch.from_numpy(d["W"]).to(dev)
    packed, gamma = tw.bitnet_quantize_weights(W)
    del W
    X0 = torch.from_numpy(d["x_bits"].view(np.int16)).to(dev).view(torch.bfloat16)
    per_set = X0.numel() * 2 + packed.numel() + M * N * 2
    R = max(2, -(-3 * l2_bytes // per_set))
    Xs = [X0] + [X0.clone() for _ in range(R - 1)]
    Ps = [packed] + [packed.clone() for _ in range(R - 1)]
    Ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(R)]
    need = tw.bitnet_w158a8_matmul_workspace_size(M, N, K, torch.bfloat16)
    wss = [torch.empty(need, dtype=torch.uint8, device=dev) for _ in range(R)]
    xq = [ws[: M * K].view(torch.int8).view(M, K) for ws in wss]
    sc = [ws[((M * K + 255) // 256) * 256:][: 4 * M].view(torch.float32) for ws in wss]

    def step(i, stream=None):
        j = i % R
        tw.bitnet_w158a8_matmul(Xs[j], Ps[j], gamma, Y=Ys[j], workspace=wss[j],
                                weights_static=True, prep_in_kernel=prep_in_kernel,
                                stream=stream)

    # The tensor-core kernel alone: int8 activations (natural K order) with
    # their scales, and per set a workspace whose int8 weight copy a first,
    # untimed call wrote; the timed calls promise that copy
    # (weights_expanded), so each is exactly one tcgen05 kernel launch.
    qx = [torch.empty((M, K), dtype=torch.int8, device=dev) for _ in range(R)]
    qs = [torch.empty(M, dtype=torch.float32, device=dev) for _ in range(R)]
    need8 = tw.bitnet_w158a8_matmul_workspace_size(M, N, K, torch.int8)
    ws8 = [torch.empty(need8, dtype=torch.uint8, device=dev) for _ in range(R)]
    for j in range(R):
        tw.bitnet_quantize_act(Xs[j], xq=qx[j], s=qs[j])
        tw.bitnet_w158a8_matmul(qx[j], Ps[j], gamma, s=qs[j], Y=Ys[j], workspace=ws8[j])

    def kernel_step(i, stream=None):
        j = i % R
        tw.bitnet_w158a8_matmul(qx[j], Ps[j], gamma, s=qs[j], Y=Ys[j], workspace=ws8[j],
                                weights_static=True, weights_expanded=True, stream=stream)

    ops = 2 * M * N * K
    return dict(
        step=step, kernel_step=kernel_step, e2e_step=lambda i, stream=None: step(0, stream),
        e2e_plans=None if prep_in_kernel else (
            lambda xh, yh, stream=None: [tw.HostMatmulPlan(xh, Ps[0], gamma, Xs[0], Ys[0], yh,
                                                           workspace=wss[0], weights_static=True,
                                                           stream=stream)]),
        units_per_step=ops, unit="TOPS",
        scale=1e-12,
        bound="tensor", launches_per_step=2, kernel_launches_per_step=1, rotate=R, X=X0,
        Y=Ys[0], path=tw.bitnet_w158a8_matmul_path(M, N, K, torch.bfloat16),
        config={**workload_identity("prefill"),
                "l2": f"inputs larger than L2: {R} rotating input/output sets",
                "timing": ("CUDA graph; step = counter reset + tcgen05 kernel that quantises the "
                           "activations and expands the weights itself" if prep_in_kernel else
                           "CUDA graph; step = activation quantiser (the weights' expansion to "
                           "int8 scratch runs in the same launch) + tcgen05 kernel")},
        kernel_key="prefill_tcgen05_M4096_K2560_N6912",
        kernel_files=["ternary_weight_linear_token_b200/csrc/gemm_prefill.cu",
                      "ternary_weight_linear_token_b200/csrc/common.cuh",
                      "ternary_weight_linear_token_b200/csrc/quant_row.cuh"],
        e2e_inputs=lambda: (d["x_bits"].view(np.int16), 2 * M * K, 2 * M * N),
    )


def make_chain(tw, torch, dev, l2_bytes, layers=30, persistent=False):
    import synth
    from ternary_weight_linear_token_b200.chain import DecodeChain
    ws = []
    for li in range(layers):
        ws.append([(torch.from_numpy(synth.layer_weights(li, p)).to(dev), synth.PROJECTIONS[p][3])
                   for p in range(4)])
    chain = DecodeChain(ws, device=dev, persistent=persistent)
    del ws
    x0 = synth.config_inputs("chain", weights=False)
    X = torch.from_numpy(x0["x_bits"].view(np.int16)).to(dev).view(torch.bfloat16)
    chain.x_in.copy_(X)
    wbytes = chain.packed_bytes

    def step(i, stream=None):
        chain.run()

    # end to end: the token captured once as a CUDA graph (DecodeChain.capture), replayed
    held = {}

    def e2e_step(i, stream=None):
        if "g" not in held:
            held["g"] = chain.capture()
        held["g"].replay()

    return dict(
        step=step, kernel_step=None, units_per_step=wbytes, unit="GB/s", scale=1e-9, bound="hbm",
        launches_per_step=chain.launches_per_token(), rotate=1, X=chain.x_in, Y=chain.outs[-1][4],
        config={**workload_identity("chain", layers=layers),
                "l2": f"inputs larger than L2: {wbytes / 1e6:.0f} MB of packed weights per token",
                "mode": ("one persistent launch per token (bitnet_decode_chain)" if persistent
                         else "one launch per projection and per normalisation"),
                "timing": "CUDA graph of the timed steps"},
        kernel_key="chain_persistent_30layers" if persistent and layers == 30 else None,
        kernel_files=(["ternary_weight_linear_token_b200/csrc/chain.cu",
                       "ternary_weight_linear_token_b200/csrc/common.cuh"] if persistent else []),
        e2e_inputs=lambda: (x0["x_bits"].view(np.int16), 5120, 5120),
        e2e_step=e2e_step,
        e2e_note=("pinned host activations copied in, the token as a CUDA graph captured once "
                  "through the Python binding (DecodeChain.capture) and replayed, bf16 result "
                  "copied out, stream synchronised, every step"),
    )


MAKERS = {"decode": make_decode, "prefill": make_prefill, "chain": make_chain,
          "sweep": make_sweep}


# ------------------------------------------------------------------ CPU oracle
def oracle_sample(workload: str, budget_s: float, sweep_m: int = 8):
    """Time the plain C oracle on a bounded sample of the workload on the host
    cores.  Returns (value, unit, cores, sample description, seconds)."""
    import synth
    from oracle import ref
    R = ref.default()
    if workload == "prefill":
        d = synth.config_inputs("prefill")
        packed, gamma = R.quantize_weights(d["W"])
        rows = 4
        t0 = time.perf_counter()
        n = 0
        while True:
            R.bitlinear(d["x"][(n * rows) % 4096:(n * rows) % 4096 + rows], packed, gamma, d["N"])
            n += 1
            if time.perf_counter() - t0 > budget_s:
                break
        dt = time.perf_counter() - t0
        ops = 2 * rows * n * d["N"] * d["K"]
        return ops / dt * 1e-12, "TOPS", R.num_threads(), f"{n * rows} token rows x N=6912 x K=2560", dt
    if workload in ("chain", "sweep"):
        # one decoder layer: the four projections at the workload's tokens per call
        M = sweep_m if workload == "sweep" else 1
        projs = []
        for p in range(4):
            d = synth.config_inputs("sweep", M=M, proj=p)
            packed, gamma = R.quantize_weights(d["W"])
            projs.append((d, packed, gamma))
        layer_bytes = sum(packed.size for _, packed, _ in projs)
        t0 = time.perf_counter()
        n = 0
        while True:
            for d, packed, gamma in projs:
                R.bitlinear(d["x"], packed, gamma, d["N"], relu2=d["relu2"])
            n += 1
            if time.perf_counter() - t0 > budget_s:
                break
        dt = time.perf_counter() - t0
        return (n * layer_bytes / dt * 1e-9, "GB/s", R.num_threads(),
                f"{n} decoder layers (qkv, o, up + ReLU^2, down) at M={M}", dt)
    d = synth.config_inputs("decode")
    packed, gamma = R.quantize_weights(d["W"])
    t0 = time.perf_counter()
    n = 0
    while True:
        R.bitlinear(d["x"], packed, gamma, d["N"], relu2=d["relu2"])
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return (n * packed.size / dt * 1e-9, "GB/s", R.num_threads(),
            f"{n} full BitLinear forwards M=1 K={d['K']} N={d['N']}", dt)


# ------------------------------------------------------------------ main
def oracle_run(workload: str, steps: int, warmup: int, per_step: float, sweep_m: int):
    """The oracle timed over `steps` bounded samples of a workload (after
    `warmup` shorter ones): (value, unit, cores, sample description, seconds)."""
    for _ in range(warmup):
        oracle_sample(workload, per_step / 4, sweep_m)
    tot_units = 0.0
    t0 = time.perf_counter()
    cores, sample, unit = 1, "", "GB/s"
    for _ in range(steps):
        v, unit, cores, sample, dt = oracle_sample(workload, per_step, sweep_m)
        tot_units += v * dt
    dt = time.perf_counter() - t0
    return tot_units / dt, unit, cores, sample, dt


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    with_prefill = args.workload == "decode" and not args.no_prefill
    budget = 60.0 if with_prefill else 120.0
    per_step = max(0.02, min(2.0, budget / max(1, args.steps + args.warmup)))
    value, unit, cores, sample, dt = oracle_run(args.workload, args.steps, args.warmup, per_step,
                                                args.sweep_m)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8",
            "data": "synthetic",
            "config": {**workload_identity(args.workload, sweep_m=args.sweep_m),
                       "timing": "the oracle (plain C) on the host cores, a bounded sample of "
                                 "the workload per step, scaled to the metric's unit"},
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": f"per step ~{per_step:.2f} s of: {sample}"},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    if with_prefill:
        pv, pu, pc, ps, pdt = oracle_run("prefill", args.steps, args.warmup, per_step,
                                         args.sweep_m)
        line["prefill"] = {
            "metric": "prefill GEMM int8 TOPS", "value": pv, "unit": pu,
            "ms_per_step": 1e3 * pdt / max(1, args.steps),
            "config": {**workload_identity("prefill"),
                       "timing": "the oracle (plain C) on the host cores, a bounded sample of "
                                 "the workload per step, scaled to the metric's unit"},
            "cpu_baseline": {"value": pv, "unit": pu, "cores": pc, "kind": "oracle",
                             "sample": f"per step ~{per_step:.2f} s of: {ps}"},
            "e2e": {"value": pv, "unit": pu, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# Spin cycles that keep the GPU busy while the host submits a timed graph
# (about 1 ms plus 1 us per graph node at ~2 GHz).
def spin_cycles(nodes: int) -> int:
    return int(2_000_000 + 2_000 * nodes)


def capture_timed(torch, stream, fn, warm: int, first: int, count: int):
    """One CUDA graph: an untimed step fn(warm), then `count` timed steps
    fn(first + i), with a timing event before and after the timed ones.

    The start event is recorded on a side branch of the graph that depends on
    the untimed step alone, so the first timed step follows that step by
    programmatic dependent launch exactly as every later step follows its
    predecessor: the two events bracket `count` steps of the steady state,
    the same per-step time whether `count` is 20 or 2000, and none of the
    graph's start-up latency."""
    ev0 = torch.cuda.Event(enable_timing=True, external=True)
    ev1 = torch.cuda.Event(enable_timing=True, external=True)
    side = torch.cuda.Stream(stream.device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn(warm, stream)
        side.wait_stream(stream)
        ev0.record(side)
        for i in range(count):
            fn(first + i, stream)
        ev1.record(stream)
        stream.wait_stream(side)
    return g, ev0, ev1


def replay_timed(torch, timed, stream, nodes: int):
    """Device time (ms) between the events of one replay of a captured timed
    graph.  A spin kernel ahead of it keeps the GPU busy while the host
    submits the graph."""
    g, ev0, ev1 = timed
    with torch.cuda.stream(stream):
        torch.cuda._sleep(spin_cycles(nodes))
        g.replay()          # replays on the current stream, i.e. `stream`
    stream.synchronize()
    return ev0.elapsed_time(ev1)


def measure(w, tw, torch, args, dev, stream, pg, world, rank, bus):
    """Warm-up, then the timed steps from one CUDA graph; the dominant
    kernel's own time; end-to-end through the API; the oracle's CPU figure."""
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            w["step"](i, stream)
    stream.synchronize()
    graph = capture_timed(torch, stream, w["step"], args.warmup - 1, args.warmup, args.steps)
    kgraph = None
    if w.get("kernel_step") is not None and w["kernel_step"] is not w["step"]:
        kgraph = capture_timed(torch, stream, w["kernel_step"], args.steps, 0, args.steps)
    with torch.cuda.stream(stream):
        graph[0].replay()  # one untimed replay of each: first-launch costs of the graphs
        if kgraph is not None:
            kgraph[0].replay()
    stream.synchronize()

    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    nodes = args.steps * w["launches_per_step"]
    with ClockSampler(bus) as clocks:
        ms = replay_timed(torch, graph, stream, nodes)
        kms = ms
        if kgraph is not None:
            kms = replay_timed(torch, kgraph, stream, args.steps * w["kernel_launches_per_step"])
    torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    ms = max_over_ranks(ms, pg, dev)
    kms = max_over_ranks(kms, pg, dev)
    value = whole_job_value(world, w["units_per_step"], args.steps, ms * 1e-3, w["scale"])

    per_launch_s = kms * 1e-3 / args.steps
    pk, src = peaks()
    if w["bound"] == "hbm":
        peak, punit = float(pk["hbm_gbs"]), "GB/s"
        achieved = w["units_per_step"] / per_launch_s * 1e-9
        peak_note = f"hbm_gbs ({src}: STREAM-style copy)"
    else:
        peak, punit = float(pk["bf16_tflops"]) * INT8_PER_BF16, "TFLOP/s"
        achieved = w["units_per_step"] / per_launch_s * 1e-12
        peak_note = f"bf16_tflops x {INT8_PER_BF16} (int8/bf16 nominal ratio; {src} burst)"
    traffic = ncu_traffic(w["kernel_key"], w["kernel_files"]) if w["kernel_key"] else None
    roofline = {"bound": w["bound"], "achieved": achieved, "peak": peak, "unit": punit,
                "frac": achieved / peak, "traffic": traffic, "peak_source": peak_note,
                "kernel_us": 1e3 * kms / args.steps,
                "kernel_timing": ("the tensor-core kernel alone: a CUDA graph of one launch "
                                  "per step on prepared int8 activations and int8 weight "
                                  "copies, CUDA events around the timed launches")
                if kgraph is not None else "CUDA-event time of the timed steps"}

    # end to end through the public API: pinned host input -> device -> result -> host
    xh_np, h2d, d2h = w["e2e_inputs"]()
    xh = torch.from_numpy(np.ascontiguousarray(xh_np)).pin_memory()
    yh = torch.empty(w["Y"].shape, dtype=w["Y"].dtype).pin_memory()
    X = w["X"]
    e2e_step = w.get("e2e_step", w["step"])  # a step that reads X and writes Y
    e2e_plans = w.get("e2e_plans")
    # host-timed calls are short: at least 20 (and 10 untimed ones first), whatever --steps is
    n = max(20, args.e2e_steps)
    with torch.cuda.stream(stream):
        if e2e_plans is not None:
            # one C call per step: pinned host input -> device, the product,
            # result -> pinned host, stream synchronised (bitnet_w158a8_matmul_host,
            # through a HostMatmulPlan per weight copy: the arguments checked once)
            xh_t = xh.view(torch.bfloat16).view(X.shape)  # the bf16 bit patterns as bf16
            plans = e2e_plans(xh_t, yh, stream)
            for i in range(10):
                plans[i % len(plans)]()
            t0 = time.perf_counter()
            for i in range(n):
                plans[i % len(plans)]()
            dt = time.perf_counter() - t0
            how = ("HostMatmulPlan (bitnet_w158a8_matmul_host over fixed buffers, arguments "
                   "checked once) every step: pinned host activations copied in, the product, the "
                   "bf16 result copied back to pinned host memory, stream synchronised")
        else:
            for i in range(3):
                X.view(torch.int16).copy_(xh.view(X.shape), non_blocking=True)
                e2e_step(i, stream)
                yh.copy_(w["Y"], non_blocking=True)
            stream.synchronize()
            t0 = time.perf_counter()
            for i in range(n):
                X.view(torch.int16).copy_(xh.view(X.shape), non_blocking=True)
                e2e_step(i, stream)
                yh.copy_(w["Y"], non_blocking=True)
                stream.synchronize()
            dt = time.perf_counter() - t0
            how = w.get("e2e_note", "pinned host activations copied in, BitLinear via the "
                        "Python binding of the C ABI, bf16 result copied out, stream "
                        "synchronised, every step")
    dt = max_over_ranks(dt, pg, dev)
    ev = whole_job_value(world, w["units_per_step"], n, dt, w["scale"])
    e2e = {"value": ev, "unit": w["unit"], "h2d_bytes_per_step": int(h2d),
           "d2h_bytes_per_step": int(d2h), "steps": n, "note": how}

    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        v, unit, cores, sample, cdt = oracle_sample(w["name"], args.cpu_seconds, args.sweep_m)
        cpu = {"value": v, "unit": unit, "cores": cores, "kind": "oracle",
               "sample": f"{sample} in {cdt:.1f} s"}
    del graph, kgraph
    return dict(value=value, ms=ms, roofline=roofline, e2e=e2e, cpu_baseline=cpu,
                clocks=clocks.summary(), gpu_launches=nodes)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", choices=sorted(MAKERS), default="decode")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--sweep-m", type=int, default=8, help="sweep workload: tokens per call")
    ap.add_argument("--chain-mode", choices=["persistent", "per-launch"], default="per-launch",
                    help="chain workload: one persistent kernel per token, or one launch per step")
    ap.add_argument("--no-prefill", action="store_true",
                    help="decode workload: leave out the prefill object of the JSON line")
    ap.add_argument("--prep-in-kernel", action="store_true",
                    help="prefill workload: the tensor-core kernel prepares its own operands "
                         "(comparison form)")
    ap.add_argument("--table-lookup", action="store_true",
                    help="decode and sweep workloads (M <= 8): run the table-lookup comparison "
                         "kernel instead of the library's default path")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    world, rank, local = dist_setup()
    if args.impl == "reference":
        return run_reference(args, world, rank)

    import torch
    from __graft_entry__ import load_builder
    load_builder().build()
    import ternary_weight_linear_token_b200 as tw

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2**20))
    bus = "%08x:%02x:%02x.0" % (getattr(props, "pci_domain_id", 0), getattr(props, "pci_bus_id", 0),
                                getattr(props, "pci_device_id", 0))
    extra = {"persistent": args.chain_mode == "persistent"} if args.workload == "chain" else {}
    if args.workload == "sweep":
        extra = {"M": args.sweep_m}
    if args.table_lookup and args.workload in ("decode", "sweep"):
        extra["table_lookup"] = True
    if args.prep_in_kernel and args.workload == "prefill":
        extra["prep_in_kernel"] = True
    stream = torch.cuda.Stream(dev)
    w = MAKERS[args.workload](tw, torch, dev, l2, **extra)
    w["name"] = args.workload
    r = measure(w, tw, torch, args, dev, stream, pg, world, rank, bus)
    cfg, unit = w["config"], w["unit"]
    del w

    prefill = None
    if args.workload == "decode" and not args.no_prefill and not args.table_lookup:
        # the other half of the metric: the prefill GEMM (M=4096, K=2560,
        # N=6912) with the same timing rules, as its own object
        wp = make_prefill(tw, torch, dev, l2)
        wp["name"] = "prefill"
        rp = measure(wp, tw, torch, args, dev, stream, pg, world, rank, bus)
        prefill = {"metric": "prefill GEMM int8 TOPS", "value": rp["value"], "unit": "TOPS",
                   "ms_per_step": rp["ms"] / args.steps,
                   "config": dict(wp["config"], parallelism=f"replicas x{world}"
                                  if world > 1 else "1 GPU"),
                   "kernel_path": tw.PATH_NAMES.get(wp["path"], str(wp["path"])),
                   "roofline": rp["roofline"], "cpu_baseline": rp["cpu_baseline"],
                   "e2e": rp["e2e"], "clocks": rp["clocks"], "gpu_launches": rp["gpu_launches"]}
        del wp

    status = tw.bitnet_get_device_status(stream)
    if rank == 0:
        line = {
            "metric": METRIC, "value": r["value"], "unit": unit,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": r["ms"] / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8",
            "data": "synthetic (seeded; no dataset or trained weights)",
            "config": dict(cfg,
                           parallelism=f"replicas x{world}" if world > 1 else "1 GPU"),
            "roofline": r["roofline"],
            "cpu_baseline": r["cpu_baseline"],
            "clocks": r["clocks"],
            "e2e": r["e2e"],
            "gpu_launches": r["gpu_launches"],
            "device_status": int(status),
        }
        if prefill is not None:
            line["prefill"] = prefill
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
