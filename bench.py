"""Benchmark of the B200 BitLinear forward (W1.58A8) -- one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode|prefill|chain]
                    [--impl ours|reference]

Metric: decode GEMV weight GB/s (packed 2-bit weight bytes streamed per
second) and, for the prefill workload, int8 tensor-core TOPS (2*M*N*K per
second), each against the B200 roofline.

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


def make_decode(tw, torch, dev, l2_bytes):
    import synth
    d = synth.config_inputs("decode")
    W = torch.from_numpy(d["W"]).to(dev)
    packed, gamma = tw.bitnet_quantize_weights(W)
    del W
    wbytes = packed.numel()
    R = max(4, -(-3 * l2_bytes // wbytes))
    copies = torch.empty((R,) + tuple(packed.shape), dtype=torch.uint8, device=dev)
    copies[:] = packed
    X = torch.from_numpy(d["x_bits"].view(np.int16)).to(dev).view(torch.bfloat16)
    Y = torch.empty((1, d["N"]), dtype=torch.bfloat16, device=dev)

    def step(i, stream=None):
        tw.bitnet_w158a8_matmul(X, copies[i % R], gamma, Y=Y, weights_static=True, stream=stream)

    return dict(
        step=step, kernel_step=step, units_per_step=wbytes, unit="GB/s", scale=1e-9, bound="hbm",
        launches_per_step=1, X=X, Y=Y, rotate=R, extra=dict(packed=copies, gamma=gamma),
        config={**workload_identity("decode"),
                "l2": f"inputs larger than L2: {R} rotating weight copies, "
                      f"{R * wbytes / 1e6:.0f} MB >= 3x L2",
                "timing": "CUDA graph of the timed steps, programmatic dependent launch, "
                          "weights flagged static"},
        kernel_key="decode_gemv_M1_K2560_N2560",
        kernel_files=["ternary_weight_linear_token_b200/csrc/gemv_rows.cu",
                      "ternary_weight_linear_token_b200/csrc/common.cuh"],
        e2e_inputs=lambda: (d["x_bits"].view(np.int16), 2 * d["K"], 2 * d["N"]),
    )


def make_sweep(tw, torch, dev, l2_bytes, M=8):
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
                                    stream=stream)

    d0 = projs[0]["d"]
    launches = 4 if M <= 3 else 8  # 4 tokens and more: quantiser + product per projection
    return dict(
        step=step, kernel_step=step, units_per_step=wbytes, unit="GB/s", scale=1e-9, bound="hbm",
        launches_per_step=launches, X=projs[0]["X"], Y=projs[3]["Y"], rotate=R,
        config={**workload_identity("sweep", sweep_m=M),
                "l2": f"inputs larger than L2: {R} rotating copies of the layer's weights, "
                      f"{R * wbytes / 1e6:.0f} MB >= 3x L2",
                "timing": "CUDA graph of the timed steps, programmatic dependent launch, "
                          "weights flagged static"},
        kernel_key=None, kernel_files=[],
        e2e_inputs=lambda: (d0["x_bits"].view(np.int16), 2 * M * d0["K"], 2 * M * 2560),
    )


def make_prefill(tw, torch, dev, l2_bytes):
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
                                weights_static=True, stream=stream)

    qx = [torch.empty((M, K), dtype=torch.int8, device=dev) for _ in range(R)]
    qs = [torch.empty(M, dtype=torch.float32, device=dev) for _ in range(R)]

    def quant_step(i, stream=None):  # the step's activation quantiser alone
        j = i % R
        tw.bitnet_quantize_act(Xs[j], xq=qx[j], s=qs[j], stream=stream)

    ops = 2 * M * N * K
    return dict(
        step=step, kernel_step=None, quant_step=quant_step, units_per_step=ops, unit="TOPS",
        scale=1e-12,
        bound="tensor", launches_per_step=2, rotate=R, X=X0, Y=Ys[0],
        config={**workload_identity("prefill"),
                "l2": f"inputs larger than L2: {R} rotating input/output sets",
                "timing": "CUDA graph; step = activation quantiser (the weights' expansion to "
                          "int8 scratch runs in the same launch) + tcgen05 kernel"},
        kernel_key="prefill_tcgen05_M4096_K2560_N6912",
        kernel_files=["ternary_weight_linear_token_b200/csrc/gemm_prefill.cu",
                      "ternary_weight_linear_token_b200/csrc/common.cuh"],
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

    return dict(
        step=step, kernel_step=None, units_per_step=wbytes, unit="GB/s", scale=1e-9, bound="hbm",
        launches_per_step=chain.launches_per_token(), rotate=1, X=chain.x_in, Y=chain.outs[-1][4],
        config={**workload_identity("chain", layers=layers),
                "l2": f"inputs larger than L2: {wbytes / 1e6:.0f} MB of packed weights per token",
                "mode": ("one persistent launch per token (bitnet_decode_chain)" if persistent
                         else "one launch per projection and per normalisation"),
                "timing": "CUDA graph of the timed steps"},
        kernel_key=None, kernel_files=[], e2e_inputs=lambda: (x0["x_bits"].view(np.int16), 5120, 5120),
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
def run_reference(args, world, rank):
    if rank != 0:
        return 0
    per_step = max(0.02, min(2.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(args.workload, per_step / 4, args.sweep_m)
    tot_units = 0.0
    t0 = time.perf_counter()
    cores = 1
    sample = ""
    unit = "GB/s"
    for _ in range(args.steps):
        v, unit, cores, sample, dt = oracle_sample(args.workload, per_step, args.sweep_m)
        tot_units += v * dt
    dt = time.perf_counter() - t0
    value = tot_units / dt
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
    print(json.dumps(line), flush=True)
    return 0


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
    extra = {"persistent": args.chain_mode == "persistent"} if args.workload == "chain" else {}
    if args.workload == "sweep":
        extra = {"M": args.sweep_m}
    w = MAKERS[args.workload](tw, torch, dev, l2, **extra)
    stream = torch.cuda.Stream(dev)

    # warm-up (eager launches), then capture the timed steps in one graph
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            w["step"](i, stream)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(args.steps):
            w["step"](args.warmup + i, stream)
    qgraph = None
    if w.get("quant_step") is not None:
        qgraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(qgraph, stream=stream):
            for i in range(args.steps):
                w["quant_step"](i, stream)
    with torch.cuda.stream(stream):
        graph.replay()  # one untimed replay: first-launch costs of the graph
    stream.synchronize()

    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    bus = "%08x:%02x:%02x.0" % (getattr(props, "pci_domain_id", 0), getattr(props, "pci_bus_id", 0),
                                getattr(props, "pci_device_id", 0))
    with ClockSampler(bus) as clocks, torch.cuda.stream(stream):
        ev0.record(stream)
        graph.replay()          # replays on the current stream, i.e. `stream`
        ev1.record(stream)
        ev1.synchronize()
    torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1), pg, dev)
    value = whole_job_value(world, w["units_per_step"], args.steps, ms * 1e-3, w["scale"])

    # dominant kernel (prefill: the tcgen05 kernel = step minus its activation
    # quantiser, each timed live with CUDA events on the same stream)
    kms = ms
    quant_ms = None
    if qgraph is not None:
        with torch.cuda.stream(stream):
            qgraph.replay()
            stream.synchronize()
            ev0.record(stream)
            qgraph.replay()
            ev1.record(stream)
            ev1.synchronize()
        quant_ms = max_over_ranks(ev0.elapsed_time(ev1), pg, dev)
        kms = ms - quant_ms
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

    # end to end through the public API: pinned host input -> device -> result -> host
    e2e = None
    xh_np, h2d, d2h = w["e2e_inputs"]()
    if True:
        xh = torch.from_numpy(np.ascontiguousarray(xh_np)).pin_memory()
        yh = torch.empty(w["Y"].shape, dtype=w["Y"].dtype).pin_memory()
        X = w["X"]
        n = max(3, min(args.e2e_steps, args.steps))
        with torch.cuda.stream(stream):
            for i in range(3):
                X.view(torch.int16).copy_(xh.view(X.shape), non_blocking=True)
                w["step"](i, stream)
                yh.copy_(w["Y"], non_blocking=True)
            stream.synchronize()
            t0 = time.perf_counter()
            for i in range(n):
                X.view(torch.int16).copy_(xh.view(X.shape), non_blocking=True)
                w["step"](i, stream)
                yh.copy_(w["Y"], non_blocking=True)
                stream.synchronize()
            dt = time.perf_counter() - t0
        dt = max_over_ranks(dt, pg, dev)
        ev = whole_job_value(world, w["units_per_step"], n, dt, w["scale"])
        e2e = {"value": ev, "unit": w["unit"], "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "steps": n,
               "note": "pinned host activations copied in, BitLinear via the Python binding of "
                       "the C ABI, bf16 result copied out, stream synchronised, every step"}

    status = tw.bitnet_get_device_status(stream)
    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        v, unit, cores, sample, dt = oracle_sample(args.workload, args.cpu_seconds, args.sweep_m)
        cpu = {"value": v, "unit": unit, "cores": cores, "kind": "oracle",
               "sample": f"{sample} in {dt:.1f} s"}
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": w["unit"], "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8",
            "data": "synthetic (seeded; no dataset or trained weights)",
            "config": dict(w["config"], parallelism=f"replicas x{world}" if world > 1 else "1 GPU"),
            "roofline": {"bound": w["bound"], "achieved": achieved, "peak": peak, "unit": punit,
                         "frac": achieved / peak, "traffic": traffic, "peak_source": peak_note,
                         "kernel_us": 1e3 * kms / args.steps,
                         "kernel_timing": ("step time minus the time of the activation quantiser "
                                           "alone (without the weight expansion, which the "
                                           "kernel's figure therefore carries), both CUDA-event "
                                           "timed on the launch stream")
                         if quant_ms is not None else "CUDA-event time of the timed steps"},
            "cpu_baseline": cpu,
            "clocks": clocks.summary(),
            "e2e": e2e,
            "gpu_launches": w["launches_per_step"] * args.steps,
            "device_status": int(status),
        }
        print(json.dumps(line), flush=True)
    del graph, qgraph
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
