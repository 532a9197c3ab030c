#!/usr/bin/env python3
"""Benchmark of the FP8 fast-math linear layer on B200.

Headline workload: a 4096-token prompt read through two chained FP8 linear
layers (K=2048 -> N=6144 -> 2048), each one per-token FP8 quantization of its
BF16 input followed by the tcgen05 W8A8 GEMM with the per-token x
per-channel scale epilogue. One step = q1 + G1 + q2 + G2 over one batch;
value = whole-job tokens per second (N GPUs run independent replicas with
their own token batches: weak scaling, no collective on the data path).

Inputs are seeded synthetic data of the workload's shapes and distributions
(BF16 activations ~N(0,1) with 1% outlier channels x30, FP32 weights ~N(0,0.02)
quantized per output channel on the GPU before timing). Four layer sets
(x, W1, W2) rotate from step to step so the working set (169 MB) exceeds the
126 MB L2.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl metis|reference]
Prints one JSON line (rank 0).
"""
import argparse
import datetime
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

METRIC = "FP8 W8A8 GEMM TFLOP/s & % FP8 peak; 4096-tok prefill tok/s; decode GB/s %HBM"
M_TOK, K_HID, N_FF = 4096, 2048, 6144
SETS = 4
ISO_CALLS = 200  # layer-1 GEMM launches per graph in the isolated roofline timing
NOMINAL_FP8_TFLOPS = 4500.0  # dense FP8 tensor peak of a B200 (nominal, for context)
NOMINAL_HBM_GBS = 8000.0  # HBM3e bandwidth of a B200 (nominal, for context)
FP8_PER_BF16 = 2.0  # nominal dense FP8 : BF16 tensor throughput (4.5 : 2.25 PFLOP/s)
FP4_PER_BF16 = 4.0  # nominal dense FP4 : BF16 tensor throughput (9 : 2.25 PFLOP/s)
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["metis", "reference"], default="metis")
    ap.add_argument("--no-secondary", action="store_true", help="skip the context figures")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work")
    ap.add_argument("--ref-budget", type=float, default=150.0,
                    help="seconds of oracle work in the reference arm (warm-up + timed steps)")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK, "fallback"


def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(set_index, rank):
    """Seed of layer set `set_index` on `rank`: every rank draws its own
    token batch and weights (weak scaling, independent replicas)."""
    return 1 + 100 * set_index + 10000 * rank


def max_over_ranks(value, dist, device, world):
    """The slowest rank's device time (all ranks take part; rank order of the
    collective is the same on every rank)."""
    if world <= 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, tokens_per_rank, ms_per_step):
    """Whole-job tokens per second: every rank processes its own batch per step."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


# ---------------------------------------------------------------- CPU oracle

def oracle_prefill_tokens(d, wq, tokens):
    """The oracle's prefill chain on the given tokens (rows are independent)."""
    import oracle
    (w1q, s1), (w2q, s2) = wq
    xq, st = oracle.quant_per_token(d["x"][tokens])
    y1, _ = oracle.gemm_w8a8(xq, st, w1q, s1)
    xq2, st2 = oracle.quant_per_token(y1)
    y2, _ = oracle.gemm_w8a8(xq2, st2, w2q, s2)
    return y2


def cpu_baseline(budget_s, batch=256):
    """Times the oracle (as it stands) on as many tokens of the workload as fit
    in about `budget_s` seconds, in batches of `batch` tokens."""
    import oracle
    from moe_gemm_token_b200 import synth
    d = synth.prefill_chain()
    wq = (oracle.quant_per_channel(d["w1"]), oracle.quant_per_channel(d["w2"]))
    done, t0 = 0, time.perf_counter()
    while done < M_TOK:
        toks = np.arange(done, min(M_TOK, done + batch))
        oracle_prefill_tokens(d, wq, toks)
        done += toks.size
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": done / dt, "unit": "tok/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{done} of the {M_TOK} tokens of the prefill chain (quantize, GEMM "
                      f"2048->6144, quantize, GEMM 6144->2048), float64 oracle, {dt:.1f} s"}


def bench_config(world):
    """The workload of the JSON line, identical in both arms."""
    return {"workload": "prefill_chain_4096tok_2048x6144x2048", "global_batch": world * M_TOK,
            "tokens_per_gpu": M_TOK, "layers": "2048->6144 then 6144->2048, no activation",
            "step": "quantize+GEMM+quantize+GEMM", "parallelism": f"replicas x{world}",
            "timed_as": "one CUDA graph of the K steps",
            "l2": f"{SETS} rotating layer sets (x, W1, W2), 169 MB > 126 MB L2"}


def run_reference(args):
    rank, world, _ = env_rank()
    if rank != 0:
        return 0
    import oracle
    from moe_gemm_token_b200 import synth
    d = synth.prefill_chain()
    wq = (oracle.quant_per_channel(d["w1"]), oracle.quant_per_channel(d["w2"]))
    t0 = time.perf_counter()
    oracle_prefill_tokens(d, wq, np.arange(8))
    per_tok = (time.perf_counter() - t0) / 8
    budget = args.ref_budget  # seconds for warm-up + timed steps
    per_step = max(1, min(M_TOK, int(budget / max(1, args.steps + args.warmup) / per_tok)))
    step_tokens = lambda i: (np.arange(per_step) + i * per_step) % M_TOK
    for i in range(args.warmup):
        oracle_prefill_tokens(d, wq, step_tokens(i))
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle_prefill_tokens(d, wq, step_tokens(args.warmup + i))
    dt = time.perf_counter() - t0
    value = args.steps * per_step / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(world),
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": f"each step a bounded sample of {per_step} of the {M_TOK} tokens of "
                                   f"the prefill chain (float64 oracle, rows are independent)"},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------- clock sampler

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML (read-only)."""

    def __init__(self, device_index, period=0.02):
        self.samples = []
        self.period = period
        self.ok = False
        try:
            import pynvml as nv
            import torch
            nv.nvmlInit()
            self.nv = nv
            # NVML ignores CUDA_VISIBLE_DEVICES: find this device by its UUID
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = nv.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that instead of clocks
            self.err = str(e)
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, r))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        nv = self.nv
        names = {
            nv.nvmlClocksEventReasonGpuIdle: "gpu_idle",
            nv.nvmlClocksEventReasonApplicationsClocksSetting: "applications_clocks",
            nv.nvmlClocksEventReasonSwPowerCap: "sw_power_cap",
            nv.nvmlClocksEventReasonHwSlowdown: "hw_slowdown",
            nv.nvmlClocksEventReasonSyncBoost: "sync_boost",
            nv.nvmlClocksEventReasonSwThermalSlowdown: "sw_thermal_slowdown",
            nv.nvmlClocksEventReasonHwThermalSlowdown: "hw_thermal_slowdown",
            nv.nvmlClocksEventReasonHwPowerBrakeSlowdown: "hw_power_brake_slowdown",
        }
        reasons = set()
        for _, r in self.samples:
            for bit, name in names.items():
                if r & bit:
                    reasons.add(name)
        mhz = [m for m, _ in self.samples]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(mhz)}


# --------------------------------------------------------------- metis arm

def moe_floor_us(T, H, I, E, k, hbm_gbs, peak_tflops, fp4):
    """Lower bound on the routed-expert layer's time: for each HBM-heavy
    kernel the larger of its algorithmic bytes over the measured HBM
    bandwidth and its FLOPs over the tensor peak, summed (the latency-bound
    routing kernels count as zero). Bytes per kernel, with S = T * k slots:
    quantizer of x (x read, codes + scales written into S rows), grouped
    up-projection (codes of x, expert weights, h written), quantizer of h,
    grouped down-projection (codes of h, weights, o written), combine (o read,
    y written). Codes are 1 byte per element in FP8 and half a byte plus one
    E4M3 scale per 16 in NVFP4."""
    S = T * k
    code = (lambda n: n / 2 + n / 16) if fp4 else (lambda n: n)
    fl = 2.0 * S * I * H
    kernels = [
        (2 * T * H + code(S * H) + 4 * S, 0.0),                  # quantize x into expert rows
        (code(S * H) + code(E * I * H) + 2 * S * I, fl),         # up-projection
        (2 * S * I + code(S * I) + 4 * S, 0.0),                  # quantize h
        (code(S * I) + code(E * H * I) + 2 * S * H, fl),         # down-projection
        (2 * S * H + 8 * S + 2 * T * H, 0.0),                    # weighted combine
    ]
    return sum(max(b / (hbm_gbs * 1e9), f / (peak_tflops * 1e12)) for b, f in kernels) * 1e6


GEMM_COUNTERS = os.path.join(ROOT, "profiles", "fp8_gemm_prefill_4096x6144x2048.json")
GEMM_SOURCES = [os.path.join(ROOT, "moe_gemm_token_b200", "csrc", f) for f in ("gemm_fp8.cu", "common.cuh")]


def gemm_source_sha():
    """sha256[:16] of the sources the prefill GEMM kernel is compiled from."""
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def gemm_traffic_from_profile():
    """DRAM bytes per layer-1 GEMM launch (dram__bytes_read.sum +
    dram__bytes_write.sum) from the committed ncu counters, if they were taken
    on the current kernel sources (else None)."""
    try:
        with open(GEMM_COUNTERS) as f:
            c = json.load(f)
    except (OSError, ValueError):
        return None
    if c.get("kernel_sources_sha256_16") != gemm_source_sha():
        return None
    try:
        return float(c["dram_bytes_read"]) + float(c["dram_bytes_write"])
    except (KeyError, TypeError, ValueError):
        return None


def run_metis(args):
    import torch
    import torch.distributed as dist
    from moe_gemm_token_b200 import metis, synth

    rank, world, local = env_rank()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=dev)
    metis.load()
    stream = torch.cuda.current_stream()

    def bf16(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    # ---- inputs: SETS layer sets, weights quantized per channel on the GPU
    sets = []
    for r in range(SETS):
        d = synth.prefill_chain(seed=rank_seed(r, rank))
        ws = []
        for w in (d["w1"], d["w2"]):
            wd = torch.from_numpy(w).to(dev)
            wq = torch.empty(w.shape, dtype=torch.uint8, device=dev)
            sw = torch.empty((w.shape[0],), dtype=torch.float32, device=dev)
            metis.metis_quant_fp8_per_channel(wd, wq, sw)
            ws.append((wq, sw))
            del wd
        sets.append({"x": bf16(d["x"]), "x_host": d["x"], "w": ws})
    xq1 = torch.empty((M_TOK, K_HID), dtype=torch.uint8, device=dev)
    st1 = torch.empty((M_TOK,), dtype=torch.float32, device=dev)
    y1 = torch.empty((M_TOK, N_FF), dtype=torch.bfloat16, device=dev)
    xq2 = torch.empty((M_TOK, N_FF), dtype=torch.uint8, device=dev)
    st2 = torch.empty((M_TOK,), dtype=torch.float32, device=dev)
    y2 = torch.empty((M_TOK, K_HID), dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize()

    def step(i, st, ev=None):
        s = sets[i % SETS]
        (w1, s1), (w2, s2) = s["w"]
        metis.metis_quant_fp8_per_token(s["x"], xq1, st1, st)
        if ev is not None:
            ev[0].record(st)
        metis.metis_fp8_gemm(xq1, metis.METIS_A_E4M3, st1, w1, s1, y1, stream=st)
        if ev is not None:
            ev[1].record(st)
        metis.metis_quant_fp8_per_token(y1, xq2, st2, st)
        if ev is not None:
            ev[2].record(st)
        metis.metis_fp8_gemm(xq2, metis.METIS_A_E4M3, st2, w2, s2, y2, stream=st)
        if ev is not None:
            ev[3].record(st)

    launches_per_step = 4
    for i in range(args.warmup):
        step(i, stream)
    torch.cuda.synchronize()
    if metis.metis_check_device_status(stream) != 0:
        raise RuntimeError("device status error after warm-up")

    # The timed region is one CUDA graph of the K steps (no host launch gaps
    # between kernels, no timing events inside); it is replayed once untimed
    # (upload, warm-up) and once timed, bracketed by events on the stream it
    # runs on.
    cap = torch.cuda.Stream(device=dev)
    cap.wait_stream(stream)
    start = torch.cuda.Event(enable_timing=True, external=True)
    end = torch.cuda.Event(enable_timing=True, external=True)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cap):
        start.record(cap)
        for i in range(args.steps):
            step(i, cap)
        end.record(cap)
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        graph.replay()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    elapsed_ms = max_over_ranks(start.elapsed_time(end), dist, dev, world)
    ms_per_step = elapsed_ms / args.steps
    value = job_throughput(world, M_TOK, ms_per_step)
    del graph

    # ---- roofline of the dominant kernel (the W8A8 GEMM, layer 1 shape)
    pk, pk_kind = peaks()
    flops = 2.0 * M_TOK * K_HID * N_FF
    burst = pk["bf16_tflops"] * FP8_PER_BF16
    sustained = pk["bf16_tflops_sustained"] * FP8_PER_BF16
    # (a) in isolation: ISO_CALLS layer-1 GEMMs in one CUDA graph, rotating
    # the SETS layer sets (A codes and W1 of every set: 84 MB, plus the 50 MB
    # output), replayed 3 times between two events on the replay stream. Its
    # denominator is the burst tensor figure (a kernel timed alone).
    xq_sets = []
    for s in sets:
        q = torch.empty((M_TOK, K_HID), dtype=torch.uint8, device=dev)
        sc = torch.empty((M_TOK,), dtype=torch.float32, device=dev)
        metis.metis_quant_fp8_per_token(s["x"], q, sc, stream)
        xq_sets.append((q, sc))
    torch.cuda.synchronize()

    def gemm1(i, st):
        (q, sc), (w1, s1) = xq_sets[i % SETS], sets[i % SETS]["w"][0]
        metis.metis_fp8_gemm(q, metis.METIS_A_E4M3, sc, w1, s1, y1, stream=st)

    for i in range(2 * SETS):
        gemm1(i, stream)
    torch.cuda.synchronize()
    iso_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(iso_graph, stream=cap):
        for i in range(ISO_CALLS):
            gemm1(i, cap)
    torch.cuda.synchronize()
    iso_graph.replay()
    torch.cuda.synchronize()
    a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 3
    # the SM clock during this window (about 26 ms): under the power cap it
    # falls while the GEMMs run, and the kernel's time follows it
    with ClockSampler(local, period=0.002) as iso_clk:
        a_ev.record(stream)
        for _ in range(reps):
            iso_graph.replay()
        b_ev.record(stream)
        torch.cuda.synchronize()
    iso_ms = a_ev.elapsed_time(b_ev) / (reps * ISO_CALLS)
    iso_clocks = iso_clk.summary()
    del iso_graph
    achieved = flops / (iso_ms * 1e-3) / 1e12
    # (b) inside the step, as a cross-check: a separate replay of the step
    # graph with events around both GEMMs of every step. An event inside a
    # graph is a node of its own: it ends the programmatic overlap of the
    # GEMM's launch and set-up with the kernel before it, so each bracketed
    # interval also holds that launch and set-up and these durations err
    # high; they do not enter the timed region.
    n_ev = max(10, min(args.steps, 50))
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)] for _ in range(n_ev)]
    ev_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ev_graph, stream=cap):
        for i in range(n_ev):
            step(i, cap, evs[i])
    torch.cuda.synchronize()
    ev_graph.replay()
    torch.cuda.synchronize()
    ev_graph.replay()
    torch.cuda.synchronize()
    g1 = [e[0].elapsed_time(e[1]) for e in evs]
    g2 = [e[2].elapsed_time(e[3]) for e in evs]
    del ev_graph
    in_step = flops / (statistics.median(g1) * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
                "frac": achieved / burst, "traffic": gemm_traffic_from_profile(),
                "kernel": "fp8_gemm_kernel (tcgen05 kind::f8f6f4, cta_group::2, 256x256 tiles per CTA pair), "
                          "M=4096 N=6144 K=2048",
                "peak_source": f"{pk_kind} bf16 burst {pk['bf16_tflops']} TFLOP/s x {FP8_PER_BF16} "
                               f"(nominal FP8:BF16 dense ratio)",
                "timed_as": f"{ISO_CALLS} GEMM launches per CUDA graph, {SETS} rotating input sets, "
                            f"{reps} replays between events",
                "us_per_launch": iso_ms * 1e3,
                "clocks": iso_clocks,
                "kcycles_per_launch": (iso_ms * iso_clocks["sm_mhz"] if iso_clocks.get("sm_mhz") else None),
                "frac_of_sustained": achieved / sustained,
                "frac_of_nominal_fp8": achieved / NOMINAL_FP8_TFLOPS,
                "in_step": {"achieved": in_step, "frac": in_step / burst, "gemm_samples": len(g1),
                            "layer1_us_median": statistics.median(g1) * 1e3,
                            "layer2_us_median": statistics.median(g2) * 1e3,
                            "note": "events inside a step graph (not the timed one); each event node "
                                    "ends the GEMM's programmatic launch overlap, so the intervals also "
                                    "hold its launch and set-up and err high"}}

    # ---- end to end through the C ABI with host buffers. Every step uploads
    # its input from pinned host memory, runs the two layers through
    # metis_linear (the user-facing call) and downloads its output. Steps are
    # pipelined over three streams with double-buffered device inputs and
    # outputs: the upload of step i+1 and the download of step i-1 overlap
    # the compute of step i (PCIe is full duplex; the copy engines run
    # beside the SMs).
    e2e_steps = min(args.steps, 200)
    x_host = torch.from_numpy(sets[0]["x_host"].view(np.int16)).view(torch.bfloat16).pin_memory()
    y_host = [torch.empty((M_TOK, K_HID), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_dev = [torch.empty((M_TOK, K_HID), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    y_dev = [torch.empty((M_TOK, K_HID), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    (w1, s1), (w2, s2) = sets[0]["w"]
    lin_ws = torch.zeros(max(metis.metis_workspace_size(metis.METIS_OP_LINEAR, M_TOK, N_FF, K_HID, 0, 0),
                             metis.metis_workspace_size(metis.METIS_OP_LINEAR, M_TOK, K_HID, N_FF, 0, 0)),
                         dtype=torch.uint8, device=dev)
    s_h2d, s_comp, s_d2h = (torch.cuda.Stream(device=dev) for _ in range(3))
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        b = i % 2
        if i >= 2:
            s_h2d.wait_event(comp_done[b])   # step i-2 has read x_dev[b]
        with torch.cuda.stream(s_h2d):
            x_dev[b].copy_(x_host, non_blocking=True)
        h2d_done[b].record(s_h2d)
        s_comp.wait_event(h2d_done[b])
        if i >= 2:
            s_comp.wait_event(d2h_done[b])   # y_dev[b] of step i-2 is on the host
        metis.metis_linear(x_dev[b], w1, s1, y1, fast_math=True, s_tok=st1, workspace=lin_ws, stream=s_comp)
        metis.metis_linear(y1, w2, s2, y_dev[b], fast_math=True, s_tok=st2, workspace=lin_ws, stream=s_comp)
        comp_done[b].record(s_comp)
        s_d2h.wait_event(comp_done[b])
        with torch.cuda.stream(s_d2h):
            y_host[b].copy_(y_dev[b], non_blocking=True)
        d2h_done[b].record(s_d2h)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for st_ in (s_h2d, s_comp, s_d2h):
        st_.wait_stream(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_stream(s_d2h)
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b) / e2e_steps, dist, dev, world)
    e2e = {"value": job_throughput(world, M_TOK, e2e_ms), "unit": "tok/s",
           "h2d_bytes_per_step": M_TOK * K_HID * 2, "d2h_bytes_per_step": M_TOK * K_HID * 2,
           "steps": e2e_steps, "api": "metis_linear x 2 per step",
           "pipelined": "upload of step i+1 and download of step i-1 overlap step i "
                        "(3 streams, double-buffered device input and output)"}

    secondary = None
    if not args.no_secondary:
        secondary = secondary_figures(metis, dev, pk)
    if metis.metis_check_device_status(stream) != 0:
        raise RuntimeError("device status error after the timed region")

    cpu = None
    if rank == 0 and world == 1:
        cpu = cpu_baseline(args.cpu_budget)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
            "data": "synthetic",
            "config": bench_config(world),
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary(), "secondary": secondary,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def secondary_figures(metis, dev, pk):
    """Context figures of the other hot-path kernels (not the headline):
    decode W8A16 GB/s, quantizer GB/s, large-M W8A8 TFLOP/s, routed experts.
    Each is timed by replaying a CUDA graph of many calls."""
    import torch
    g = torch.Generator(device=dev)
    g.manual_seed(7)

    def codes(n, k):
        c = torch.randint(0, 256, (n, k), dtype=torch.uint8, device=dev, generator=g)
        c[(c & 0x7F) == 0x7F] = 0x38
        return c

    clk_samples = []

    def figure_mhz():
        """Median SM clock over the timed replays since the previous call."""
        m = statistics.median(clk_samples) if clk_samples else None
        clk_samples.clear()
        return m

    def timeit(fn, iters):
        """GPU time per call: `iters` calls captured once in a CUDA graph and
        replayed, so host-side launch overhead does not enter the figure.
        The SM clock is sampled during the timed replays (figure_mhz)."""
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        stream = torch.cuda.Stream()
        stream.wait_stream(torch.cuda.current_stream())
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(graph, stream=stream):
                for _ in range(iters):
                    fn()
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 3
        with ClockSampler(torch.cuda.current_device(), period=0.002) as clk:
            a.record()
            for _ in range(reps):
                graph.replay()
            b.record()
            torch.cuda.synchronize()
        clk_samples.extend(m for m, _ in getattr(clk, "samples", []))
        del graph
        return a.elapsed_time(b) / (reps * iters) * 1e-3

    class Figures(dict):
        """Each figure records the median SM clock of its timed replays."""

        def __setitem__(self, key, value):
            super().__setitem__(key, dict(value, sm_mhz=figure_mhz()))

    out = Figures()
    hbm = pk["hbm_gbs"]
    peak8 = pk["bf16_tflops"] * FP8_PER_BF16
    # the tiny linear layer (16 tokens, 256 -> 512): launch-latency bound,
    # quantizer + E4M3 GEMM per call
    xt = torch.randn(16, 256, device=dev, generator=g).to(torch.bfloat16)
    wt, swt = codes(512, 256), torch.rand(512, device=dev, generator=g) * 1e-3
    xqt = torch.empty(16, 256, dtype=torch.uint8, device=dev)
    stt = torch.empty(16, device=dev)
    yt = torch.empty(16, 512, dtype=torch.bfloat16, device=dev)

    def tiny():
        metis.metis_quant_fp8_per_token(xt, xqt, stt)
        metis.metis_fp8_gemm(xqt, 0, stt, wt, swt, yt)
    out["tiny_linear_16x512x256"] = {"us": timeit(tiny, 200) * 1e6}
    del xt, wt, swt, xqt, stt, yt
    # decode: 5 rotating weight sets (294 MB, more than twice the 126 MB L2)
    N, K = 14336, 4096
    DSETS = 5
    ws = [codes(N, K) for _ in range(DSETS)]
    sw = torch.rand(N, device=dev, generator=g) * 1e-3
    for M in (1, 2, 4, 8):
        x = torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        i = [0]

        def f():
            i[0] = (i[0] + 1) % DSETS
            metis.metis_w8a16_gemm(x, ws[i[0]], sw, y)
        t = timeit(f, 200)
        byt = N * K + 4 * N + 2 * M * K + 2 * M * N
        out[f"decode_w8a16_M{M}"] = {"us": t * 1e6, "GB/s": byt / t / 1e9,
                                     "frac_of_measured_hbm": byt / t / 1e9 / hbm,
                                     "frac_of_nominal_hbm": byt / t / 1e9 / NOMINAL_HBM_GBS}
    del ws
    # quantizer at the prefill and large-M shapes (2 rotating inputs > L2)
    for (M, K) in [(4096, 2048), (4096, 6144), (16384, 8192)]:
        # enough rotating inputs that they cannot stay in the 126 MB L2
        # (inputs and outputs: an output rewritten every call would stay in L2)
        n_in = max(2, -(-2 * 126 * 2 ** 20 // (3 * M * K)) + 1)
        xs = [torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16) for _ in range(n_in)]
        xqs = [torch.empty(M, K, dtype=torch.uint8, device=dev) for _ in range(n_in)]
        s = torch.empty(M, device=dev)
        i = [0]

        def f():
            i[0] = (i[0] + 1) % n_in
            metis.metis_quant_fp8_per_token(xs[i[0]], xqs[i[0]], s)
        t = timeit(f, 100)
        out[f"quant_{M}x{K}"] = {"us": t * 1e6, "GB/s": (3 * M * K + 4 * M) / t / 1e9,
                                 "frac_of_measured_hbm": (3 * M * K + 4 * M) / t / 1e9 / hbm,
                                 "frac_of_nominal_hbm": (3 * M * K + 4 * M) / t / 1e9 / NOMINAL_HBM_GBS}
        del xs, xqs
    # routed experts: 4096 tokens, hidden 2048, latent 1024, 64 experts, top-8
    # (a generator of its own, so the workload does not depend on the figures
    # timed before it)
    g.manual_seed(3)
    T, H, I, E, k = 4096, 2048, 1024, 64, 8
    x = torch.randn(T, H, device=dev, generator=g).to(torch.bfloat16)
    logits = torch.randn(T, E, device=dev, generator=g)
    logits[:, :4] += 0.93  # skew toward four hot experts
    top = torch.topk(logits, k, dim=1)
    ids = top.indices.to(torch.int32).contiguous()
    w = torch.softmax(top.values, dim=1).float().contiguous()
    wu = codes(E * I, H).view(E, I, H)
    su = torch.rand(E, I, device=dev, generator=g) * 1e-3
    wd = codes(E * H, I).view(E, H, I)
    sd = torch.rand(E, H, device=dev, generator=g) * 1e-3
    y = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    wsp = torch.empty(metis.metis_workspace_size(metis.METIS_OP_MOE, T, I, H, k, E),
                      dtype=torch.uint8, device=dev)
    ids_g = torch.empty_like(ids)
    w_g = torch.empty_like(w)
    t_r = timeit(lambda: metis.metis_moe_route_topk(logits, ids_g, w_g), 50)
    out["router_topk_4096tok_64e_top8"] = {"us": t_r * 1e6,
                                           "GB/s": (T * E * 4 + T * k * 8) / t_r / 1e9}
    t = timeit(lambda: metis.metis_moe_fp8_grouped_gemm(x, ids, w, wu, su, wd, sd, y, wsp), 20)
    tf = 2 * 2 * T * k * H * I / t / 1e12
    floor = moe_floor_us(T, H, I, E, k, hbm, peak8, fp4=False)
    load = torch.bincount(ids.flatten().long(), minlength=E).float()
    out["moe_4096tok_64e_top8"] = {"us": t * 1e6, "tok/s": T / t, "TFLOP/s": tf,
                                   "frac_of_fp8_peak": tf / peak8, "floor_us": floor,
                                   "frac_of_floor": floor / (t * 1e6),
                                   "hot_expert_load_ratio": float(load[:4].mean() / load.mean()),
                                   "rows_per_expert_min_max": [int(load.min()), int(load.max())]}
    # the layer with its shared expert (BF16, latent 1024): the routed layer
    # with y = NULL, then the shared expert with the routed combine fused into
    # its down-projection's epilogue
    Is = 1024
    wsu = (torch.randn(Is, H, device=dev, generator=g) * 0.03).to(torch.bfloat16)
    wsd = (torch.randn(H, Is, device=dev, generator=g) * 0.03).to(torch.bfloat16)
    wss = torch.empty(metis.metis_workspace_size(metis.METIS_OP_SHARED, T, Is, H, k, 0),
                      dtype=torch.uint8, device=dev)
    o_off = metis.metis_moe_workspace_offset("O", T, k, E, H, I)
    r_off = metis.metis_moe_workspace_offset("SLOT_TO_ROW", T, k, E, H, I)
    o_reg = wsp[o_off:].view(torch.bfloat16)
    s2r_reg = wsp[r_off:r_off + 4 * T * k].view(torch.int32)

    def shared():
        metis.metis_moe_shared_fused_combine(x, wsu, wsd, o_reg, s2r_reg, w, y, wss)

    def layer():
        metis.metis_moe_fp8_grouped_gemm(x, ids, w, wu, su, wd, sd, None, wsp)
        shared()
    hs = torch.empty(T, Is, dtype=torch.bfloat16, device=dev)
    t_l = timeit(layer, 20)
    t_s = timeit(shared, 20)
    t_g = timeit(lambda: metis.metis_bf16_gemm(x, wsu, hs), 20)
    out["moe_with_shared_4096tok_64e_top8"] = {
        "us": t_l * 1e6, "tok/s": T / t_l, "shared_fused_combine_us": t_s * 1e6,
        "bf16_gemm_4096x1024x2048_us": t_g * 1e6,
        "bf16_gemm_TFLOP/s": 2 * T * Is * H / t_g / 1e12,
        "bf16_gemm_frac_of_bf16_peak": 2 * T * Is * H / t_g / 1e12 / pk["bf16_tflops"]}
    del wu, wd, wsp, o_reg, s2r_reg
    # the same routed-expert layer with NVFP4 experts (E2M1 codes, E4M3 scale
    # per 16, FP32 scale per expert; inputs rounded to NVFP4 per token)
    peak4 = pk["bf16_tflops"] * FP4_PER_BF16

    def sf_codes(n):  # E4M3 scales 2^-3 .. 2^2, no NaN code
        return torch.randint(0x20, 0x48, (n,), dtype=torch.uint8, device=dev, generator=g)
    wu4 = torch.randint(0, 256, (E, I, H // 2), dtype=torch.uint8, device=dev, generator=g)
    wd4 = torch.randint(0, 256, (E, H, I // 2), dtype=torch.uint8, device=dev, generator=g)
    sfu, sfd = sf_codes(E * I * H // 16), sf_codes(E * H * I // 16)
    gu = torch.rand(E, device=dev, generator=g) * 1e-3 + 1e-4
    gd = torch.rand(E, device=dev, generator=g) * 1e-3 + 1e-4
    ws4 = torch.empty(metis.metis_workspace_size(metis.METIS_OP_MOE_NVFP4, T, I, H, k, E),
                      dtype=torch.uint8, device=dev)
    t = timeit(lambda: metis.metis_moe_nvfp4_grouped_gemm(x, ids, w, wu4, sfu, gu, wd4, sfd, gd,
                                                          y, ws4), 20)
    tf = 2 * 2 * T * k * H * I / t / 1e12
    floor = moe_floor_us(T, H, I, E, k, hbm, peak4, fp4=True)
    out["moe_nvfp4_4096tok_64e_top8"] = {"us": t * 1e6, "tok/s": T / t, "TFLOP/s": tf,
                                         "frac_of_fp4_peak": tf / peak4, "floor_us": floor,
                                         "frac_of_floor": floor / (t * 1e6)}
    del wu4, wd4, sfu, sfd, ws4
    # large-M W8A8 GEMM from BF16 activations (per-token magnitudes
    # log-uniform in [1e-2, 1e2]): the GEMM alone, the separate quantizer +
    # GEMM (the product path), and the fused-quantization variant
    for (M, K) in [(8192, 4096), (16384, 4096), (8192, 8192), (16384, 8192)]:
        mag = torch.exp(torch.empty(M, 1, device=dev).uniform_(-4.6052, 4.6052, generator=g))
        x = (torch.randn(M, K, device=dev, generator=g) * mag).to(torch.bfloat16)
        b = codes(K, K)
        sa = torch.empty(M, device=dev)
        sb = torch.rand(K, device=dev, generator=g)
        xq = torch.empty(M, K, dtype=torch.uint8, device=dev)
        y = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
        wsf = torch.empty(metis.metis_workspace_size(metis.METIS_OP_FP8_GEMM_FUSED, M, K, K, 0, 0),
                          dtype=torch.uint8, device=dev)
        metis.metis_quant_fp8_per_token(x, xq, sa)

        def separate():
            metis.metis_quant_fp8_per_token(x, xq, sa)
            metis.metis_fp8_gemm(xq, 0, sa, b, sb, y)
        fl = 2 * M * K * K
        t_g = timeit(lambda: metis.metis_fp8_gemm(xq, 0, sa, b, sb, y), 20)
        t_s = timeit(separate, 20)
        t_f = timeit(lambda: metis.metis_fp8_gemm(x, 1, sa, b, sb, y, workspace=wsf), 10)
        out[f"gemm_{M}x{K}x{K}"] = {
            "us": t_g * 1e6, "TFLOP/s": fl / t_g / 1e12, "frac_of_fp8_peak": fl / t_g / 1e12 / peak8,
            "frac_of_nominal_fp8": fl / t_g / 1e12 / NOMINAL_FP8_TFLOPS,
            "quant+gemm_us": t_s * 1e6, "quant+gemm_TFLOP/s": fl / t_s / 1e12,
            "fused_quant_us": t_f * 1e6, "fused_quant_TFLOP/s": fl / t_f / 1e12}
        del x, xq, b, y
    # the default maths for many tokens: the same 4096-token chain through
    # W8A16 (weights widened exactly to BF16), no quantizers. metis_linear
    # widens each layer's weights into the workspace and runs the BF16
    # CTA-pair GEMM; metis_w8a16_gemm widens them inside its kernel.
    T, K1, N1 = M_TOK, K_HID, N_FF
    xd = torch.randn(T, K1, device=dev, generator=g).to(torch.bfloat16)
    w1c, w2c = codes(N1, K1), codes(K1, N1)
    s1c = torch.rand(N1, device=dev, generator=g) * 1e-3
    s2c = torch.rand(K1, device=dev, generator=g) * 1e-3
    h1 = torch.empty(T, N1, dtype=torch.bfloat16, device=dev)
    h2 = torch.empty(T, K1, dtype=torch.bfloat16, device=dev)
    wsw = torch.empty(metis.metis_workspace_size(metis.METIS_OP_W8A16_WIDENED, T, N1, K1),
                      dtype=torch.uint8, device=dev)

    def chain16():
        metis.metis_linear(xd, w1c, s1c, h1, fast_math=False, workspace=wsw)
        metis.metis_linear(h1, w2c, s2c, h2, fast_math=False, workspace=wsw)

    def chain16_in_kernel():
        metis.metis_w8a16_gemm(xd, w1c, s1c, h1)
        metis.metis_w8a16_gemm(h1, w2c, s2c, h2)
    t = timeit(chain16, 10)
    t1 = timeit(lambda: metis.metis_linear(xd, w1c, s1c, h1, fast_math=False, workspace=wsw), 10)
    t_in = timeit(chain16_in_kernel, 10)
    fl = 2 * T * K1 * N1
    peak16 = pk["bf16_tflops"]
    out["prefill_default_maths_4096tok"] = {
        "us": t * 1e6, "tok/s": T / t, "TFLOP/s": 2 * fl / t / 1e12,
        "frac_of_bf16_peak": 2 * fl / t / 1e12 / peak16,
        "layer1_us": t1 * 1e6, "layer1_TFLOP/s": fl / t1 / 1e12,
        "in_kernel_widening_us": t_in * 1e6, "in_kernel_widening_TFLOP/s": 2 * fl / t_in / 1e12}
    del xd, w1c, w2c, h1, h2, wsw
    # dense NVFP4 GEMM (codes and tiled scales resident, 2 rotating B > L2 at the large size)
    for (M, K) in [(8192, 4096), (16384, 8192)]:
        qa = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=dev, generator=g)
        sa = sf_codes(M * K // 16)
        ga = torch.rand(M, device=dev, generator=g) + 0.5
        qb = torch.randint(0, 256, (K, K // 2), dtype=torch.uint8, device=dev, generator=g)
        sb = sf_codes(K * K // 16)
        gb = torch.ones(1, device=dev)
        y = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
        t = timeit(lambda: metis.metis_nvfp4_gemm(qa, sa, ga, qb, sb, gb, y), 20)
        fl = 2 * M * K * K
        out[f"nvfp4_gemm_{M}x{K}x{K}"] = {"us": t * 1e6, "TFLOP/s": fl / t / 1e12,
                                          "frac_of_fp4_peak": fl / t / 1e12 / peak4}
        del qa, sa, qb, sb, y
    return out


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_metis(args)


if __name__ == "__main__":
    sys.exit(main())
